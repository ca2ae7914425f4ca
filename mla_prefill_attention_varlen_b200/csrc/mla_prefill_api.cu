// Host side of libmla_prefill.so: argument validation, the per-GPU workspace,
// TMA tensor-map encoding and the two launches (plan kernel, attention kernel)
// behind the C ABI declared in include/mla_prefill.h.
#include <cuda.h>
#include <cublas_v2.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/mla_prefill.h"
#include "mla_prefill_pair_sm100.cuh"
#include "mla_prefill_sm100.cuh"
#include "paged_cache_load.cuh"
#include "prolog_norm_rope.cuh"
#include "prolog_q_sm100.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kVersion = 10000 * 0 + 100 * 1 + 0;

struct DeviceState {
    bool ready = false;
    int sm_count = 0;
    int *status = nullptr;  // sticky device status word (own 256-byte allocation)
    void *ws = nullptr;     // plan workspace
    size_t ws_bytes = 0;
    bool attr_set[32] = {};  // dynamic shared memory opt-in done, per kernel instantiation
    int pair_clusters = 0;   // co-resident clusters of two CTAs of the pair kernel (0: not yet queried)
    bool prolog_attr[4] = {};     // dynamic shared memory opt-in of the fused q-projection kernel, per d / 128 - 1
    int prolog_clusters[4] = {};  // its co-resident clusters (0: not yet queried)
};

std::mutex g_mu;
thread_local cudaEvent_t t_prof_start = nullptr, t_prof_stop = nullptr;
thread_local int t_split_tiles = -1;  // split-KV chunk in key tiles: -1 automatic, 0 off
thread_local int t_kernel = -1;       // attention kernel: -1 automatic, 1 single-CTA, 2 CTA pair
thread_local int t_prolog_path = -1;  // MLA Prolog q path: -1 automatic (fused where the sizes allow), 0 library
thread_local int t_prolog_fused = 0;  // the last mla_prolog call of this thread ran the fused q kernel
thread_local int t_last_launches = 0;  // kernels the last prefill call of this thread enqueued
thread_local int t_last_kernel = 0;    // attention kernel of that call: 1 single-CTA, 2 CTA pair
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Views of one input after validation, as [tokens, heads, width] with element strides.
struct View3 {
    void *data;
    int64_t tokens, heads, width;
    int64_t st_tok, st_head;
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Accepts [T, N, W] or [T, N*W]; the last dimension must be contiguous.
int view3(const mla_tensor *t, int dtype, int64_t heads, int64_t width, View3 *v) {
    if (!t) return MLA_ERR_NULL;
    if (!t->data && !(t->ndim >= 1 && t->ndim <= 4 && t->shape[0] == 0)) return MLA_ERR_NULL;
    if (t->dtype != dtype) return MLA_ERR_DTYPE;
    if (t->ndim == 3) {
        if (t->shape[1] != heads || t->shape[2] != width) return MLA_ERR_SHAPE;
        if (t->stride[2] != 1) return MLA_ERR_ALIGN;
        v->tokens = t->shape[0];
        v->st_tok = t->stride[0];
        v->st_head = t->stride[1];
    } else if (t->ndim == 2) {
        if (t->shape[1] != heads * width) return MLA_ERR_SHAPE;
        if (t->stride[1] != 1) return MLA_ERR_ALIGN;
        v->tokens = t->shape[0];
        v->st_tok = t->stride[0];
        v->st_head = width;
    } else {
        return MLA_ERR_SHAPE;
    }
    v->data = t->data;
    v->heads = heads;
    v->width = width;
    if (v->tokens < 0 || v->tokens > INT32_MAX) return MLA_ERR_SHAPE;
    if (v->data && !aligned16(v->data)) return MLA_ERR_ALIGN;
    if (v->tokens > 1 && (v->st_tok <= 0 || v->st_tok % 8 != 0)) return MLA_ERR_ALIGN;
    if (heads > 1 && (v->st_head <= 0 || v->st_head % 8 != 0)) return MLA_ERR_ALIGN;
    if (v->st_tok % 8 != 0 || v->st_head % 8 != 0) return MLA_ERR_ALIGN;
    if (v->st_tok * 2 >= (int64_t(1) << 40) || v->st_head * 2 >= (int64_t(1) << 40)) return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

// The padded [batch, max_seq, G*W] K/V form of the page: 3-D with a last dim of
// G*W and a middle extent other than G (G == 1 and max_seq == 1 read the same
// either way).
bool is_padded_kv(const mla_tensor *t, int64_t heads, int64_t width) {
    return t && t->ndim == 3 && t->shape[2] == heads * width && !(t->shape[1] == heads && t->shape[2] == width);
}

// A dense padded tensor [batch, max_seq, G*W] viewed as packed tokens
// [batch*max_seq, G, W]: sequence b's keys start at token b*max_seq.
int padded_view(const mla_tensor *t, int dtype, int64_t heads, int64_t width, int64_t batch, int64_t max_seq,
                View3 *v) {
    if (!t || (!t->data && t->shape[0] * t->shape[1] != 0)) return MLA_ERR_NULL;
    if (t->dtype != dtype) return MLA_ERR_DTYPE;
    if (t->shape[0] != batch || t->shape[1] != max_seq || t->shape[2] != heads * width) return MLA_ERR_SHAPE;
    if (t->stride[2] != 1) return MLA_ERR_ALIGN;
    if (batch > 1 && t->stride[0] != max_seq * t->stride[1]) return MLA_ERR_UNSUPPORTED;  // batch rows must be dense
    v->data = t->data;
    v->tokens = batch * max_seq;
    v->heads = heads;
    v->width = width;
    v->st_tok = t->stride[1];
    v->st_head = width;
    if (v->tokens > INT32_MAX) return MLA_ERR_SHAPE;
    if (v->data && !aligned16(v->data)) return MLA_ERR_ALIGN;
    if (v->st_tok % 8 != 0 || (v->tokens > 1 && v->st_tok < heads * width)) return MLA_ERR_ALIGN;
    if (v->st_tok * 2 >= (int64_t(1) << 40)) return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

// [lo, hi) byte range a view touches (for the no-alias check).
void byte_range(const View3 &v, uintptr_t *lo, uintptr_t *hi) {
    const uintptr_t base = reinterpret_cast<uintptr_t>(v.data);
    int64_t last = 0;
    if (v.tokens > 0) last = (v.tokens - 1) * v.st_tok + (v.heads - 1) * v.st_head + v.width;
    *lo = base;
    *hi = base + static_cast<uintptr_t>(last) * 2;
}

bool overlaps(const View3 &a, const View3 &b) {
    uintptr_t alo, ahi, blo, bhi;
    byte_range(a, &alo, &ahi);
    byte_range(b, &blo, &bhi);
    return alo < bhi && blo < ahi && ahi > alo && bhi > blo;
}

int ensure_encode() {
    if (g_encode) return MLA_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return MLA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return MLA_OK;
}

// 3-D map {width, heads, tokens} with a {64, 1, box_tokens} box and 128-byte swizzle.
int encode_map(CUtensorMap *m, const View3 &v, bool bf16, void *dummy, int box_tokens) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(v.width), static_cast<cuuint64_t>(v.heads),
                                static_cast<cuuint64_t>(v.tokens > 0 ? v.tokens : 1)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>((v.heads > 1 ? v.st_head : v.width) * 2),
                                   static_cast<cuuint64_t>((v.tokens > 1 ? v.st_tok : v.heads * v.width) * 2)};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_tokens)};
    const cuuint32_t estr[3] = {1, 1, 1};
    // An empty tensor is never read (no work item touches it); encode a valid dummy base.
    void *base = (v.tokens > 0 && v.data) ? v.data : dummy;
    CUresult r = g_encode(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base,
                          dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_UNSUPPORTED;
}

// 4-D map over a paged cache {channels, heads, slots, blocks} with a
// {64, 1, box_rows, 1} box and 128-byte swizzle.
int encode_cache_map(CUtensorMap *m, const void *data, int64_t blocks, int64_t slots, int64_t heads, int64_t channels,
                     int64_t block_bytes, int64_t slot_bytes, int64_t head_bytes, bool bf16, int box_rows) {
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(channels), static_cast<cuuint64_t>(heads),
                                static_cast<cuuint64_t>(slots), static_cast<cuuint64_t>(blocks)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(head_bytes), static_cast<cuuint64_t>(slot_bytes),
                                   static_cast<cuuint64_t>(block_bytes)};
    const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                          const_cast<void *>(data), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_UNSUPPORTED;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
    size_t status;  // offset of the per-call status word (caller-owned workspaces only)
    size_t seq_info, unit_off, hist, units, num_units, total;
    size_t split_off, entry_tab, part_lse, part_o;  // split-KV sections (empty without split)
    int hist_len;
    int split_tiles;
};

int64_t max_units_for(int64_t batch, int64_t t_q) { return (t_q + mla::kUnitRows - 1) / mla::kUnitRows + batch; }

// Upper bound of work-list entries when each unit's key tiles go in chunks of `split` (at most
// ceil(key_extent / 128) tiles per unit).
int64_t max_entries_for(int64_t max_units, int64_t key_extent, int split) {
    const int64_t tiles = (key_extent + mla::kBN - 1) / mla::kBN;
    return split > 0 ? max_units * ((tiles + split - 1) / split > 1 ? (tiles + split - 1) / split : 1) : max_units;
}

// t_k: key tokens of the K/V tensors; key_extent: the most keys one sequence can have;
// split: key tiles per split-KV chunk (0: none); heads: query heads; status_header: the first
// kWsHeaderBytes hold the call's status word (a caller-owned workspace).
constexpr size_t kWsHeaderBytes = 256;
WsLayout ws_layout(int64_t batch, int64_t t_q, int64_t t_k, int64_t key_extent = 0, int split = 0,
                   int64_t heads = 0, bool status_header = false) {
    WsLayout l;
    const int64_t max_units = max_units_for(batch, t_q);
    l.hist_len = static_cast<int>((t_k + mla::kBN - 1) / mla::kBN + 2);
    l.split_tiles = split;
    l.status = 0;
    size_t off = status_header ? kWsHeaderBytes : 0;
    l.num_units = off;
    off = align_up(off + 16, 256);
    l.seq_info = off;
    off = align_up(off + sizeof(int4) * batch, 256);
    l.unit_off = off;
    off = align_up(off + sizeof(int) * (batch + 1), 256);
    l.hist = off;
    off = align_up(off + sizeof(int) * l.hist_len, 256);
    l.units = off;
    off = align_up(off + sizeof(int2) * max_units, 256);
    l.split_off = l.entry_tab = l.part_lse = l.part_o = off;
    if (split > 0) {
        const int64_t entries = max_entries_for(max_units, key_extent, split);
        l.split_off = off;
        off = align_up(off + sizeof(int) * (max_units + 1), 256);
        l.entry_tab = off;
        off = align_up(off + sizeof(int2) * entries, 256);
        l.part_lse = off;
        off = align_up(off + sizeof(float) * entries * heads * mla::kUnitRows, 256);
        l.part_o = off;
        off = align_up(off + sizeof(float) * entries * heads * mla::kUnitRows * mla::kDn, 256);
    }
    l.total = off;
    return l;
}

int device_state(int dev, cudaStream_t stream, size_t ws_need, DeviceState **out) {
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    DeviceState &d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MLA_ERR_CUDA;
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (major != 10 || minor != 0) return MLA_ERR_UNSUPPORTED;  // built for sm_100a only
        if (cudaMalloc(&d.status, 256) != cudaSuccess) return MLA_ERR_CUDA;
        if (cudaMemset(d.status, 0, 256) != cudaSuccess) return MLA_ERR_CUDA;
        d.ready = true;
    }
    if (d.ws_bytes < ws_need) {
        // Stream-ordered: the old workspace is released behind the work already queued on this
        // stream and the new one is ready for the work queued next; the host never waits.
        if (d.ws) {
            if (cudaFreeAsync(d.ws, stream) != cudaSuccess) return MLA_ERR_CUDA;
            d.ws = nullptr;
            d.ws_bytes = 0;
        }
        const size_t bytes = align_up(ws_need, size_t(1) << 20);
        if (cudaMallocAsync(&d.ws, bytes, stream) != cudaSuccess) {
            d.ws = nullptr;
            return MLA_ERR_CUDA;
        }
        d.ws_bytes = bytes;
    }
    *out = &d;
    return MLA_OK;
}

template <typename T, bool kCausal, bool kPos, bool kGeneral>
int launch_attention(DeviceState *ds, int slot, int grid, cudaStream_t stream, const CUtensorMap (&maps)[5],
                     const mla::Params &p) {
    auto kern = mla::mla_prefill_sm100_kernel<T, kCausal, kPos, kGeneral>;
    if (!ds->attr_set[slot]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, mla::kSmemAlloc) != cudaSuccess)
            return MLA_ERR_CUDA;
        ds->attr_set[slot] = true;
    }
    if (t_prof_start && cudaEventRecord(t_prof_start, stream) != cudaSuccess) return MLA_ERR_CUDA;
    // programmatic dependent launch: the CTAs start (barriers, tensor memory) while the plan
    // kernel runs, and wait for it in the kernel before reading the work list
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(mla::kThreads);
    cfg.dynamicSmemBytes = mla::kSmemAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = t_prof_start ? 0 : 1;  // with the timing hook on, its events bracket this kernel alone
    if (cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4], p) != cudaSuccess)
        return MLA_ERR_CUDA;
    if (t_prof_stop && cudaEventRecord(t_prof_stop, stream) != cudaSuccess) return MLA_ERR_CUDA;
    return MLA_OK;
}

// The CTA-pair kernel: clusters of two CTAs, one per SM, persistent over the work list.
template <typename T, bool kCausal, bool kPos>
int launch_pair(DeviceState *ds, int slot, int64_t max_items, cudaStream_t stream, const CUtensorMap (&maps)[5],
                const mla::Params &p) {
    auto kern = mla::pair::mla_prefill_pair_kernel<T, kCausal, kPos>;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(mla::kThreads);
    cfg.dynamicSmemBytes = mla::pair::kSmemAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    if (!ds->attr_set[slot]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, mla::pair::kSmemAlloc) !=
            cudaSuccess)
            return MLA_ERR_CUDA;
        ds->attr_set[slot] = true;
    }
    if (ds->pair_clusters <= 0) {
        int n = 0;
        cfg.gridDim = dim3(2);
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return MLA_ERR_CUDA;
        ds->pair_clusters = n;
    }
    const int64_t clusters = max_items < ds->pair_clusters ? max_items : ds->pair_clusters;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
    cfg.numAttrs = t_prof_start ? 1 : 2;  // with the timing hook on, its events bracket this kernel alone
    if (t_prof_start && cudaEventRecord(t_prof_start, stream) != cudaSuccess) return MLA_ERR_CUDA;
    if (cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4], p) != cudaSuccess)
        return MLA_ERR_CUDA;
    if (t_prof_stop && cudaEventRecord(t_prof_stop, stream) != cudaSuccess) return MLA_ERR_CUDA;
    return MLA_OK;
}

// Everything a call needs after host-side validation.
struct Problem {
    View3 q, qr, k, kr, v, o;
    const int *q_seqlen, *kv_seqlen;
    int64_t batch;
    int64_t kv_pad;  // 0: packed K/V; else the padded layout's max_seq
    // paged K/V (mla_prefill_paged): caches [blocks, block_size, G, 192 | 128] and the block table
    bool paged = false;
    const void *key_cache = nullptr, *value_cache = nullptr;
    int64_t num_blocks = 0, block_size = 0, table_width = 0, table_stride = 0;
    int64_t kc_block = 0, kc_slot = 0, kc_head = 0, vc_block = 0, vc_slot = 0, vc_head = 0;
    const int *tables = nullptr;
    bool bf16, causal;
    int head_num, kv_head_num;
    float qk_scale;
};

// Arguments every prefill entry point shares: queries, output, seqlens, scalars.
int validate_common(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *q_seqlen,
                    const mla_tensor *kv_seqlen, int mask_type, int head_num, int kv_head_num, float qk_scale,
                    const mla_tensor *out, Problem *pr) {
    if (!q || !q_rope || !q_seqlen || !kv_seqlen || !out) return MLA_ERR_NULL;
    if (head_num < 1 || kv_head_num < 1 || head_num % kv_head_num != 0) return MLA_ERR_HEADS;
    if (mask_type != MLA_MASK_CAUSAL && mask_type != MLA_MASK_NONE) return MLA_ERR_UNSUPPORTED;
    if (!std::isfinite(qk_scale)) return MLA_ERR_UNSUPPORTED;
    const int dt = q->dtype;
    if (dt != MLA_BF16 && dt != MLA_F16) return MLA_ERR_DTYPE;

    if (q_seqlen->dtype != MLA_I32 || kv_seqlen->dtype != MLA_I32) return MLA_ERR_DTYPE;
    if (q_seqlen->ndim != 1 || kv_seqlen->ndim != 1 || q_seqlen->shape[0] != kv_seqlen->shape[0])
        return MLA_ERR_SHAPE;
    if (q_seqlen->shape[0] > 0 && (!q_seqlen->data || !kv_seqlen->data)) return MLA_ERR_NULL;
    if (q_seqlen->shape[0] > 1 && (q_seqlen->stride[0] != 1 || kv_seqlen->stride[0] != 1)) return MLA_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(q_seqlen->data) & 3u) || (reinterpret_cast<uintptr_t>(kv_seqlen->data) & 3u))
        return MLA_ERR_ALIGN;
    const int64_t batch = q_seqlen->shape[0];
    if (batch < 0 || batch > INT32_MAX / 2) return MLA_ERR_SHAPE;

    int rc;
    if ((rc = view3(q, dt, head_num, mla::kDn, &pr->q)) != MLA_OK) return rc;
    if ((rc = view3(q_rope, dt, head_num, mla::kDr, &pr->qr)) != MLA_OK) return rc;
    if ((rc = view3(out, dt, head_num, mla::kDn, &pr->o)) != MLA_OK) return rc;
    if (pr->qr.tokens != pr->q.tokens || pr->o.tokens != pr->q.tokens) return MLA_ERR_SHAPE;
    for (const View3 *in : {&pr->q, &pr->qr})
        if (overlaps(pr->o, *in)) return MLA_ERR_UNSUPPORTED;
    pr->q_seqlen = static_cast<const int *>(q_seqlen->data);
    pr->kv_seqlen = static_cast<const int *>(kv_seqlen->data);
    pr->batch = batch;
    pr->bf16 = dt == MLA_BF16;
    pr->causal = mask_type == MLA_MASK_CAUSAL;
    pr->head_num = head_num;
    pr->kv_head_num = kv_head_num;
    pr->qk_scale = qk_scale;
    return MLA_OK;
}

int validate(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *k, const mla_tensor *k_rope,
             const mla_tensor *v, const mla_tensor *q_seqlen, const mla_tensor *kv_seqlen, int mask_type,
             int head_num, int kv_head_num, float qk_scale, const mla_tensor *out, Problem *pr) {
    if (!k || !k_rope || !v) return MLA_ERR_NULL;
    int rc = validate_common(q, q_rope, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num, qk_scale, out, pr);
    if (rc != MLA_OK) return rc;
    const int dt = q->dtype;
    const int64_t batch = pr->batch;
    const bool pk = is_padded_kv(k, kv_head_num, mla::kDn), pkr = is_padded_kv(k_rope, kv_head_num, mla::kDr),
               pv = is_padded_kv(v, kv_head_num, mla::kDn);
    pr->kv_pad = 0;
    if (pk || pkr || pv) {
        if (!(pk && pkr && pv)) return MLA_ERR_UNSUPPORTED;  // all three padded, or none
        const int64_t max_seq = k->shape[1];
        if (max_seq < 1 || max_seq > INT32_MAX) return MLA_ERR_SHAPE;
        if ((rc = padded_view(k, dt, kv_head_num, mla::kDn, batch, max_seq, &pr->k)) != MLA_OK) return rc;
        if ((rc = padded_view(k_rope, dt, kv_head_num, mla::kDr, batch, max_seq, &pr->kr)) != MLA_OK) return rc;
        if ((rc = padded_view(v, dt, kv_head_num, mla::kDn, batch, max_seq, &pr->v)) != MLA_OK) return rc;
        pr->kv_pad = max_seq;
    } else {
        if ((rc = view3(k, dt, kv_head_num, mla::kDn, &pr->k)) != MLA_OK) return rc;
        if ((rc = view3(k_rope, dt, kv_head_num, mla::kDr, &pr->kr)) != MLA_OK) return rc;
        if ((rc = view3(v, dt, kv_head_num, mla::kDn, &pr->v)) != MLA_OK) return rc;
    }
    if (pr->kr.tokens != pr->k.tokens || pr->v.tokens != pr->k.tokens) return MLA_ERR_SHAPE;
    for (const View3 *in : {&pr->k, &pr->kr, &pr->v})
        if (overlaps(pr->o, *in)) return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

// Encodes the tensor maps and enqueues the plan and attention kernels.  `ws`
// holds the workspace described by `lay`; `launch_flags` records the
// per-instantiation shared-memory opt-in for the current GPU.
int enqueue(const Problem &pr, const WsLayout &lay, uint8_t *ws, int *status, int sm_count, DeviceState *launch_flags,
            cudaStream_t stream, bool reset_status = false) {
    int rc;
    if ((rc = ensure_encode()) != MLA_OK) return rc;
    const bool general = pr.paged || pr.kv_pad > 0 || lay.split_tiles > 0;  // padded / paged K/V or split-KV
    // The CTA-pair kernel serves packed, unsplit K/V.  Automatically it runs long sequences (on
    // average 3072 keys or more per sequence), where a 512-row unit walks many key tiles; short
    // units (a few key tiles each) run faster on the single-CTA kernel, whose per-unit start and
    // end cost less.  Either needs at least one work item per SM pair to pay off.
    // With an even number of query heads per kv head the pair kernel's two groups take two heads of
    // one kv head over the same 256 rows (both walk the same key tiles); else 512 rows of one head,
    // whose first 256 rows see fewer keys than the second.
    const bool head_pair = (pr.head_num / pr.kv_head_num) % 2 == 0;
    const int64_t pair_unit_rows = head_pair ? mla::pair::kGroupRows : mla::pair::kUnitRows;
    const int64_t pair_items = ((pr.q.tokens + pair_unit_rows - 1) / pair_unit_rows + pr.batch) *
                               (head_pair ? pr.head_num / 2 : pr.head_num);
    const bool long_keys = pr.batch > 0 && pr.k.tokens >= 3072 * pr.batch;
    const bool use_pair = !general && pair_items > 0 &&
                          (t_kernel == 2 || (t_kernel < 0 && long_keys && pair_items >= sm_count / 2));
    CUtensorMap maps[5];
    if ((rc = encode_map(&maps[0], pr.q, pr.bf16, ws, 128)) != MLA_OK) return rc;
    if ((rc = encode_map(&maps[1], pr.qr, pr.bf16, ws, 128)) != MLA_OK) return rc;
    const int rows_k = static_cast<int>(pr.block_size < mla::kBN ? pr.block_size : mla::kBN);
    const int rows_v = static_cast<int>(pr.block_size < 64 ? pr.block_size : 64);
    if (pr.paged) {
        const int64_t G = pr.kv_head_num;
        if ((rc = encode_cache_map(&maps[2], pr.key_cache, pr.num_blocks, pr.block_size, G, mla::kDn + mla::kDr,
                                   pr.kc_block, pr.kc_slot, pr.kc_head, pr.bf16, rows_k)) != MLA_OK)
            return rc;
        maps[3] = maps[2];
        if ((rc = encode_cache_map(&maps[4], pr.value_cache, pr.num_blocks, pr.block_size, G, mla::kDn,
                                   pr.vc_block, pr.vc_slot, pr.vc_head, pr.bf16, rows_v)) != MLA_OK)
            return rc;
    } else {
        // pair kernel: each CTA loads 32 keys of K per 64-key tile
        const int kbox = use_pair ? 32 : 128;
        if ((rc = encode_map(&maps[2], pr.k, pr.bf16, ws, kbox)) != MLA_OK) return rc;
        if ((rc = encode_map(&maps[3], pr.kr, pr.bf16, ws, kbox)) != MLA_OK) return rc;
        if ((rc = encode_map(&maps[4], pr.v, pr.bf16, ws, 64)) != MLA_OK) return rc;
    }

    int *num_units = reinterpret_cast<int *>(ws + lay.num_units);
    int *work_counter = num_units + 1;  // second word of the 16-byte header
    int *num_entries = num_units + 2;   // third word
    int *split_off = reinterpret_cast<int *>(ws + lay.split_off);
    int2 *entry_tab = reinterpret_cast<int2 *>(ws + lay.entry_tab);
    int4 *seq_info = reinterpret_cast<int4 *>(ws + lay.seq_info);
    int *unit_off = reinterpret_cast<int *>(ws + lay.unit_off);
    int *hist = reinterpret_cast<int *>(ws + lay.hist);
    int2 *units = reinterpret_cast<int2 *>(ws + lay.units);

    mla::mla_plan_kernel<<<1, mla::kPlanThreads, 0, stream>>>(
        pr.q_seqlen, pr.kv_seqlen, static_cast<int>(pr.batch), pr.q.tokens, pr.k.tokens, pr.kv_pad,
        pr.paged ? 1 : 0, pr.causal ? 1 : 0, seq_info, unit_off, hist, lay.hist_len, units, num_units, work_counter,
        lay.split_tiles, split_off, entry_tab, num_entries, status, reset_status ? 1 : 0,
        use_pair ? static_cast<int>(pair_unit_rows) : mla::kUnitRows);
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;

    mla::Params p;
    p.seq_info = seq_info;
    p.units = units;
    p.num_units = num_units;
    p.work_counter = work_counter;
    p.status = status;
    p.out = pr.o.data;
    p.out_st = pr.o.st_tok;
    p.out_sh = pr.o.st_head;
    p.out_v8 = (reinterpret_cast<uintptr_t>(pr.o.data) % 32 == 0) && (pr.o.st_tok * 2) % 32 == 0 &&
               (pr.o.st_head * 2) % 32 == 0;
    p.head_num = pr.head_num;
    p.group = pr.head_num / pr.kv_head_num;
    p.head_pair = use_pair && head_pair ? 1 : 0;
    // unit-major (longest-first) item order when all of K, K_rope and V fit in 48 MB of the L2
    p.lpt = !pr.paged && pr.k.tokens * pr.kv_head_num * (2 * mla::kDn + mla::kDr) * 2 <= (int64_t(48) << 20);
    p.scale_log2 = pr.qk_scale * 1.4426950408889634f;
    p.tables = pr.tables;
    p.table_stride = pr.table_stride;
    p.table_width = static_cast<int>(pr.table_width);
    p.num_blocks = static_cast<int>(pr.num_blocks);
    p.block_size = static_cast<int>(pr.block_size > 0 ? pr.block_size : 1);
    p.rows_k = rows_k > 0 ? rows_k : 1;
    p.rows_v = rows_v > 0 ? rows_v : 1;
    p.paged = pr.paged ? 1 : 0;
    p.split_tiles = lay.split_tiles;
    p.entry_tab = entry_tab;
    p.num_entries = num_entries;
    p.part_lse = reinterpret_cast<float *>(ws + lay.part_lse);
    p.part_o = reinterpret_cast<float *>(ws + lay.part_o);
    const bool pos = pr.qk_scale > 0.f;
    DeviceState *ls = launch_flags;
    if (use_pair) {
        const int slot = 16 + (pr.bf16 ? 0 : 4) + (pr.causal ? 0 : 2) + (pos ? 0 : 1);
#define MLA_PAIR(T, C, P) launch_pair<T, C, P>(ls, slot, pair_items, stream, maps, p)
        if (pr.bf16) {
            if (pr.causal) rc = pos ? MLA_PAIR(__nv_bfloat16, true, true) : MLA_PAIR(__nv_bfloat16, true, false);
            else rc = pos ? MLA_PAIR(__nv_bfloat16, false, true) : MLA_PAIR(__nv_bfloat16, false, false);
        } else {
            if (pr.causal) rc = pos ? MLA_PAIR(__half, true, true) : MLA_PAIR(__half, true, false);
            else rc = pos ? MLA_PAIR(__half, false, true) : MLA_PAIR(__half, false, false);
        }
#undef MLA_PAIR
        t_last_launches = 2;  // plan + attention
        t_last_kernel = 2;
        return rc;
    }

    const int64_t max_units = max_units_for(pr.batch, pr.q.tokens);
    const int64_t max_items =
        max_entries_for(max_units, pr.kv_pad > 0 ? pr.kv_pad : pr.k.tokens, lay.split_tiles) * pr.head_num;
    const int grid = static_cast<int>(max_items < sm_count ? max_items : sm_count);
    const int slot = (pr.bf16 ? 0 : 4) + (pr.causal ? 0 : 2) + (pos ? 0 : 1) + (general ? 8 : 0);
#define MLA_LAUNCH(T, C, P, G) launch_attention<T, C, P, G>(ls, slot, grid, stream, maps, p)
#define MLA_PICK(T, C, P) (general ? MLA_LAUNCH(T, C, P, true) : MLA_LAUNCH(T, C, P, false))
    if (pr.bf16) {
        if (pr.causal) rc = pos ? MLA_PICK(__nv_bfloat16, true, true) : MLA_PICK(__nv_bfloat16, true, false);
        else rc = pos ? MLA_PICK(__nv_bfloat16, false, true) : MLA_PICK(__nv_bfloat16, false, false);
    } else {
        if (pr.causal) rc = pos ? MLA_PICK(__half, true, true) : MLA_PICK(__half, true, false);
        else rc = pos ? MLA_PICK(__half, false, true) : MLA_PICK(__half, false, false);
    }
#undef MLA_PICK
#undef MLA_LAUNCH
    t_last_launches = 2;  // plan + attention
    t_last_kernel = 1;
    if (rc != MLA_OK || lay.split_tiles <= 0) return rc;
    t_last_launches = 3;  // + combine
    // split-KV: merge the chunks of every unit that has several
    mla::CombineParams c;
    c.seq_info = seq_info;
    c.units = units;
    c.num_units = num_units;
    c.split_off = split_off;
    c.part_o = p.part_o;
    c.part_lse = p.part_lse;
    c.out = pr.o.data;
    c.out_st = pr.o.st_tok;
    c.out_sh = pr.o.st_head;
    c.head_num = pr.head_num;
    const dim3 cgrid(static_cast<unsigned>(max_units), static_cast<unsigned>(pr.head_num), mla::kCombineRowGroups);
    if (pr.bf16) mla::mla_split_combine_kernel<__nv_bfloat16><<<cgrid, mla::kCombineThreads, 0, stream>>>(c);
    else mla::mla_split_combine_kernel<__half><<<cgrid, mla::kCombineThreads, 0, stream>>>(c);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// Split-KV chunk (key tiles) for a problem: the thread's override, else automatic -- only when the
// (unit, head) items cannot fill the GPU twice over and there are at least 16 key tiles of work per
// SM, in chunks that make about three items per SM.
// The fp32 partial rows are kept under 2 GiB.
int choose_split(const Problem &pr, int sm_count) {  // sm_count is read in automatic mode only
    const int64_t units = max_units_for(pr.batch, pr.q.tokens);
    const int64_t ext = pr.kv_pad > 0 ? pr.kv_pad : pr.k.tokens;
    const int64_t tiles = (ext + mla::kBN - 1) / mla::kBN;
    int64_t split = t_split_tiles;
    if (split < 0) {
        if (units * pr.head_num >= 2LL * sm_count) return 0;
        const int64_t work = pr.head_num * units * tiles / (pr.causal ? 2 : 1);  // key tiles, at most
        if (work < 16LL * sm_count) return 0;  // too little work to be worth a second kernel
        split = (work + 3LL * sm_count - 1) / (3LL * sm_count);
        if (split < 4) split = 4;
    }
    if (split <= 0) return 0;
    const auto bytes = [&](int64_t c) {
        return max_entries_for(units, ext, static_cast<int>(c)) * pr.head_num * mla::kUnitRows * (mla::kDn + 1) * 4;
    };
    while (split < tiles && bytes(split) > (int64_t(2) << 30)) split *= 2;
    return split >= tiles ? 0 : static_cast<int>(split);
}


// ---------------------------------------------------------------------------
// Allocation-free entry point.  Same validation and the same two kernels as
// mla_prefill, but the plan workspace and the status word live in one static
// device array of fixed size instead of library-allocated device memory.
// ---------------------------------------------------------------------------

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;               // 1 MiB on every GPU that loads the library
constexpr size_t kNoAllocStatusOffset = kNoAllocScratchBytes - 256;    // last 256 bytes: status word

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocDevice {
    bool ready = false;
    int sm_count = 0;
    uint8_t *scratch = nullptr;  // device address of g_noalloc_scratch on this GPU
    DeviceState launch;          // only its dynamic-shared-memory opt-in flags are used
};

NoAllocDevice g_noalloc[kMaxDevices];

// One-time set-up per GPU, with that GPU current: the array's device address
// (the host-side symbol is only a stand-in), the SM count, the arch check.
int noalloc_setup(int dev, NoAllocDevice **out) {
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    NoAllocDevice &d = g_noalloc[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MLA_ERR_CUDA;
        if (major != 10 || minor != 0) return MLA_ERR_UNSUPPORTED;
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MLA_ERR_CUDA;
        d.scratch = static_cast<uint8_t *>(ptr);
        d.ready = true;
    }
    *out = &d;
    return MLA_OK;
}

// Per-GPU facts for the caller-workspace entry points, gathered without allocating anything:
// the architecture check, the SM count, and the kernels' shared-memory opt-in flags.
struct LaunchInfo {
    bool ready = false;
    int sm_count = 0;
    DeviceState launch;  // only its dynamic-shared-memory opt-in flags are used
};
LaunchInfo g_launch_info[kMaxDevices];

int launch_info(int dev, LaunchInfo **out) {
    if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
    LaunchInfo &d = g_launch_info[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MLA_ERR_CUDA;
        if (major != 10 || minor != 0) return MLA_ERR_UNSUPPORTED;
        d.ready = true;
    }
    *out = &d;
    return MLA_OK;
}

// Validation and workspace layout shared by mla_prefill_get_workspace_size and mla_prefill_ws.
// The split-KV choice depends on the thread's split setting and, in automatic mode, on the SM
// count of the current GPU, so both calls must be made with the same settings on the same GPU.
int ws_problem(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *k, const mla_tensor *k_rope,
               const mla_tensor *v, const mla_tensor *q_seqlen, const mla_tensor *kv_seqlen, int mask_type,
               int head_num, int kv_head_num, float qk_scale, const mla_tensor *out, Problem *pr, WsLayout *lay,
               LaunchInfo **li) {
    int rc = validate(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num, qk_scale, out,
                      pr);
    if (rc != MLA_OK) return rc;
    *li = nullptr;
    int sm_count = 0;
    if (t_split_tiles < 0 && pr->batch > 0 && pr->q.tokens > 0) {  // automatic split: needs the SM count
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
        std::lock_guard<std::mutex> lock(g_mu);
        if ((rc = launch_info(dev, li)) != MLA_OK) return rc;
        sm_count = (*li)->sm_count;
    }
    const int split = (pr->batch > 0 && pr->q.tokens > 0) ? choose_split(*pr, sm_count) : 0;
    *lay = ws_layout(pr->batch, pr->q.tokens, pr->k.tokens, pr->kv_pad > 0 ? pr->kv_pad : pr->k.tokens, split,
                     pr->head_num, true);
    return MLA_OK;
}

}  // namespace

extern "C" {

int mla_prefill(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *k, const mla_tensor *k_rope,
                const mla_tensor *v, const mla_tensor *q_seqlen, const mla_tensor *kv_seqlen, int mask_type,
                int head_num, int kv_head_num, float qk_scale, mla_tensor *out, mla_stream_t stream_) {
    t_last_launches = 0;
    t_last_kernel = 0;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    Problem pr;
    int rc = validate(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num, qk_scale, out,
                      &pr);
    if (rc != MLA_OK) return rc;
    if (pr.batch == 0 || pr.q.tokens == 0) return MLA_OK;  // nothing to compute

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    DeviceState *ds = nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if ((rc = device_state(dev, stream, 0, &ds)) != MLA_OK) return rc;  // SM count
    const int split = choose_split(pr, ds->sm_count);
    const WsLayout lay = ws_layout(pr.batch, pr.q.tokens, pr.k.tokens, pr.kv_pad > 0 ? pr.kv_pad : pr.k.tokens,
                                   split, pr.head_num);
    if ((rc = device_state(dev, stream, lay.total, &ds)) != MLA_OK) return rc;
    return enqueue(pr, lay, static_cast<uint8_t *>(ds->ws), ds->status, ds->sm_count, ds, stream);
}

int mla_prefill_device_status(mla_stream_t stream_, int *status) {
    if (!status) return MLA_ERR_NULL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    // the library's word (mla_prefill and the other allocating entry points) and the word in the
    // static array of mla_prefill_noalloc: the first error of either is reported, both are cleared
    int *words[2] = {g_dev[dev].ready ? g_dev[dev].status : nullptr,
                     g_noalloc[dev].ready
                         ? reinterpret_cast<int *>(g_noalloc[dev].scratch + kNoAllocStatusOffset)
                         : nullptr};
    int first = MLA_OK;
    for (int *w : words) {
        if (!w) continue;
        int h = 0;
        if (cudaMemcpy(&h, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
        if (h != MLA_OK && cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
        if (first == MLA_OK) first = h;
    }
    *status = first;
    return MLA_OK;
}

int mla_prefill_get_workspace_size(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *k,
                                   const mla_tensor *k_rope, const mla_tensor *v, const mla_tensor *q_seqlen,
                                   const mla_tensor *kv_seqlen, int mask_type, int head_num, int kv_head_num,
                                   float qk_scale, const mla_tensor *out, uint64_t *workspace_bytes) {
    if (!workspace_bytes) return MLA_ERR_NULL;
    Problem pr;
    WsLayout lay;
    LaunchInfo *li;
    const int rc = ws_problem(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num,
                              qk_scale, out, &pr, &lay, &li);
    if (rc != MLA_OK) return rc;
    *workspace_bytes = lay.total;
    return MLA_OK;
}

int mla_prefill_ws(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *k, const mla_tensor *k_rope,
                   const mla_tensor *v, const mla_tensor *q_seqlen, const mla_tensor *kv_seqlen, int mask_type,
                   int head_num, int kv_head_num, float qk_scale, mla_tensor *out, void *workspace,
                   uint64_t workspace_bytes, mla_stream_t stream_) {
    t_last_launches = 0;
    t_last_kernel = 0;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    Problem pr;
    WsLayout lay;
    LaunchInfo *li;
    int rc = ws_problem(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num, qk_scale,
                        out, &pr, &lay, &li);
    if (rc != MLA_OK) return rc;
    if (!workspace) return MLA_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kWsHeaderBytes - 1)) || workspace_bytes < lay.total)
        return MLA_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int *status = reinterpret_cast<int *>(ws + lay.status);
    if (pr.batch == 0 || pr.q.tokens == 0)  // nothing to compute: the call's status is OK
        return cudaMemsetAsync(status, 0, sizeof(int), stream) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!li && (rc = launch_info(dev, &li)) != MLA_OK) return rc;
    return enqueue(pr, lay, ws, status, li->sm_count, &li->launch, stream, true);
}

int mla_prefill_ws_status(const void *workspace, mla_stream_t stream_, int *status) {
    if (!workspace || !status) return MLA_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(workspace) & (kWsHeaderBytes - 1)) return MLA_ERR_WORKSPACE;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MLA_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
    *status = h;
    return MLA_OK;
}

const char *mla_status_string(int status) {
    switch (status) {
        case MLA_OK: return "MLA_OK";
        case MLA_ERR_NULL: return "MLA_ERR_NULL: a required pointer is NULL";
        case MLA_ERR_DTYPE: return "MLA_ERR_DTYPE: unsupported or mismatched dtype";
        case MLA_ERR_SHAPE: return "MLA_ERR_SHAPE: inconsistent shapes";
        case MLA_ERR_ALIGN: return "MLA_ERR_ALIGN: misaligned pointer or stride";
        case MLA_ERR_HEADS: return "MLA_ERR_HEADS: invalid head_num / kv_head_num";
        case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: unsupported argument, layout or device";
        case MLA_ERR_CUDA: return "MLA_ERR_CUDA: a CUDA call failed";
        case MLA_ERR_SEQLEN: return "MLA_ERR_SEQLEN: seqlens inconsistent with tensor extents (clamped)";
        case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT: a device pipeline wait gave up";
        case MLA_ERR_INDEX: return "MLA_ERR_INDEX: a paged-cache block index was out of range (row zeroed)";
        case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: workspace smaller than required or not 256-byte aligned";
        default: return "unknown mla_status";
    }
}

int mla_selftest_wait_timeout(int wait_ms, mla_stream_t stream_) {
    if (wait_ms < 1 || wait_ms > 10000) return MLA_ERR_UNSUPPORTED;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    DeviceState *ds = nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    int rc;
    if ((rc = device_state(dev, stream, 0, &ds)) != MLA_OK) return rc;
    mla::mla_selftest_wait_kernel<<<1, 32, 0, stream>>>(ds->status, static_cast<unsigned long long>(wait_ms) * 1000000ull);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_prefill_last_launches(void) { return t_last_launches; }

int mla_prefill_last_kernel(void) { return t_last_kernel; }

int mla_prefill_set_kernel(int kernel) {
    if (kernel != -1 && kernel != 1 && kernel != 2) return MLA_ERR_UNSUPPORTED;
    t_kernel = kernel;
    return MLA_OK;
}

int mla_prefill_set_split_tiles(int tiles) {
    if (tiles < -1) return MLA_ERR_UNSUPPORTED;
    t_split_tiles = tiles;
    return MLA_OK;
}

int mla_prefill_set_profile_events(struct CUevent_st *start, struct CUevent_st *stop) {
    if (start && stop) {
        t_prof_start = reinterpret_cast<cudaEvent_t>(start);
        t_prof_stop = reinterpret_cast<cudaEvent_t>(stop);
    } else {
        t_prof_start = t_prof_stop = nullptr;
    }
    return MLA_OK;
}

int mla_prefill_version(void) { return kVersion; }

}  // extern "C"


extern "C" int mla_prefill_noalloc(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *k,
                                   const mla_tensor *k_rope, const mla_tensor *v, const mla_tensor *q_seqlen,
                                   const mla_tensor *kv_seqlen, int mask_type, int head_num, int kv_head_num,
                                   float qk_scale, mla_tensor *out, mla_stream_t stream_) {
    t_last_launches = 0;
    t_last_kernel = 0;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    Problem pr;
    int rc = validate(q, q_rope, k, k_rope, v, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num, qk_scale, out,
                      &pr);
    if (rc != MLA_OK) return rc;
    // The whole plan workspace must fit in the static array, ahead of the status word.
    const WsLayout lay = ws_layout(pr.batch, pr.q.tokens, pr.k.tokens);
    if (lay.total > kNoAllocStatusOffset) return MLA_ERR_UNSUPPORTED;
    if (pr.batch == 0 || pr.q.tokens == 0) return MLA_OK;  // nothing to compute

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    NoAllocDevice *nd = nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if ((rc = noalloc_setup(dev, &nd)) != MLA_OK) return rc;
    // Every entry the kernels read is rewritten by the plan kernel on each call
    // (including the zeroed histogram and work counter), so the array's previous
    // contents never leak into a result.
    return enqueue(pr, lay, nd->scratch, reinterpret_cast<int *>(nd->scratch + kNoAllocStatusOffset), nd->sm_count,
                   &nd->launch, stream);
}

// ---------------------------------------------------------------------------
// Paged KV-cache gather
// ---------------------------------------------------------------------------
namespace {

int elem_bytes(int dtype) {
    if (dtype == MLA_I8) return 1;
    if (dtype == MLA_F16 || dtype == MLA_BF16) return 2;
    return 0;
}

// A token-rows view: rows of `row_bytes` contiguous bytes, `stride` bytes apart.
struct Rows {
    uint8_t *data;
    int64_t count, row_bytes, stride;
};

// Output [T, H, D] or [T, H*D] with each token's H x D block contiguous.
int paged_output(const mla_tensor *t, int dtype, int64_t heads, int64_t dim, Rows *r) {
    if (!t) return MLA_ERR_NULL;
    if (t->dtype != dtype) return MLA_ERR_DTYPE;
    const int es = elem_bytes(dtype);
    if (t->ndim == 3) {
        if (t->shape[1] != heads || t->shape[2] != dim) return MLA_ERR_SHAPE;
        if (t->stride[2] != 1 || (heads > 1 && t->stride[1] != dim)) return MLA_ERR_ALIGN;
    } else if (t->ndim == 2) {
        if (t->shape[1] != heads * dim) return MLA_ERR_SHAPE;
        if (t->stride[1] != 1) return MLA_ERR_ALIGN;
    } else {
        return MLA_ERR_SHAPE;
    }
    r->count = t->shape[0];
    r->row_bytes = heads * dim * es;
    r->stride = t->stride[0] * es;
    r->data = static_cast<uint8_t *>(t->data);
    if (r->count < 0 || r->count > INT32_MAX) return MLA_ERR_SHAPE;
    if (r->count > 0 && !r->data) return MLA_ERR_NULL;
    if ((r->data && !aligned16(r->data)) || r->row_bytes % 16 != 0) return MLA_ERR_ALIGN;
    if (r->count > 1 && (r->stride % 16 != 0 || r->stride < r->row_bytes)) return MLA_ERR_ALIGN;
    return MLA_OK;
}

// Cache [num_blocks, block_size, H, D] with each slot's H x D block contiguous.
int paged_cache(const mla_tensor *t, int *dtype, int64_t *heads, int64_t *dim, int64_t *block_bytes,
                int64_t *slot_bytes) {
    if (!t || !t->data) return MLA_ERR_NULL;
    if (t->ndim != 4) return MLA_ERR_SHAPE;
    const int es = elem_bytes(t->dtype);
    if (!es) return MLA_ERR_DTYPE;
    *dtype = t->dtype;
    *heads = t->shape[2];
    *dim = t->shape[3];
    if (t->shape[0] < 1 || t->shape[1] < 1 || *heads < 1 || *dim < 1) return MLA_ERR_SHAPE;
    if (t->shape[0] > INT32_MAX) return MLA_ERR_SHAPE;
    if (t->stride[3] != 1 || (*heads > 1 && t->stride[2] != *dim)) return MLA_ERR_ALIGN;
    *block_bytes = t->stride[0] * es;
    *slot_bytes = t->stride[1] * es;
    const int64_t row = *heads * *dim * es;
    if (!aligned16(t->data) || row % 16 != 0 || *block_bytes % 16 != 0 || *slot_bytes % 16 != 0)
        return MLA_ERR_ALIGN;
    if (*slot_bytes < row || *block_bytes <= 0) return MLA_ERR_ALIGN;
    return MLA_OK;
}

bool rows_overlap(const Rows &r, const void *base, int64_t bytes) {
    if (r.count == 0 || bytes <= 0) return false;
    const uintptr_t lo = reinterpret_cast<uintptr_t>(r.data), hi = lo + (r.count - 1) * r.stride + r.row_bytes;
    const uintptr_t blo = reinterpret_cast<uintptr_t>(base), bhi = blo + bytes;
    return lo < bhi && blo < hi;
}

}  // namespace

extern "C" int mla_paged_cache_load(const mla_tensor *key_cache, const mla_tensor *value_cache,
                                    const mla_tensor *block_tables, const mla_tensor *context_lens,
                                    const mla_tensor *seq_starts, int context_lens_cumsum, mla_tensor *key,
                                    mla_tensor *value, mla_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (!key_cache || !value_cache || !block_tables || !context_lens || !key || !value) return MLA_ERR_NULL;
    int kdt, vdt, rc;
    int64_t H, Dk, Hv, Dv, kc_block, kc_slot, vc_block, vc_slot;
    if ((rc = paged_cache(key_cache, &kdt, &H, &Dk, &kc_block, &kc_slot)) != MLA_OK) return rc;
    if ((rc = paged_cache(value_cache, &vdt, &Hv, &Dv, &vc_block, &vc_slot)) != MLA_OK) return rc;
    if (value_cache->shape[0] != key_cache->shape[0] || value_cache->shape[1] != key_cache->shape[1] || Hv != H)
        return MLA_ERR_SHAPE;
    Rows ko, vo;
    if ((rc = paged_output(key, kdt, H, Dk, &ko)) != MLA_OK) return rc;
    if ((rc = paged_output(value, vdt, H, Dv, &vo)) != MLA_OK) return rc;
    if (ko.count != vo.count) return MLA_ERR_SHAPE;

    if (block_tables->dtype != MLA_I32 || context_lens->dtype != MLA_I32) return MLA_ERR_DTYPE;
    if (block_tables->ndim != 2 || context_lens->ndim != 1) return MLA_ERR_SHAPE;
    const int64_t batch = block_tables->shape[0], width = block_tables->shape[1];
    if (batch < 0 || batch > INT32_MAX / 2 || width < 0 || width > INT32_MAX) return MLA_ERR_SHAPE;
    if (context_lens->shape[0] != batch + (context_lens_cumsum ? 1 : 0)) return MLA_ERR_SHAPE;
    if (batch > 0 && (!block_tables->data || !context_lens->data)) return MLA_ERR_NULL;
    if (width > 1 && block_tables->stride[1] != 1) return MLA_ERR_ALIGN;
    if (batch > 1 && block_tables->stride[0] < width) return MLA_ERR_ALIGN;
    if (context_lens->shape[0] > 1 && context_lens->stride[0] != 1) return MLA_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(block_tables->data) & 3u) || (reinterpret_cast<uintptr_t>(context_lens->data) & 3u))
        return MLA_ERR_ALIGN;
    if (seq_starts) {
        if (seq_starts->dtype != MLA_I32) return MLA_ERR_DTYPE;
        if (seq_starts->ndim != 1 || seq_starts->shape[0] != batch) return MLA_ERR_SHAPE;
        if (batch > 0 && !seq_starts->data) return MLA_ERR_NULL;
        if (batch > 1 && seq_starts->stride[0] != 1) return MLA_ERR_ALIGN;
        if (reinterpret_cast<uintptr_t>(seq_starts->data) & 3u) return MLA_ERR_ALIGN;
    }
    const int64_t kc_bytes = (key_cache->shape[0] - 1) * kc_block + (key_cache->shape[1] - 1) * kc_slot + H * Dk *
                             elem_bytes(kdt);
    const int64_t vc_bytes = (value_cache->shape[0] - 1) * vc_block + (value_cache->shape[1] - 1) * vc_slot + H * Dv *
                             elem_bytes(vdt);
    if (rows_overlap(ko, key_cache->data, kc_bytes) || rows_overlap(ko, value_cache->data, vc_bytes) ||
        rows_overlap(vo, key_cache->data, kc_bytes) || rows_overlap(vo, value_cache->data, vc_bytes) ||
        rows_overlap(ko, vo.data, vo.count > 0 ? (vo.count - 1) * vo.stride + vo.row_bytes : 0))
        return MLA_ERR_UNSUPPORTED;
    if (batch == 0 || ko.count == 0) return MLA_OK;  // nothing to copy

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    DeviceState *ds = nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if ((rc = device_state(dev, stream, align_up(sizeof(int) * (batch + 1), 256), &ds)) != MLA_OK) return rc;
    int *offs = static_cast<int *>(ds->ws);
    mla::paged_plan_kernel<<<1, mla::kPagedPlanThreads, 0, stream>>>(
        static_cast<const int *>(context_lens->data), static_cast<int>(batch), context_lens_cumsum ? 1 : 0, ko.count,
        offs, ds->status);
    if (cudaGetLastError() != cudaSuccess) return MLA_ERR_CUDA;

    mla::GatherParams p;
    p.key_cache = static_cast<const uint8_t *>(key_cache->data);
    p.value_cache = static_cast<const uint8_t *>(value_cache->data);
    p.kc_block = kc_block;
    p.kc_slot = kc_slot;
    p.vc_block = vc_block;
    p.vc_slot = vc_slot;
    p.key_row = static_cast<int>(ko.row_bytes);
    p.value_row = static_cast<int>(vo.row_bytes);
    p.key = ko.data;
    p.value = vo.data;
    p.key_tok = ko.stride;
    p.value_tok = vo.stride;
    p.tables = static_cast<const int *>(block_tables->data);
    p.table_stride = batch > 1 ? block_tables->stride[0] : width;
    p.width = static_cast<int>(width);
    p.num_blocks = static_cast<int>(key_cache->shape[0]);
    p.block_size = static_cast<int>(key_cache->shape[1]);
    p.starts = seq_starts ? static_cast<const int *>(seq_starts->data) : nullptr;
    p.offs = offs;
    p.batch = static_cast<int>(batch);
    p.status = ds->status;
    const int64_t rows = ko.count;
    const int64_t want = (rows + mla::kGatherThreads / 32 - 1) / (mla::kGatherThreads / 32);
    const int64_t cap = static_cast<int64_t>(ds->sm_count) * 8;
    const int grid = static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
    mla::paged_gather_kernel<<<grid, mla::kGatherThreads, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Prefill reading K / K_rope / V in place from paged caches
// ---------------------------------------------------------------------------
namespace {

// A [blocks, block_size, G, W] cache of the query dtype, read by 4-D TMA maps.
int attention_cache(const mla_tensor *t, int dtype, int64_t heads, int64_t width, int64_t *blocks,
                    int64_t *block_size, int64_t *bb, int64_t *sb, int64_t *hb) {
    if (!t || !t->data) return MLA_ERR_NULL;
    if (t->dtype != dtype) return MLA_ERR_DTYPE;
    if (t->ndim != 4 || t->shape[2] != heads || t->shape[3] != width) return MLA_ERR_SHAPE;
    if (t->shape[0] < 1 || t->shape[0] > INT32_MAX || t->shape[1] < 1) return MLA_ERR_SHAPE;
    if (t->stride[3] != 1) return MLA_ERR_ALIGN;
    *blocks = t->shape[0];
    *block_size = t->shape[1];
    *bb = t->stride[0] * 2;
    *sb = t->stride[1] * 2;
    *hb = (heads > 1 ? t->stride[2] : width) * 2;
    if (!aligned16(t->data) || *bb % 16 || *sb % 16 || *hb % 16 || *bb <= 0 || *sb <= 0 || *hb <= 0)
        return MLA_ERR_ALIGN;
    if (*bb >= (int64_t(1) << 40) || *sb >= (int64_t(1) << 40) || *hb >= (int64_t(1) << 40))
        return MLA_ERR_UNSUPPORTED;
    return MLA_OK;
}

}  // namespace

extern "C" int mla_prefill_paged(const mla_tensor *q, const mla_tensor *q_rope, const mla_tensor *key_cache,
                                 const mla_tensor *value_cache, const mla_tensor *block_tables,
                                 const mla_tensor *q_seqlen, const mla_tensor *kv_seqlen, int mask_type, int head_num,
                                 int kv_head_num, float qk_scale, mla_tensor *out, mla_stream_t stream_) {
    t_last_launches = 0;
    t_last_kernel = 0;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (!key_cache || !value_cache || !block_tables) return MLA_ERR_NULL;
    Problem pr;
    int rc = validate_common(q, q_rope, q_seqlen, kv_seqlen, mask_type, head_num, kv_head_num, qk_scale, out, &pr);
    if (rc != MLA_OK) return rc;
    const int dt = q->dtype;
    int64_t nb, bs, nbv, bsv;
    if ((rc = attention_cache(key_cache, dt, kv_head_num, mla::kDn + mla::kDr, &nb, &bs, &pr.kc_block, &pr.kc_slot,
                              &pr.kc_head)) != MLA_OK)
        return rc;
    if ((rc = attention_cache(value_cache, dt, kv_head_num, mla::kDn, &nbv, &bsv, &pr.vc_block, &pr.vc_slot,
                              &pr.vc_head)) != MLA_OK)
        return rc;
    if (nbv != nb || bsv != bs) return MLA_ERR_SHAPE;
    // a block holds whole 8-row swizzle atoms, and a 128-key tile covers whole blocks (or lies in one)
    if (bs % 8 != 0 || (bs <= mla::kBN ? mla::kBN % bs != 0 : bs % mla::kBN != 0)) return MLA_ERR_UNSUPPORTED;
    if (block_tables->dtype != MLA_I32) return MLA_ERR_DTYPE;
    if (block_tables->ndim != 2 || block_tables->shape[0] != pr.batch) return MLA_ERR_SHAPE;
    const int64_t width = block_tables->shape[1];
    if (width < 0 || width * bs > INT32_MAX) return MLA_ERR_SHAPE;
    if (pr.batch > 0 && width > 0 && !block_tables->data) return MLA_ERR_NULL;
    if (width > 1 && block_tables->stride[1] != 1) return MLA_ERR_ALIGN;
    if (pr.batch > 1 && block_tables->stride[0] < width) return MLA_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(block_tables->data) & 3u) return MLA_ERR_ALIGN;
    // out must not overlap the caches
    uintptr_t olo, ohi;
    byte_range(pr.o, &olo, &ohi);
    const uintptr_t klo = reinterpret_cast<uintptr_t>(key_cache->data),
                    khi = klo + (nb - 1) * pr.kc_block + (bs - 1) * pr.kc_slot + (kv_head_num - 1) * pr.kc_head + 384;
    const uintptr_t vlo = reinterpret_cast<uintptr_t>(value_cache->data),
                    vhi = vlo + (nb - 1) * pr.vc_block + (bs - 1) * pr.vc_slot + (kv_head_num - 1) * pr.vc_head + 256;
    if ((olo < khi && klo < ohi) || (olo < vhi && vlo < ohi)) return MLA_ERR_UNSUPPORTED;

    pr.paged = true;
    pr.key_cache = key_cache->data;
    pr.value_cache = value_cache->data;
    pr.num_blocks = nb;
    pr.block_size = bs;
    pr.table_width = width;
    pr.table_stride = pr.batch > 1 ? block_tables->stride[0] : width;
    pr.tables = static_cast<const int *>(block_tables->data);
    pr.kv_pad = width * bs;  // per-sequence key capacity of the table
    pr.k.tokens = width * bs;
    if (pr.batch == 0 || pr.q.tokens == 0) return MLA_OK;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    DeviceState *ds = nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if ((rc = device_state(dev, stream, 0, &ds)) != MLA_OK) return rc;  // SM count
    const int split = choose_split(pr, ds->sm_count);
    const WsLayout lay = ws_layout(pr.batch, pr.q.tokens, pr.k.tokens, pr.kv_pad > 0 ? pr.kv_pad : pr.k.tokens,
                                   split, pr.head_num);
    if ((rc = device_state(dev, stream, lay.total, &ds)) != MLA_OK) return rc;
    return enqueue(pr, lay, static_cast<uint8_t *>(ds->ws), ds->status, ds->sm_count, ds, stream);
}

// ---------------------------------------------------------------------------
// MLA Prolog: the three projections as library GEMMs (bf16 operands, fp32
// results), then the RmsNorm / RoPE rows of prolog_norm_rope.cuh
// ---------------------------------------------------------------------------
namespace {

constexpr int64_t kPrologSlab = 4096;  // tokens per pass: bounds the fp32 scratch
cublasHandle_t g_blas[kMaxDevices] = {};

// A 2-D bf16 matrix [rows, cols] with a contiguous last dimension and a row stride that is a
// multiple of 8 elements (16 bytes).  want_rows / want_cols < 0 accept any extent.
struct Mat {
    void *data;
    int64_t rows, cols, ld;
};

int mat2(const mla_tensor *t, int64_t want_rows, int64_t want_cols, Mat *m) {
    if (!t) return MLA_ERR_NULL;
    if (t->dtype != MLA_BF16) return MLA_ERR_DTYPE;
    if (t->ndim != 2) return MLA_ERR_SHAPE;
    if ((want_rows >= 0 && t->shape[0] != want_rows) || (want_cols >= 0 && t->shape[1] != want_cols))
        return MLA_ERR_SHAPE;
    if (t->shape[0] < 0 || t->shape[1] < 1 || t->shape[0] > INT32_MAX || t->shape[1] > INT32_MAX)
        return MLA_ERR_SHAPE;
    if (t->shape[0] > 0 && !t->data) return MLA_ERR_NULL;
    if (t->shape[1] > 1 && t->stride[1] != 1) return MLA_ERR_ALIGN;
    const int64_t ld = t->shape[0] > 1 ? t->stride[0] : t->shape[1];
    if (ld < t->shape[1] || ld % 8 || ld > INT32_MAX || !aligned16(t->data)) return MLA_ERR_ALIGN;
    *m = Mat{t->data, t->shape[0], t->shape[1], ld};
    return MLA_OK;
}

int vec1(const mla_tensor *t, int64_t n, const void **p) {
    if (!t || !t->data) return MLA_ERR_NULL;
    if (t->dtype != MLA_BF16) return MLA_ERR_DTYPE;
    if (t->ndim != 1 || t->shape[0] != n) return MLA_ERR_SHAPE;
    if (n > 1 && t->stride[0] != 1) return MLA_ERR_ALIGN;
    if (!aligned16(t->data)) return MLA_ERR_ALIGN;
    *p = t->data;
    return MLA_OK;
}

struct Range {
    uintptr_t lo, hi;
};
Range mat_range(const Mat &m) {
    const uintptr_t lo = reinterpret_cast<uintptr_t>(m.data);
    return Range{lo, m.rows > 0 ? lo + static_cast<uintptr_t>(((m.rows - 1) * m.ld + m.cols) * 2) : lo};
}
Range view_range(const View3 &v) {
    Range r;
    byte_range(v, &r.lo, &r.hi);
    return r;
}
bool ranges_overlap(const Range &a, const Range &b) { return a.lo < b.hi && b.lo < a.hi; }

// C[M, N] (fp32, row stride ldc) = A[M, K] B[K, N] (bf16, row-major): the column-major library
// call computes C^T = B^T A^T.
int gemm_rowmajor(cublasHandle_t h, int64_t M, int64_t N, int64_t K, const void *A, int64_t lda, const void *B,
                  int64_t ldb, float *C, int64_t ldc) {
    const float one = 1.f, zero = 0.f;
    const cublasStatus_t s =
        cublasGemmEx(h, CUBLAS_OP_N, CUBLAS_OP_N, static_cast<int>(N), static_cast<int>(M), static_cast<int>(K), &one,
                     B, CUDA_R_16BF, static_cast<int>(ldb), A, CUDA_R_16BF, static_cast<int>(lda), &zero, C,
                     CUDA_R_32F, static_cast<int>(ldc), CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
    return s == CUBLAS_STATUS_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// 2-D map over a bf16 matrix {cols, rows} (row stride row_bytes) with a {64, box_rows} box and
// 128-byte swizzle.
int encode_map2d(CUtensorMap *m, const void *base, int64_t cols, int64_t rows, int64_t row_bytes, int box_rows) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_UNSUPPORTED;
}

// q_out rows of a slab {d, H, tokens} for the fused q kernel's TMA stores: a {32, 1, 128} box with
// 64-byte swizzle (its staging buffers' layout).
int encode_out_map(CUtensorMap *m, const View3 &v) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(v.width), static_cast<cuuint64_t>(v.heads),
                                static_cast<cuuint64_t>(v.tokens)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>((v.heads > 1 ? v.st_head : v.width) * 2),
                                   static_cast<cuuint64_t>((v.tokens > 1 ? v.st_tok : v.heads * v.width) * 2)};
    const cuuint32_t box[3] = {32, 1, 128};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v.data, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_UNSUPPORTED;
}

// The fused q projection + per-head RmsNorm + RoPE (prolog_q_sm100.cuh): clusters of two CTAs, one
// per SM, static tiles of 256 tokens x one head; one instantiation per head size.
template <int kD>
int launch_prolog_q_d(DeviceState *ds, cudaStream_t stream, const CUtensorMap &tm_a, const CUtensorMap &tm_b,
                      const CUtensorMap &tm_o, const mla::prolog::QParams &qp) {
    constexpr int di = kD / 128 - 1;
    auto kern = mla::prolog::mla_prolog_q_kernel<kD>;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(mla::prolog::kThreads);
    cfg.dynamicSmemBytes = mla::prolog::kSmemAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (!ds->prolog_attr[di]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, mla::prolog::kSmemAlloc) !=
            cudaSuccess)
            return MLA_ERR_CUDA;
        ds->prolog_attr[di] = true;
    }
    if (ds->prolog_clusters[di] <= 0) {
        int n = 0;
        cfg.gridDim = dim3(2);
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return MLA_ERR_CUDA;
        ds->prolog_clusters[di] = n;
    }
    const int64_t tiles = static_cast<int64_t>((qp.tokens + mla::prolog::kTileTokens - 1) / mla::prolog::kTileTokens) *
                          qp.heads;
    const int64_t clusters = tiles < ds->prolog_clusters[di] ? tiles : ds->prolog_clusters[di];
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
    if (cudaLaunchKernelEx(&cfg, kern, tm_a, tm_b, tm_o, qp) != cudaSuccess) return MLA_ERR_CUDA;
    return MLA_OK;
}

int launch_prolog_q(DeviceState *ds, cudaStream_t stream, const CUtensorMap &tm_a, const CUtensorMap &tm_b,
                    const CUtensorMap &tm_o, const mla::prolog::QParams &qp) {
    switch (qp.d) {
        case 128: return launch_prolog_q_d<128>(ds, stream, tm_a, tm_b, tm_o, qp);
        case 256: return launch_prolog_q_d<256>(ds, stream, tm_a, tm_b, tm_o, qp);
        case 384: return launch_prolog_q_d<384>(ds, stream, tm_a, tm_b, tm_o, qp);
        case 512: return launch_prolog_q_d<512>(ds, stream, tm_a, tm_b, tm_o, qp);
        default: return MLA_ERR_UNSUPPORTED;
    }
}

int launch_norm(const mla::NormParams &np, int sm_count, cudaStream_t stream) {
    const long long rows = np.job[0].rows + (np.njobs > 1 ? np.job[1].rows : 0);
    if (rows == 0) return MLA_OK;
    const long long want = (rows + mla::kNormThreads / 32 - 1) / (mla::kNormThreads / 32);
    const long long cap = static_cast<long long>(sm_count) * 8;
    mla::rms_norm_rope_kernel<<<static_cast<int>(want < cap ? want : cap), mla::kNormThreads, 0, stream>>>(np);
    return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

extern "C" int mla_prolog(const mla_tensor *token_x, const mla_tensor *wq_a, const mla_tensor *wq_b,
                          const mla_tensor *wkv, const mla_tensor *rope_cos, const mla_tensor *rope_sin,
                          const mla_tensor *gamma_cq, const mla_tensor *gamma_ckv, int num_heads, float eps,
                          mla_tensor *q_out, mla_tensor *kv_out, mla_tensor *cq_out, mla_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (!q_out || !kv_out) return MLA_ERR_NULL;
    if (num_heads < 1) return MLA_ERR_HEADS;
    if (!std::isfinite(eps) || eps < 0.f) return MLA_ERR_UNSUPPORTED;
    int rc;
    Mat x, wa, wb, wk, cs, sn, kvo, cqo{};
    if ((rc = mat2(token_x, -1, -1, &x)) != MLA_OK) return rc;
    const int64_t t = x.rows, h = x.cols;
    if ((rc = mat2(wq_a, h, -1, &wa)) != MLA_OK) return rc;
    if ((rc = mat2(wkv, h, -1, &wk)) != MLA_OK) return rc;
    const int64_t r = wa.cols, d = wk.cols, H = num_heads;
    if (H * d > INT32_MAX) return MLA_ERR_SHAPE;
    if ((rc = mat2(wq_b, r, H * d, &wb)) != MLA_OK) return rc;
    if ((rc = mat2(rope_cos, t, -1, &cs)) != MLA_OK) return rc;
    const int64_t R = cs.cols;
    if ((rc = mat2(rope_sin, t, R, &sn)) != MLA_OK) return rc;
    if (r % 4 || d % 4 || R % 4 || R > d) return MLA_ERR_UNSUPPORTED;  // rows move in groups of 4 channels
    const void *g_cq, *g_ckv;
    if ((rc = vec1(gamma_cq, r, &g_cq)) != MLA_OK) return rc;
    if ((rc = vec1(gamma_ckv, d, &g_ckv)) != MLA_OK) return rc;
    View3 qo;
    if ((rc = view3(q_out, MLA_BF16, H, d, &qo)) != MLA_OK) return rc;
    if (qo.tokens != t) return MLA_ERR_SHAPE;
    if ((rc = mat2(kv_out, t, d, &kvo)) != MLA_OK) return rc;
    if (cq_out && (rc = mat2(cq_out, t, r, &cqo)) != MLA_OK) return rc;
    // outputs overlap neither each other nor any input
    const Range outs[3] = {view_range(qo), mat_range(kvo), cq_out ? mat_range(cqo) : Range{0, 0}};
    const Range ins[6] = {mat_range(x), mat_range(wa), mat_range(wb), mat_range(wk), mat_range(cs), mat_range(sn)};
    for (int i = 0; i < 3; ++i) {
        for (int k = i + 1; k < 3; ++k)
            if (ranges_overlap(outs[i], outs[k])) return MLA_ERR_UNSUPPORTED;
        for (const Range &in : ins)
            if (ranges_overlap(outs[i], in)) return MLA_ERR_UNSUPPORTED;
    }
    if (t == 0) return MLA_OK;

    // The q projection runs fused with its norm and rotation (prolog_q_sm100.cuh) where the sizes fit
    // the kernel's tiles: head_dim a multiple of 128 up to 512 (the accumulator of a head row in
    // tensor memory), q_lora_rank a multiple of 64 (its k-stages), rope_dim a multiple of 32 (the
    // epilogue's column chunks are rotated whole).
    const bool fused = t_prolog_path != 0 && d % 128 == 0 && d <= 512 && r % 64 == 0 && R % 32 == 0;
    // scratch per slab: [S, r + d] fp32 (x wq_a | x wkv), [S, H d] fp32 (c^Q wq_b; library path
    // only), [S, r] bf16 c^Q
    const int64_t slab = t < kPrologSlab ? t : kPrologSlab;
    const size_t pre_bytes = align_up(static_cast<size_t>(slab * (r + d)) * 4, 256);
    const size_t q_bytes = fused ? 0 : align_up(static_cast<size_t>(slab * H * d) * 4, 256);
    const size_t cq_bytes = cq_out ? 0 : align_up(static_cast<size_t>(slab * r) * 2, 256);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState *ds = nullptr;
    if ((rc = device_state(dev, stream, pre_bytes + q_bytes + cq_bytes, &ds)) != MLA_OK) return rc;
    if (!g_blas[dev] && cublasCreate(&g_blas[dev]) != CUBLAS_STATUS_SUCCESS) {
        g_blas[dev] = nullptr;
        return MLA_ERR_CUDA;
    }
    cublasHandle_t bl = g_blas[dev];
    if (cublasSetStream(bl, stream) != CUBLAS_STATUS_SUCCESS) return MLA_ERR_CUDA;
    uint8_t *ws = static_cast<uint8_t *>(ds->ws);
    float *pre = reinterpret_cast<float *>(ws);
    float *qpre = reinterpret_cast<float *>(ws + pre_bytes);
    __nv_bfloat16 *cq_scratch = reinterpret_cast<__nv_bfloat16 *>(ws + pre_bytes + q_bytes);
    const auto bf = [](const void *p, int64_t elems) {
        return reinterpret_cast<__nv_bfloat16 *>(const_cast<uint8_t *>(static_cast<const uint8_t *>(p)) + elems * 2);
    };
    CUtensorMap tm_b;
    if (fused) {
        if ((rc = ensure_encode()) != MLA_OK) return rc;
        if ((rc = encode_map2d(&tm_b, wb.data, H * d, r, wb.ld * 2, 64)) != MLA_OK) return rc;
    }
    t_prolog_fused = fused ? 1 : 0;

    for (int64_t s0 = 0; s0 < t; s0 += slab) {
        const int64_t S = t - s0 < slab ? t - s0 : slab;
        const void *xs = bf(x.data, s0 * x.ld);
        // x wq_a -> pre[:, 0:r],  x wkv -> pre[:, r:r+d]
        if ((rc = gemm_rowmajor(bl, S, r, h, xs, x.ld, wa.data, wa.ld, pre, r + d)) != MLA_OK) return rc;
        if ((rc = gemm_rowmajor(bl, S, d, h, xs, x.ld, wk.data, wk.ld, pre + r, r + d)) != MLA_OK) return rc;
        __nv_bfloat16 *cq = cq_out ? bf(cqo.data, s0 * cqo.ld) : cq_scratch;
        const int64_t cq_ld = cq_out ? cqo.ld : r;
        mla::NormParams np{};
        np.eps = eps;
        np.njobs = 2;
        np.job[0] = mla::NormJob{pre, r + d, cq, cq_ld, 0, static_cast<const __nv_bfloat16 *>(g_cq), nullptr,
                                 nullptr, 0, 0, static_cast<int>(r), 0, 1, S};
        np.job[1] = mla::NormJob{pre + r, r + d, bf(kvo.data, s0 * kvo.ld), kvo.ld, 0,
                                 static_cast<const __nv_bfloat16 *>(g_ckv), bf(cs.data, s0 * cs.ld),
                                 bf(sn.data, s0 * sn.ld), cs.ld, sn.ld, static_cast<int>(d), static_cast<int>(R), 1,
                                 S};
        if ((rc = launch_norm(np, ds->sm_count, stream)) != MLA_OK) return rc;
        if (fused) {
            // c^Q wq_b with the per-head RmsNorm and rope as the epilogue, straight into q_out
            CUtensorMap tm_a, tm_o;
            if ((rc = encode_map2d(&tm_a, cq, r, S, cq_ld * 2, 128)) != MLA_OK) return rc;
            View3 qs = qo;  // this slab's rows of q_out
            qs.data = bf(qo.data, s0 * qo.st_tok);
            qs.tokens = S;
            if ((rc = encode_out_map(&tm_o, qs)) != MLA_OK) return rc;
            mla::prolog::QParams qp{};
            qp.cos = bf(cs.data, s0 * cs.ld);
            qp.sin = bf(sn.data, s0 * sn.ld);
            qp.cos_tok = cs.ld;
            qp.sin_tok = sn.ld;
            qp.tokens = static_cast<int>(S);
            qp.heads = static_cast<int>(H);
            qp.d = static_cast<int>(d);
            qp.nc = d % 256 == 0 ? 256 : 128;
            qp.rope = static_cast<int>(R);
            qp.k_stages = static_cast<int>(r / 64);
            qp.eps = eps;
            qp.status = ds->status;
            if (t_prof_start && cudaEventRecord(t_prof_start, stream) != cudaSuccess) return MLA_ERR_CUDA;
            if ((rc = launch_prolog_q(ds, stream, tm_a, tm_b, tm_o, qp)) != MLA_OK) return rc;
            if (t_prof_stop && cudaEventRecord(t_prof_stop, stream) != cudaSuccess) return MLA_ERR_CUDA;
            continue;
        }
        // c^Q wq_b -> qpre [S, H d]; per-head RmsNorm (weight 1) and rope into q_out
        if ((rc = gemm_rowmajor(bl, S, H * d, r, cq, cq_ld, wb.data, wb.ld, qpre, H * d)) != MLA_OK) return rc;
        mla::NormParams nq{};
        nq.eps = eps;
        nq.njobs = 1;
        nq.job[0] = mla::NormJob{qpre, H * d, bf(qo.data, s0 * qo.st_tok), qo.st_tok, qo.st_head, nullptr,
                                 bf(cs.data, s0 * cs.ld), bf(sn.data, s0 * sn.ld), cs.ld, sn.ld,
                                 static_cast<int>(d), static_cast<int>(R), static_cast<int>(H), S * H};
        if (t_prof_start && cudaEventRecord(t_prof_start, stream) != cudaSuccess) return MLA_ERR_CUDA;
        if ((rc = launch_norm(nq, ds->sm_count, stream)) != MLA_OK) return rc;
        if (t_prof_stop && cudaEventRecord(t_prof_stop, stream) != cudaSuccess) return MLA_ERR_CUDA;
    }
    return MLA_OK;
}

extern "C" int mla_prolog_set_path(int path) {
    if (path != -1 && path != 0) return MLA_ERR_UNSUPPORTED;
    t_prolog_path = path;
    return MLA_OK;
}

extern "C" int mla_prolog_last_fused(void) { return t_prolog_fused; }
