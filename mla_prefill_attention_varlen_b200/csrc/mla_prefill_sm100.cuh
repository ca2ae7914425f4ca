// Varlen causal MLA prefill on sm_100a: the plan kernel (sequence offsets and
// a longest-first work list) and the persistent, warp-specialised attention
// kernel (TMA -> shared memory, tcgen05 MMAs accumulating in tensor memory,
// online softmax in registers, direct vectorised stores).
//
// Operation (the "MLA Prefill" page of the Ascend Transformer Boost C API,
// AtbMLAPreFillGetWorkspaceSize members table): for sequence b, query head h,
// kv head kh = h / (headNum / kvHeadNum), query row i and key j,
//   s_ij = qkScale * (Q_nope[i,h] . K_nope[j,kh] + Q_rope[i,h] . K_rope[j,kh])
//   key j visible iff j <= i + (Lk - Lq)          (causal, bottom-right)
//   O[i,h] = sum_j softmax_j(s_ij) V[j,kh]
//
// Work unit: 256 query rows (two 128-row tiles t = 0, 1) of one sequence for
// one query head.  Both tiles share every K/V tile the kernel loads.  Per
// unit the kernel walks 128-key tiles j = 0 .. n-1; tiles wholly above the
// causal diagonal of a query tile are never visited for that tile:
//   MMA warp    S_t = [Qn|Qr]_t [Kn|Kr]_j^T  (12 MMAs 128x128x16 into TMEM; the
//               nope and rope k-steps accumulate into one accumulator)
//               O_t += P_t V_j                (8 MMAs, P read from TMEM)
//   softmax     warpgroup t owns tile t: rows of S_t -> mask -> running max /
//               sum -> P_t (16-bit) written back over S_t in TMEM; lazy rescale
//               of O_t when the running max grows by more than 2^8
//   load warp   TMA: Q tiles once per unit, then K_j (3 x 16 KB) and V_j
//               (2 x 16 KB) through a ring of eight 16 KB chunks
// MMA issue order per key tile: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1): while
// one warpgroup computes a softmax the tensor pipe works on the other tile.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,384),
// O1 [384,512); P_t occupies columns [64,128) of S_t.  S_t(j+1) is issued
// behind PV_t(j), which reads P_t(j); tcgen05.mma operations issued by one
// thread execute in issue order.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <type_traits>

#include "sm100_ptx.cuh"

namespace mla {

constexpr int kBM = 128;         // query rows per tile (= TMEM lanes)
constexpr int kUnitRows = 256;   // query rows per work unit (two tiles)
constexpr int kBN = 128;         // keys per key tile
constexpr int kDn = 128;         // nope width of Q/K, width of V (embeddimV)
constexpr int kDr = 64;          // rope width

constexpr int kChunkBytes = 16384;            // one ring chunk
constexpr int kQTileBytes = 3 * kChunkBytes;  // Qn cols 0-63 | Qn cols 64-127 | Qr  (128 rows each)
constexpr int kRing = 8;                      // ring chunks
constexpr int kKChunks = 3;                   // Kn lo | Kn hi | Kr            (128 keys each)
constexpr int kVChunks = 2;                   // keys 0-63 | keys 64-127      (V cols 0-63 then 64-127 inside)
constexpr int kVHalfBytes = 8192;             // 64 keys x 64 V columns
constexpr int kSched = 4;                     // depth of the work-item hand-off ring
constexpr int kTileBars = 4;                  // key-tile barrier sets (tiles in flight are at most 3)

constexpr int kSmemQ = 0;
constexpr int kSmemRing = kSmemQ + 2 * kQTileBytes;
constexpr int kSmemBar = kSmemRing + kRing * kChunkBytes;
constexpr int kSmemBytes = kSmemBar + 512;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024 B

constexpr uint32_t kTmemS = 0;      // S_t at t * 128
constexpr uint32_t kTmemO = 256;    // O_t at 256 + t * 128
constexpr uint32_t kTmemPOff = 64;  // P_t at S_t + 64
constexpr uint32_t kTmemCols = 512;

constexpr int kThreads = 384;  // warpgroup 0: TMA (warp 0), MMA (warp 1); warpgroups 1, 2: softmax of tiles 0, 1
constexpr int kRegsLow = 104;
constexpr int kRegsHigh = 200;
static_assert(kRegsLow * 128 + kRegsHigh * 256 <= 65536 / kThreads / 8 * 8 * kThreads,
              "register split exceeds the launch's register file share");

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // a pipeline wait gives up after 2 s

// Status codes the device writes (mirror mla_status in include/mla_prefill.h).
constexpr int kStatusSeqlen = 8;
constexpr int kStatusTimeout = 9;
constexpr int kStatusIndex = 10;

struct Params {
    const int4 *seq_info;  // per sequence {cq, ck, lq, lk} after clamping
    const int2 *units;     // (sequence, 256-row unit) pairs, most key tiles first
    const int *num_units;  // number of valid entries in units
    int *work_counter;     // dynamic work counter (zeroed by the plan kernel)
    int *status;           // sticky device status word
    void *out;
    long long out_st, out_sh;  // token / head strides of out, elements
    int out_v8;                // every output row starts on a 32-byte boundary: 256-bit stores
    int head_num;
    int group;         // head_num / kv_head_num
    int lpt;           // 1: items unit-major (longest first across all heads); 0: kv-head-major
    int head_pair;     // CTA-pair kernel only: 1 when its two groups run two query heads of one kv head over the
                       // same 256 rows (an item is a unit and a head pair), 0 when they run 512 rows of one head
    float scale_log2;  // qk_scale * log2(e)
    // paged K/V only: logical block i of sequence b is physical block tables[b * table_stride + i]
    const int *tables;
    long long table_stride;
    int table_width, num_blocks, block_size;
    int rows_k, rows_v;  // tokens per TMA box: min(128, block_size), min(64, block_size)
    int paged;  // K/V read from paged caches through the block table (kGeneral kernels only)
    // split-KV (kGeneral kernels only): a unit's key tiles go in chunks of split_tiles (0: none); entry e of the work
    // list is chunk entry_tab[e].y of unit entry_tab[e].x.  Chunks of a unit with more than one
    // write O / l (fp32) and the base-2 log-sum-exp of each row to part_o / part_lse at
    // ((e * head_num + h) * 256 + row); mla_split_combine_kernel merges them.
    int split_tiles;
    const int2 *entry_tab;
    const int *num_entries;
    float *part_o, *part_lse;
};

struct Barriers {
    uint64_t q_full[2], q_empty[2];
    // key tile g (counted per CTA across its units) occupies ring chunks 5g .. 5g + 4 (slot = chunk % kRing):
    // K_g in 5g .. 5g + 2, V_g in 5g + 3, 5g + 4.  Set g % kTileBars of these barriers tracks it:
    // k_full / v_full complete when its K / V bytes have landed; k_empty / v_empty when the last MMA
    // reading its K / V has completed.
    uint64_t k_full[kTileBars], v_full[kTileBars], k_empty[kTileBars], v_empty[kTileBars];
    uint64_t s_full[2], p_full[2];
    uint64_t o_full[2], o_empty[2];
    uint64_t sched_full[kSched], sched_empty[kSched];
    uint64_t drain;
    int sched_item[kSched];
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Barriers) <= 512, "barrier block too large");

// Number of 128-key tiles a 128-row query tile touches: the keys visible to its
// last row (causal) or all keys.  0 when the tile has no rows or sees no key.
__host__ __device__ __forceinline__ int kv_tiles_for(int q0, int rows, int lq, int lk, bool causal) {
    if (rows <= 0) return 0;
    const int kv_end = causal ? min(q0 + rows + (lk - lq), lk) : lk;
    return kv_end > 0 ? (kv_end + kBN - 1) / kBN : 0;
}

__host__ __device__ __forceinline__ int tile_rows(int q0, int lq) { return max(0, min(kBM, lq - q0)); }

// Key tiles a unit of unit_rows query rows (256: two tiles, 512: four) walks: the largest count
// among its 128-row tiles.
__host__ __device__ __forceinline__ int unit_cost(int u0, int lq, int lk, bool causal, int unit_rows = kUnitRows) {
    int c = 0;
    for (int r = 0; r < unit_rows; r += kBM) {
        const int n = kv_tiles_for(u0 + r, tile_rows(u0 + r, lq), lq, lk, causal);
        c = n > c ? n : c;
    }
    return c;
}

struct WorkItem {
    int b;  // sequence
    int h, kh;
    int u0;              // first query row of the unit within its sequence
    int q_tok0, k_tok0;  // first packed token of the unit / of the sequence's keys
    int lq, lk, off;     // off = Lk - Lq
    int rows[2];         // valid rows of tile 0 / 1
    int j0;              // first key tile of this item (split-KV chunk start; 0 without split)
    int n[2];            // key tiles of tile 0 / 1 from j0 on
    int n_max;
    int e, nsplit;       // work-list entry; chunks of its unit (1: the item writes attenOut itself)
};

// Work items are ordered kv-head-major: for each kv head, its units in the
// sorted (longest-first) order, and for each unit the query heads of the group.
// Concurrently running CTAs then read the same kv head's K/V (L2 reuse), and the
// last items of each kv head are its cheapest units.  When all of K/V fits in L2
// with room to spare (p.lpt), reuse needs no such order: the items go unit-major
// instead (every head of the longest unit first), the longest-first order over the
// whole grid, which shortens the tail when there are only a few items per SM.
__device__ __forceinline__ void item_unit_head(const Params &p, int it, int num_entries, int &e, int &h) {
    if (p.lpt) {
        e = it / p.head_num;
        h = it - e * p.head_num;
    } else {
        const int per_kh = num_entries * p.group;
        const int kh = it / per_kh;
        const int rem = it - kh * per_kh;
        e = rem / p.group;
        h = kh * p.group + (rem - e * p.group);
    }
}

template <bool kSplit>  // kSplit: the kernel may run split-KV work lists
__device__ __forceinline__ WorkItem decode_item(const Params &p, int it, int num_entries, bool causal) {
    WorkItem x;
    item_unit_head(p, it, num_entries, x.e, x.h);
    x.kh = x.h / p.group;
    int u = x.e, chunk = 0;
    if (kSplit && p.split_tiles > 0) {
        const int2 uc = p.entry_tab[x.e];
        u = uc.x;
        chunk = uc.y;
    }
    const int2 bm = p.units[u];
    x.b = bm.x;
    const int4 s = p.seq_info[bm.x];
    x.u0 = bm.y * kUnitRows;
    x.q_tok0 = s.x + x.u0;
    x.k_tok0 = s.y;
    x.lq = s.z;
    x.lk = s.w;
    x.off = s.w - s.z;
    x.j0 = 0;
    x.nsplit = 1;
    if constexpr (!kSplit) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            x.rows[t] = tile_rows(x.u0 + t * kBM, s.z);
            x.n[t] = kv_tiles_for(x.u0 + t * kBM, x.rows[t], s.z, s.w, causal);
        }
        x.n_max = max(x.n[0], x.n[1]);
    } else {
        int full[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            x.rows[t] = tile_rows(x.u0 + t * kBM, s.z);
            full[t] = kv_tiles_for(x.u0 + t * kBM, x.rows[t], s.z, s.w, causal);
        }
        const int nf = max(full[0], full[1]);
        int j1 = nf;
        if (p.split_tiles > 0 && nf > p.split_tiles) {
            x.nsplit = (nf + p.split_tiles - 1) / p.split_tiles;
            x.j0 = chunk * p.split_tiles;
            j1 = min(nf, x.j0 + p.split_tiles);
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) x.n[t] = max(0, min(full[t], j1) - x.j0);
        x.n_max = j1 - x.j0;
    }
    return x;
}

// Bounded mbarrier wait.  Gives up (and makes every role give up) when another
// role has aborted or after kWaitLimitNs, recording kStatusTimeout.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, Barriers *bars, int *status,
                                         uint64_t limit_ns = kWaitLimitNs) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (*reinterpret_cast<volatile int *>(&bars->abort)) return false;
            if (ptx::globaltimer_ns() - t0 > limit_ns) {
                *reinterpret_cast<volatile int *>(&bars->abort) = 1;
                atomicCAS(status, 0, kStatusTimeout);
                return false;
            }
        }
    }
}

// The same wait for a whole warp: every lane polls, and the result is made
// warp-uniform so that all lanes take the same path afterwards.
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, Barriers *bars, int *status,
                                              uint64_t limit_ns = kWaitLimitNs) {
    const bool ok = wait_bar(bar, parity, bars, status, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

template <typename T>
struct DType;
template <>
struct DType<__nv_bfloat16> {
    static constexpr bool kBf16 = true;
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
};
template <>
struct DType<__half> {
    static constexpr bool kBf16 = false;
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t *>(&v);
    }
};

// 32 output columns (64 bytes) of one row: two 256-bit stores when rows are 32-byte aligned,
// else four 128-bit stores.
template <typename T>
__device__ __forceinline__ void store_row_chunk(T *dst, const uint32_t (&w)[16], int v8) {
    if (v8) {
        ptx::st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
        ptx::st_global_v8(dst + 16, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
    } else {
        uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
        for (int e = 0; e < 4; ++e) d[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
    }
}

// ---------------------------------------------------------------------------
// Plan kernel: one block of 1024 threads.  Clamps the seqlens to the tensor
// extents (recording kStatusSeqlen on any inconsistency), writes per-sequence
// offsets, and writes the (sequence, unit of unit_rows rows) list sorted by descending
// number of key tiles (a counting sort; ties in arbitrary order).  With
// reset_status, the status word is zeroed first (a word that reports one call).
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;

__device__ __forceinline__ long long block_exclusive_scan(long long v, long long &total, long long *warp_sums) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[w] = x;
    __syncthreads();
    if (w == 0) {
        long long y = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long z = __shfl_up_sync(0xffffffffu, y, o);
            if (lane >= o) y += z;
        }
        warp_sums[lane] = y;
    }
    __syncthreads();
    const long long before = (w ? warp_sums[w - 1] : 0) + x - v;
    total = warp_sums[nw - 1];
    __syncthreads();
    return before;
}

__device__ __forceinline__ int seq_of_unit(const int *unit_off, int batch, int t) {
    int lo = 0, hi = batch - 1;  // last b with unit_off[b] <= t (sequences without units are skipped)
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (unit_off[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kPlanThreads) mla_plan_kernel(const int *__restrict__ q_seqlen,
                                                                const int *__restrict__ kv_seqlen, int batch,
                                                                long long t_q, long long t_k, long long kv_pad,
                                                                int paged, int causal,
                                                                int4 *seq_info, int *unit_off, int *hist,
                                                                int hist_len, int2 *units, int *num_units,
                                                                int *work_counter, int split_tiles, int *split_off,
                                                                int2 *entry_tab, int *num_entries, int *status,
                                                                int reset_status, int unit_rows) {
    __shared__ long long warp_sums[32];
    __shared__ int bad;
    // the attention grid may be scheduled now: it sets itself up and then waits for this grid
    ptx::griddep_launch_dependents();
    if (threadIdx.x == 0) {
        bad = 0;
        // a per-call status word (caller-owned workspace) starts each call at 0; the attention
        // kernel writes it only after this grid has completed
        if (reset_status) *status = 0;
    }
    __syncthreads();

    // 1. clamped prefix sums and unit counts, in chunks of blockDim.x sequences
    long long carry_q = 0, carry_k = 0, carry_u = 0;
    for (int base = 0; base < batch; base += blockDim.x) {
        const int b = base + threadIdx.x;
        long long lq = 0, lk = 0;
        if (b < batch) {
            lq = q_seqlen[b];
            lk = kv_seqlen[b];
            if (lq < 0 || lk < 0) bad = 1;
            lq = lq < 0 ? 0 : lq;
            lk = lk < 0 ? 0 : lk;
        }
        long long tot_q, tot_k;
        const long long pq = carry_q + block_exclusive_scan(lq, tot_q, warp_sums);
        const long long pk = carry_k + block_exclusive_scan(lk, tot_k, warp_sums);
        const long long cq = pq < t_q ? pq : t_q, eq = pq + lq < t_q ? pq + lq : t_q;
        // packed K/V: sequences follow each other; padded K/V: sequence b starts at b * kv_pad
        // paged K/V: keys are addressed through the block table; kv_pad is the table's capacity
        const long long kb = paged ? 0 : (kv_pad ? (long long)b * kv_pad : pk);
        const long long kcap = kv_pad ? kb + kv_pad : t_k;
        const long long ck = kb < t_k ? kb : t_k, ek = kb + lk < kcap ? (kb + lk < t_k ? kb + lk : t_k) : (kcap < t_k ? kcap : t_k);
        if (b < batch && (eq - cq != lq || ek - ck != lk)) bad = 1;
        const int lqc = static_cast<int>(eq - cq), lkc = static_cast<int>(ek - ck);
        const long long nu = (b < batch) ? (lqc + unit_rows - 1) / unit_rows : 0;
        long long tot_u;
        const long long pu = carry_u + block_exclusive_scan(nu, tot_u, warp_sums);
        if (b < batch) {
            seq_info[b] = make_int4(static_cast<int>(cq), static_cast<int>(ck), lqc, lkc);
            unit_off[b] = static_cast<int>(pu);
        }
        carry_q += tot_q;
        carry_k += tot_k;
        carry_u += tot_u;
    }
    const int total = static_cast<int>(carry_u);
    if (threadIdx.x == 0) unit_off[batch] = total;
    for (int c = threadIdx.x; c < hist_len; c += blockDim.x) hist[c] = 0;
    __syncthreads();

    // 2. histogram of key-tile counts
    for (int t = threadIdx.x; t < total; t += blockDim.x) {
        const int b = seq_of_unit(unit_off, batch, t);
        const int4 s = seq_info[b];
        const int cost = unit_cost((t - unit_off[b]) * unit_rows, s.z, s.w, causal != 0, unit_rows);
        atomicAdd(&hist[min(cost, hist_len - 1)], 1);
    }
    __syncthreads();

    // 3. bucket starts, largest cost first
    long long carry = 0;
    for (int base = 0; base < hist_len; base += blockDim.x) {
        const int r = base + threadIdx.x;
        const int c = hist_len - 1 - r;
        const long long n = r < hist_len ? hist[c] : 0;
        long long tot;
        const long long start = carry + block_exclusive_scan(n, tot, warp_sums);
        if (r < hist_len) hist[c] = static_cast<int>(start);
        carry += tot;
    }
    __syncthreads();

    // 4. scatter
    for (int t = threadIdx.x; t < total; t += blockDim.x) {
        const int b = seq_of_unit(unit_off, batch, t);
        const int4 s = seq_info[b];
        const int m = t - unit_off[b];
        const int cost = unit_cost(m * unit_rows, s.z, s.w, causal != 0, unit_rows);
        const int pos = atomicAdd(&hist[min(cost, hist_len - 1)], 1);
        units[pos] = make_int2(b, m);
    }
    __syncthreads();

    // 5. split-KV: unit u (sorted order) becomes ceil(cost / split_tiles) entries, in unit order
    long long entries = total;
    if (split_tiles > 0) {
        long long carry_e = 0;
        for (int base = 0; base < total; base += blockDim.x) {
            const int u = base + threadIdx.x;
            long long ns = 0;
            if (u < total) {
                const int2 bm = units[u];
                const int4 s = seq_info[bm.x];
                const int cost = unit_cost(bm.y * unit_rows, s.z, s.w, causal != 0, unit_rows);
                ns = cost > split_tiles ? (cost + split_tiles - 1) / split_tiles : 1;
            }
            long long tot;
            const long long pe = carry_e + block_exclusive_scan(ns, tot, warp_sums);
            if (u < total) {
                split_off[u] = static_cast<int>(pe);
                for (int c = 0; c < ns; ++c) entry_tab[pe + c] = make_int2(u, c);
            }
            carry_e += tot;
        }
        entries = carry_e;
        if (threadIdx.x == 0) split_off[total] = static_cast<int>(carry_e);
    }
    if (threadIdx.x == 0) {
        *num_units = total;
        *num_entries = static_cast<int>(entries);
        *work_counter = 0;
        if (bad) atomicCAS(status, 0, kStatusSeqlen);
    }
}

// Max of a 128-element row: eight independent chains of three-input max
// (two new elements per instruction), then a short tree.
__device__ __forceinline__ float row_max(const float (&s)[kBN]) {
    static_assert(kBN == 128, "the block split below assumes 128 keys per tile");
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = ptx::fmax3(s[i], s[i + 8], s[i + 16]);  // s[0..23]
#pragma unroll
    for (int c = 24; c + 16 <= kBN; c += 16) {                                 // s[24..119]
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = ptx::fmax3(m[i], s[c + i], s[c + 8 + i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], s[120 + i]);                // s[120..127]
    return ptx::fmax3(ptx::fmax3(m[0], m[1], m[2]), ptx::fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// Exponentials of one row of a key tile: p = 2^(s * sc - m) for the 128 scores, packed to the
// 16-bit P operand (pk) and summed in fp32 (returned): one packed FMA per pair, one MUFU ex2 per
// element, four packed partial sums, one 16-bit pair conversion per pair.
template <typename T>
__device__ __forceinline__ float exp_pack_sum(const float (&s)[kBN], float2 sc2, float2 nm2, uint32_t (&pk)[kBN / 2]) {
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int e = 0; e < kBN / 2; ++e) {
        const float2 x2 = ptx::ffma2(make_float2(s[2 * e], s[2 * e + 1]), sc2, nm2);
        const float2 p2 = make_float2(ptx::ex2(x2.x), ptx::ex2(x2.y));
        acc[e & 3] = ptx::fadd2(acc[e & 3], p2);
        pk[e] = DType<T>::pack(p2.x, p2.y);
    }
    const float2 acc01 = ptx::fadd2(acc[0], acc[1]), acc23 = ptx::fadd2(acc[2], acc[3]);
    const float2 acc2 = ptx::fadd2(acc01, acc23);
    return acc2.x + acc2.y;
}

// ---------------------------------------------------------------------------
// Attention kernel
// ---------------------------------------------------------------------------
// kGeneral: padded or paged K/V, where rows of the last key tile past Lk may hold anything
// (padding, unwritten cache slots), or a split-KV work list.  The packed, unsplit kernels
// (kGeneral = false) carry none of that code: their last key tile holds only real keys or
// TMA's zero fill.
template <typename T, bool kCausal, bool kPositiveScale, bool kGeneral>
__global__ void __launch_bounds__(kThreads, 1)
    mla_prefill_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                             const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kr,
                             const __grid_constant__ CUtensorMap tm_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Barriers *bars = reinterpret_cast<Barriers *>(smem + kSmemBar);
    const uint32_t sQ = ptx::smem_addr(smem + kSmemQ);
    const uint32_t sRing = ptx::smem_addr(smem + kSmemRing);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    auto bar = [&](uint64_t &b) { return ptx::smem_addr(&b); };

    if (threadIdx.x == 32) {
        // the tensor maps' descriptors are fetched while the CTA sets up (and, with programmatic
        // dependent launch, while the plan kernel still runs)
        ptx::tma_prefetch_desc(&tm_q);
        ptx::tma_prefetch_desc(&tm_qr);
        ptx::tma_prefetch_desc(&tm_k);
        ptx::tma_prefetch_desc(&tm_kr);
        ptx::tma_prefetch_desc(&tm_v);
    }
    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            ptx::mbar_init(bar(bars->q_full[t]), 1);
            ptx::mbar_init(bar(bars->q_empty[t]), 1);
            ptx::mbar_init(bar(bars->s_full[t]), 1);
            ptx::mbar_init(bar(bars->p_full[t]), kBM);
            ptx::mbar_init(bar(bars->o_full[t]), 1);
            ptx::mbar_init(bar(bars->o_empty[t]), kBM);
        }
        for (int c = 0; c < kTileBars; ++c) {
            ptx::mbar_init(bar(bars->k_full[c]), 1);
            ptx::mbar_init(bar(bars->v_full[c]), 1);
            ptx::mbar_init(bar(bars->k_empty[c]), 1);
            ptx::mbar_init(bar(bars->v_empty[c]), 1);
        }
        for (int i = 0; i < kSched; ++i) {
            ptx::mbar_init(bar(bars->sched_full[i]), 1);
            ptx::mbar_init(bar(bars->sched_empty[i]), 1 + 8);  // the MMA warp + each softmax warp
        }
        ptx::mbar_init(bar(bars->drain), 1);
        bars->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_addr(&bars->tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    // everything above overlaps the plan kernel; the work list is read only after it has finished
    ptx::griddep_wait();
    const int num_entries = *p.num_entries;
    const int n_items = num_entries * p.head_num;

    if (warp < 4) {
        ptx::regs_dec<kRegsLow>();
        if (warp == 0) {
            // -------------------------------------------------------- TMA producer
            // Lane 0 alone for packed and padded K/V.  For paged K/V the whole warp runs the
            // loop (its state is warp-uniform): lane e looks up physical block e of a key tile
            // (one tile ahead), and lane r issues the r-th TMA box of a chunk, so the work per
            // tile does not grow as the blocks get smaller.
            auto producer = [&](auto warp_wide) {
                constexpr bool kW = decltype(warp_wide)::value;
                const bool lead = !kW || lane == 0;
                auto wait = [&](uint32_t b, uint32_t parity) -> bool {
                    return kW ? wait_bar_warp(b, parity, bars, p.status) : wait_bar(b, parity, bars, p.status);
                };
                const uint64_t pol_q = ptx::policy_evict_first();
                const uint64_t pol_kv = ptx::policy_evict_last();
                uint32_t tk = 0, tv = 0;    // key tiles whose K / V loads have been issued
                uint32_t ql0 = 0, ql1 = 0;  // Q tiles loaded per tile slot
                bool ok = true;
                auto chunk = [&](uint32_t c) { return sRing + (c % kRing) * kChunkBytes; };
                // K_g's chunks last held K_{g-2}[2] and V_{g-2}: free once the last MMA reading V_{g-2} has
                // completed (it was issued after every MMA reading K_{g-2}).  V_g's chunks last held
                // K_{g-1}[0, 1].  Each returns the tile's full barrier, armed with its byte count.
                auto begin_k = [&](uint32_t g, uint32_t &fb) -> bool {
                    if (g >= 2 && !wait(bar(bars->v_empty[(g - 2) % kTileBars]), ((g - 2) / kTileBars) & 1))
                        return false;
                    fb = bar(bars->k_full[g % kTileBars]);
                    if (lead) ptx::mbar_arrive_expect_tx(fb, kKChunks * kChunkBytes);
                    ++tk;
                    return true;
                };
                auto begin_v = [&](uint32_t g, uint32_t &fb) -> bool {
                    if (g >= 1 && !wait(bar(bars->k_empty[(g - 1) % kTileBars]), ((g - 1) / kTileBars) & 1))
                        return false;
                    fb = bar(bars->v_full[g % kTileBars]);
                    if (lead) ptx::mbar_arrive_expect_tx(fb, kVChunks * kChunkBytes);
                    ++tv;
                    return true;
                };
                // Dynamic scheduling: the first item is blockIdx.x, later ones come from a global
                // counter; each claimed item index (or -1 at the end) is handed to the MMA and
                // softmax warps through a small ring in shared memory.  The next item is claimed
                // when the loads of the current one's last key tile are about to be issued, about
                // one key tile before this CTA runs out of work: claimed at an item's start, a
                // CTA that drew a long item would also take the next item of the longest-first
                // list from CTAs that free up sooner.
                uint32_t sc = 0;
                int next = blockIdx.x < n_items ? (int)blockIdx.x : -1;
                while (ok) {
                    const int it = next;
                    const uint32_t slot = sc % kSched;
                    ok = wait(bar(bars->sched_empty[slot]), ((sc / kSched) & 1) ^ 1);
                    if (!ok) break;
                    if (lead) {
                        *reinterpret_cast<volatile int *>(&bars->sched_item[slot]) = it;
                        ptx::mbar_arrive(bar(bars->sched_full[slot]));
                    }
                    ++sc;
                    if (it < 0) break;
                    auto claim = [&]() {
                        if (lead) {
                            next = (int)gridDim.x + atomicAdd(p.work_counter, 1);
                            if (next >= n_items) next = -1;
                        }
                        if (kW) next = __shfl_sync(0xffffffffu, next, 0);
                    };
                    const WorkItem x = decode_item<kGeneral>(p, it, num_entries, kCausal);
                    if (x.n_max == 0) {
                        claim();
                        continue;
                    }
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (!ok || x.n[t] == 0) continue;
                        uint32_t &ql = t ? ql1 : ql0;
                        // Q_t of the previous unit is free once its last S_t MMA has completed.
                        ok = wait(bar(bars->q_empty[t]), (ql & 1) ^ 1);
                        if (!ok) continue;
                        const uint32_t fb = bar(bars->q_full[t]);
                        const uint32_t dst = sQ + t * kQTileBytes;
                        const int tok = x.q_tok0 + t * kBM;
                        if (lead) {
                            ptx::mbar_arrive_expect_tx(fb, kQTileBytes);
                            ptx::tma_load_3d(dst, &tm_q, fb, 0, x.h, tok, pol_q);
                            ptx::tma_load_3d(dst + kChunkBytes, &tm_q, fb, 64, x.h, tok, pol_q);
                            ptx::tma_load_3d(dst + 2 * kChunkBytes, &tm_qr, fb, 0, x.h, tok, pol_q);
                        }
                        ++ql;
                    }
                    if constexpr (kW) {
                        // Paged caches.  Key tile j spans `per` logical blocks (128 / block_size, or 1
                        // for blocks of 128 keys or more); lane e < per holds the physical id of block
                        // e.  A block wholly past Lk, or one without a valid id, becomes block
                        // num_blocks: out of the map, so TMA fills its boxes with zeros and reads nothing.
                        const int bs = p.block_size;
                        const int per = bs < kBN ? kBN / bs : 1;
                        auto first_key = [&](int j) { return max((j * kBN / bs + lane) * bs, j * kBN); };
                        auto raw_id = [&](int j) -> int {  // issues the table load; checked when used
                            const int lb = j * kBN / bs + lane;
                            if (lane >= per || first_key(j) >= x.lk) return p.num_blocks;
                            return lb < p.table_width ? __ldg(p.tables + (long long)x.b * p.table_stride + lb) : -1;
                        };
                        // `count` TMA boxes of `rows` keys each, from logical position pos0 (a multiple
                        // of rows); box r comes from one block and lands on whole 1 KB swizzle atoms.
                        auto boxes = [&](int id, int j, uint32_t dst, const void *map, uint32_t fb, int c0, int pos0,
                                         int rows, int count) {
                            const int r = lane < count ? lane : 0;
                            const int pos = pos0 + r * rows;
                            const int lb = pos / bs;
                            const int blk = __shfl_sync(0xffffffffu, id, lb - j * kBN / bs);
                            if (lane < count)
                                ptx::tma_load_4d(dst + r * rows * 128, map, fb, c0, x.kh, pos - lb * bs, blk, pol_kv);
                        };
                        const int nk = kBN / p.rows_k, nv = 64 / p.rows_v;
                        int id_next = raw_id(x.j0);
                        for (int jl = 0; jl < x.n_max && ok; ++jl) {
                            if (jl == x.n_max - 1) claim();
                            const int j = x.j0 + jl;  // absolute key tile
                            int id = id_next;
                            if (jl + 1 < x.n_max) id_next = raw_id(j + 1);  // in flight during tile j
                            if (lane < per && first_key(j) < x.lk && (id < 0 || id >= p.num_blocks)) {
                                atomicCAS(p.status, 0, kStatusIndex);  // a visible key without a block
                                id = p.num_blocks;
                            }
                            const uint32_t g = tk, c0 = 5 * g;
                            uint32_t fb;
                            // K_j from the [nope | rope] key cache: columns 0-63, 64-127, 128-191
                            if (!(ok = begin_k(g, fb))) break;
                            for (int c = 0; c < kKChunks; ++c)
                                boxes(id, j, chunk(c0 + c), &tm_k, fb, 64 * c, j * kBN, p.rows_k, nk);
                            // V_j: keys 0-63, keys 64-127; each chunk holds V cols 0-63 then 64-127
                            if (!(ok = begin_v(g, fb))) break;
                            for (int hh = 0; hh < kVChunks; ++hh) {
                                const uint32_t dst = chunk(c0 + kKChunks + hh);
                                boxes(id, j, dst, &tm_v, fb, 0, j * kBN + hh * 64, p.rows_v, nv);
                                boxes(id, j, dst + kVHalfBytes, &tm_v, fb, 64, j * kBN + hh * 64, p.rows_v, nv);
                            }
                        }
                    } else {
                        for (int jl = 0; jl < x.n_max && ok; ++jl) {
                            if (jl == x.n_max - 1) claim();
                            const int tok = x.k_tok0 + (x.j0 + jl) * kBN;
                            const uint32_t g = tk, c0 = 5 * g;
                            uint32_t fb;
                            // K_j: nope cols 0-63, nope cols 64-127, rope
                            if (!(ok = begin_k(g, fb))) break;
                            ptx::tma_load_3d(chunk(c0), &tm_k, fb, 0, x.kh, tok, pol_kv);
                            ptx::tma_load_3d(chunk(c0 + 1), &tm_k, fb, 64, x.kh, tok, pol_kv);
                            ptx::tma_load_3d(chunk(c0 + 2), &tm_kr, fb, 0, x.kh, tok, pol_kv);
                            // V_j: keys 0-63, keys 64-127; each chunk holds V cols 0-63 then 64-127
                            if (!(ok = begin_v(g, fb))) break;
                            for (int hh = 0; hh < kVChunks; ++hh) {
                                const uint32_t dst = chunk(c0 + kKChunks + hh);
                                ptx::tma_load_3d(dst, &tm_v, fb, 0, x.kh, tok + hh * 64, pol_kv);
                                ptx::tma_load_3d(dst + kVHalfBytes, &tm_v, fb, 64, x.kh, tok + hh * 64, pol_kv);
                            }
                        }
                    }
                }
                // Let every copy this warp started land before the block can exit.
                if (ql0) wait(bar(bars->q_full[0]), (ql0 - 1) & 1);
                if (ql1) wait(bar(bars->q_full[1]), (ql1 - 1) & 1);
                // (older tiles have been consumed by the MMA warp, so their bytes have landed)
                for (uint32_t g = tk > kTileBars ? tk - kTileBars : 0; g < tk; ++g)
                    wait(bar(bars->k_full[g % kTileBars]), (g / kTileBars) & 1);
                for (uint32_t g = tv > kTileBars ? tv - kTileBars : 0; g < tv; ++g)
                    wait(bar(bars->v_full[g % kTileBars]), (g / kTileBars) & 1);
            };
            if constexpr (kGeneral) {
                if (p.paged) producer(std::true_type{});
                else if (lane == 0) producer(std::false_type{});
            } else {
                if (lane == 0) producer(std::false_type{});
            }
        } else if (warp == 1) {
            // -------------------------------------------------------- MMA issuer
            // The whole warp runs this loop (all its state is warp-uniform); one
            // elected lane issues each batch of MMAs and each commit.
            constexpr bool kBf16 = DType<T>::kBf16;
            constexpr uint32_t kIdQK = ptx::instr_desc_f16(kBf16, kBM, kBN, false);
            constexpr uint32_t kIdPV = ptx::instr_desc_f16(kBf16, kBM, kDn, true);
            constexpr uint32_t kHi = ptx::desc_hi_sw128(1024);
            // Descriptor low words: K-major Q / K blocks (leading offset unused: 16 B) and
            // MN-major V blocks (leading offset = distance between the two 64-column halves).
            const uint32_t q_lo = ptx::desc_lo(sQ, 16);
            const uint32_t ring_k_lo = ptx::desc_lo(sRing, 16);
            const uint32_t ring_v_lo = ptx::desc_lo(sRing, kVHalfBytes);
            uint32_t tg = 0;  // key tiles of earlier units: the unit's key tile j is tile tg + j
            uint32_t qf0 = 0, qf1 = 0, pf0 = 0, pf1 = 0, oe0 = 0, oe1 = 0;
            bool ok = true;
            auto wait_tile = [&](uint64_t (&full)[kTileBars], uint32_t g) -> bool {
                return wait_bar_warp(bar(full[g % kTileBars]), (g / kTileBars) & 1, bars, p.status);
            };
            auto commit = [&](uint64_t &b) {
                if (ptx::elect_one()) ptx::mma_commit(bar(b));
                __syncwarp();
            };
            // S_t = Q_t K^T for the K chunks starting at ring index kc
            auto issue_s = [&](int t, uint32_t kc) {
                const uint32_t d = tmem + kTmemS + t * kBN;
                const uint32_t a0 = q_lo + ((t * kQTileBytes) >> 4);
                const uint32_t b0 = ring_k_lo + (((kc + 0) % kRing) * (kChunkBytes >> 4));
                const uint32_t b1 = ring_k_lo + (((kc + 1) % kRing) * (kChunkBytes >> 4));
                const uint32_t b2 = ring_k_lo + (((kc + 2) % kRing) * (kChunkBytes >> 4));
                if (ptx::elect_one()) {
                    constexpr uint32_t kC = kChunkBytes >> 4;  // one chunk, in descriptor units
                    ptx::mma_ss_lo<kHi, kIdQK, 0>(d, a0 + 0, b0 + 0);  // 16 elements = 2 units per k-step
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + 2, b0 + 2);
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + 4, b0 + 4);
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + 6, b0 + 6);
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + kC + 0, b1 + 0);
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + kC + 2, b1 + 2);
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + kC + 4, b1 + 4);
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + kC + 6, b1 + 6);
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + 2 * kC + 0, b2 + 0);
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + 2 * kC + 2, b2 + 2);
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + 2 * kC + 4, b2 + 4);
                    ptx::mma_ss_lo<kHi, kIdQK, 1>(d, a0 + 2 * kC + 6, b2 + 6);
                    ptx::mma_commit(bar(bars->s_full[t]));
                }
                __syncwarp();
            };
            // O_t (+)= P_t V for the V chunks starting at ring index vc
            auto issue_pv = [&](int t, uint32_t vc, bool accumulate) {
                const uint32_t d = tmem + kTmemO + t * kDn;
                const uint32_t pa = tmem + kTmemS + t * kBN + kTmemPOff;
                const uint32_t v0 = ring_v_lo + (((vc + 0) % kRing) * (kChunkBytes >> 4));
                const uint32_t v1 = ring_v_lo + (((vc + 1) % kRing) * (kChunkBytes >> 4));
                if (ptx::elect_one()) {
                    // 16 keys x 128 B = 2048 B = 128 units per k-step; P advances 8 columns per k-step
                    if (accumulate) ptx::mma_ts_lo<kHi, kIdPV, 1>(d, pa, v0);
                    else ptx::mma_ts_lo<kHi, kIdPV, 0>(d, pa, v0);
                    ptx::mma_ts_lo<kHi, kIdPV, 1>(d, pa + 8, v0 + 128);
                    ptx::mma_ts_lo<kHi, kIdPV, 1>(d, pa + 16, v0 + 256);
                    ptx::mma_ts_lo<kHi, kIdPV, 1>(d, pa + 24, v0 + 384);
                    ptx::mma_ts_lo<kHi, kIdPV, 1>(d, pa + 32, v1);
                    ptx::mma_ts_lo<kHi, kIdPV, 1>(d, pa + 40, v1 + 128);
                    ptx::mma_ts_lo<kHi, kIdPV, 1>(d, pa + 48, v1 + 256);
                    ptx::mma_ts_lo<kHi, kIdPV, 1>(d, pa + 56, v1 + 384);
                }
                __syncwarp();
            };
            uint32_t ss = 0;
            while (ok) {
                const uint32_t slot = ss % kSched;
                ok = wait_bar_warp(bar(bars->sched_full[slot]), (ss / kSched) & 1, bars, p.status);
                if (!ok) break;
                const int it = *reinterpret_cast<volatile int *>(&bars->sched_item[slot]);
                __syncwarp();
                if (ptx::elect_one()) ptx::mbar_arrive(bar(bars->sched_empty[slot]));
                __syncwarp();
                ++ss;
                if (it < 0) break;
                const WorkItem x = decode_item<kGeneral>(p, it, num_entries, kCausal);
                if (x.n_max == 0) continue;
                if (x.n[0]) ok = wait_bar_warp(bar(bars->q_full[0]), qf0++ & 1, bars, p.status);
                if (ok && x.n[1]) ok = wait_bar_warp(bar(bars->q_full[1]), qf1++ & 1, bars, p.status);
                if (!ok) break;
                // key tile g = tg + j: K_g in ring chunks 5g + {0,1,2}, V_g in 5g + {3,4}.  The last MMA
                // reading a key tile is tile 1's when tile 1 reads it (issued after tile 0's), else tile 0's.
                ok = wait_tile(bars->k_full, tg);
                if (!ok) break;
                ptx::tc_fence_after();
                if (x.n[0] > 0) {
                    issue_s(0, 5 * tg);
                    if (x.n[0] == 1) commit(bars->q_empty[0]);
                }
                if (x.n[1] > 0) {
                    issue_s(1, 5 * tg);
                    if (x.n[1] == 1) commit(bars->q_empty[1]);
                }
                commit(bars->k_empty[tg % kTileBars]);
                for (int j = 0; j < x.n_max && ok; ++j) {
                    const uint32_t g = tg + j, kc = 5 * g, vc = kc + 3, kn = kc + 5;
                    bool v_ready = false, k_next_ready = false;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (ok && j < x.n[t]) {
                            uint32_t &pf = t ? pf1 : pf0;
                            uint32_t &oe = t ? oe1 : oe0;
                            ok = wait_bar_warp(bar(bars->p_full[t]), pf++ & 1, bars, p.status);
                            if (ok && !v_ready) {
                                ok = wait_tile(bars->v_full, g);
                                v_ready = true;
                            }
                            if (ok && j == 0) ok = wait_bar_warp(bar(bars->o_empty[t]), (oe++ & 1) ^ 1, bars, p.status);
                            if (ok) {
                                ptx::tc_fence_after();
                                issue_pv(t, vc, j > 0);
                                if (j == x.n[t] - 1) commit(bars->o_full[t]);
                                if (t == 1 || j >= x.n[1]) commit(bars->v_empty[g % kTileBars]);  // last P V_g
                            }
                        }
                        if (ok && j + 1 < x.n[t]) {
                            if (!k_next_ready) {
                                ok = wait_tile(bars->k_full, g + 1);
                                k_next_ready = true;
                                if (ok) ptx::tc_fence_after();
                            }
                            if (ok) {
                                issue_s(t, kn);
                                if (j + 2 == x.n[t]) commit(bars->q_empty[t]);  // last S_t of the unit
                                if (t == 1 || j + 1 >= x.n[1]) commit(bars->k_empty[(g + 1) % kTileBars]);  // last S of K_{g+1}
                            }
                        }
                    }
                }
                if (!ok) break;
                tg += x.n_max;
            }
            // Drain: wait until every MMA this warp issued has completed.
            commit(bars->drain);
            wait_bar_warp(bar(bars->drain), 0, bars, p.status);
        }
    } else {
        ptx::regs_inc<kRegsHigh>();
        // ------------------------------------------------------------ softmax + epilogue
        const int t = (warp >> 2) - 1;   // query tile of this warpgroup
        const int wq = warp & 3;         // TMEM lane quarter this warp may access
        const int row = wq * 32 + lane;  // query row within the tile
        const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_addr + kTmemS + t * kBN;
        const uint32_t tO = tmem + lane_addr + kTmemO + t * kDn;
        const float sl2 = p.scale_log2;
        uint32_t sf = 0, of = 0;
        bool ok = true;
        uint32_t ss = 0, tiles_seen = 0;
        while (ok) {
            const uint32_t slot = ss % kSched;
            ok = wait_bar_warp(bar(bars->sched_full[slot]), (ss / kSched) & 1, bars, p.status);
            if (!ok) break;
            const int it = *reinterpret_cast<volatile int *>(&bars->sched_item[slot]);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(bars->sched_empty[slot]));
            ++ss;
            if (it < 0) break;
            const WorkItem x = decode_item<kGeneral>(p, it, num_entries, kCausal);
            // the unit's key tile j is this CTA's key tile g = g0 + j, its V in ring chunks 5g + {3, 4}
            const uint32_t g0 = tiles_seen;
            tiles_seen += x.n_max;
            const int n_t = t ? x.n[1] : x.n[0];
            const bool row_valid = row < (t ? x.rows[1] : x.rows[0]);
            const int i = x.u0 + t * kBM + row;  // query row within the sequence
            T *orow = reinterpret_cast<T *>(p.out) + (long long)(x.q_tok0 + t * kBM + row) * p.out_st +
                      (long long)x.h * p.out_sh;
            // split-KV chunk of a unit with several: partial row at part_o / part_lse
            const long long prow = ((long long)x.e * p.head_num + x.h) * kUnitRows + t * kBM + row;
            if (n_t == 0) {
                if (row_valid) {
                    if (kGeneral && x.nsplit > 1) {
                        p.part_lse[prow] = -INFINITY;  // no key of this chunk is visible to the row
                    } else {
                        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int c = 0; c < kDn * 2 / 16; ++c) reinterpret_cast<uint4 *>(orow)[c] = z;
                    }
                }
                continue;
            }
            const int lim_row = kCausal ? min(i + x.off + 1, x.lk) : x.lk;  // keys [0, lim_row) visible
            const int tile_q0 = x.u0 + t * kBM;
            float m_run = -INFINITY, l_run = 0.f;
            for (int j = 0; j < n_t; ++j) {
                // Keys past Lk have p = 0, but 0 * (NaN or Inf) is NaN: where those V rows may hold
                // anything, this thread zeroes key row `row` of V_j once it has landed (both
                // warpgroups write the same zeros; P V_j is issued only after this warpgroup's
                // P-ready arrival for this tile, and the chunk is refilled only after that MMA).
                if (kGeneral && (x.j0 + j + 1) * kBN > x.lk) {
                    const uint32_t g = g0 + j, vch = 5 * g + kKChunks + (row >> 6);
                    ok = wait_bar_warp(bar(bars->v_full[g % kTileBars]), (g / kTileBars) & 1, bars, p.status);
                    if (!ok) break;
                    if ((x.j0 + j) * kBN + row >= x.lk) {
                        uint4 *vr = reinterpret_cast<uint4 *>(smem + kSmemRing + (vch % kRing) * kChunkBytes +
                                                              (row & 63) * 128);
                        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            vr[e] = z;
                            vr[kVHalfBytes / 16 + e] = z;
                        }
                        ptx::fence_proxy_async_smem();
                    }
                }
                ok = wait_bar_warp(bar(bars->s_full[t]), sf & 1, bars, p.status);
                ++sf;
                if (!ok) break;
                ptx::tc_fence_after();
                float s[kBN];
                {
                    uint32_t r0[64], r1[64];
                    ptx::tmem_ld64(tS, r0);
                    ptx::tmem_ld64(tS + 64, r1);
                    ptx::tmem_wait_ld_dep64(r0);
                    ptx::tmem_wait_ld_dep64(r1);
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        s[e] = __uint_as_float(r0[e]);
                        s[64 + e] = __uint_as_float(r1[e]);
                    }
                }
                const int kv0 = (x.j0 + j) * kBN;
                const bool tile_masked = (kv0 + kBN > x.lk) || (kCausal && kv0 + kBN - 1 > tile_q0 + x.off);
                float m_tile;
                if (kPositiveScale) {
                    if (tile_masked) {
                        const int lim = lim_row - kv0;
#pragma unroll
                        for (int c = 0; c < kBN; ++c) s[c] = c < lim ? s[c] : -INFINITY;
                    }
                    m_tile = row_max(s) * sl2;
                } else {
                    const int lim = tile_masked ? lim_row - kv0 : kBN;
#pragma unroll
                    for (int c = 0; c < kBN; ++c) s[c] = c < lim ? s[c] * sl2 : -INFINITY;
                    m_tile = row_max(s);
                }
                // Lazy rescaling: keep the old reference max unless the new one is 2^8 larger.
                float alpha = 1.f;
                if (m_tile > m_run + 8.f) {
                    alpha = ptx::ex2(m_run - m_tile);  // 0 when m_run = -inf
                    m_run = m_tile;
                }
                const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
                // p = 2^(s * scale * log2 e - m): one packed FMA per pair, packed partial sums,
                // one 16-bit pair conversion per pair.
                const float2 sc2 = kPositiveScale ? make_float2(sl2, sl2) : make_float2(1.f, 1.f);
                const float2 nm2 = make_float2(-m_use, -m_use);
                uint32_t pk[64];
                const float rowsum = exp_pack_sum<T>(s, sc2, nm2, pk);
                ptx::tmem_st64(tS + kTmemPOff, pk);
                // O_t holds P(j-1) V(j-1) already (the MMAs behind S_t(j) have completed);
                // rescale it before PV_t(j) may start.
                if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                    const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                    for (int c = 0; c < kDn / 64; ++c) {
                        uint32_t r[64];
                        ptx::tmem_ld64(tO + c * 64, r);
                        ptx::tmem_wait_ld_dep64(r);
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const float2 v2 = ptx::fmul2(
                                make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1])), a2);
                            r[2 * e] = __float_as_uint(v2.x);
                            r[2 * e + 1] = __float_as_uint(v2.y);
                        }
                        ptx::tmem_st64(tO + c * 64, r);
                    }
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(bar(bars->p_full[t]));
                l_run = l_run * alpha + rowsum;
            }
            if (!ok) break;
            // Epilogue: O / l -> 16-bit, one 256-byte row per thread.
            ok = wait_bar_warp(bar(bars->o_full[t]), of & 1, bars, p.status);
            ++of;
            if (!ok) break;
            ptx::tc_fence_after();
            const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
            if (kGeneral && x.nsplit > 1) {
                // O / l in fp32 and log2(sum 2^s') = m + log2(l) over this chunk's keys
                float *po = p.part_o + prow * kDn;
#pragma unroll
                for (int c = 0; c < kDn / 32; ++c) {
                    uint32_t r[32];
                    ptx::tmem_ld32(tO + c * 32, r);
                    ptx::tmem_wait_ld_dep(r);
                    if (row_valid) {
                        float4 *dst = reinterpret_cast<float4 *>(po + c * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(r[4 * e]) * inv_l, __uint_as_float(r[4 * e + 1]) * inv_l,
                                                 __uint_as_float(r[4 * e + 2]) * inv_l,
                                                 __uint_as_float(r[4 * e + 3]) * inv_l);
                    }
                }
                if (row_valid) p.part_lse[prow] = l_run > 0.f ? m_run + log2f(l_run) : -INFINITY;
                ptx::tc_fence_before();
                ptx::mbar_arrive(bar(bars->o_empty[t]));
                continue;
            }
#pragma unroll
            for (int c = 0; c < kDn / 32; ++c) {
                uint32_t r[32];
                ptx::tmem_ld32(tO + c * 32, r);
                ptx::tmem_wait_ld_dep(r);
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = DType<T>::pack(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
                if (row_valid) store_row_chunk(orow + c * 32, w, p.out_v8);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar(bars->o_empty[t]));
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Split-KV combine: for each unit with several chunks and each head, merges the
// chunks' partial rows (O_c / l_c in fp32 and lse_c = log2 sum_j 2^s'_j) as
//   O = sum_c 2^(lse_c - M) (O_c / l_c) / sum_c 2^(lse_c - M),  M = max_c lse_c,
// the same softmax over the union of the chunks' keys.  One warp per row, four
// channels per lane; a row no chunk saw any key of is written as zeros.
// ---------------------------------------------------------------------------
constexpr int kCombineThreads = 256;
constexpr int kCombineRowGroups = 8;  // blockIdx.z: rows [z * 32, z * 32 + 32) of the unit

struct CombineParams {
    const int4 *seq_info;
    const int2 *units;
    const int *num_units;
    const int *split_off;  // [units + 1] first entry of each unit
    const float *part_o, *part_lse;
    void *out;
    long long out_st, out_sh;
    int head_num;
};

template <typename T>
__global__ void __launch_bounds__(kCombineThreads) mla_split_combine_kernel(const CombineParams c) {
    const int u = blockIdx.x, h = blockIdx.y;
    if (u >= *c.num_units) return;
    const int e0 = c.split_off[u], ns = c.split_off[u + 1] - e0;
    if (ns <= 1) return;  // the attention kernel wrote this unit's rows itself
    const int2 bm = c.units[u];
    const int4 s = c.seq_info[bm.x];
    const int u0 = bm.y * kUnitRows;
    const int rows = min(kUnitRows, s.z - u0);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r_end = min(rows, (int)(blockIdx.z + 1) * (kUnitRows / kCombineRowGroups));
    for (int r = blockIdx.z * (kUnitRows / kCombineRowGroups) + warp; r < r_end; r += kCombineThreads / 32) {
        const long long base = (long long)e0 * c.head_num * kUnitRows + (long long)h * kUnitRows + r;
        const long long step = (long long)c.head_num * kUnitRows;  // between chunks of the same row
        // every chunk's log-sum-exp at once (lane k holds chunk k0 + k), then the warp maximum
        float m = -INFINITY;
        for (int k0 = 0; k0 < ns; k0 += 32)
            if (k0 + lane < ns) m = fmaxf(m, c.part_lse[base + (k0 + lane) * step]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float wsum = 0.f;
        if (m != -INFINITY) {
            for (int k0 = 0; k0 < ns; k0 += 32) {
                const float l = k0 + lane < ns ? c.part_lse[base + (k0 + lane) * step] : -INFINITY;
                const float wl = l == -INFINITY ? 0.f : exp2f(l - m);  // 0: that chunk saw no key of the row
                const int kn = min(32, ns - k0);
#pragma unroll 4
                for (int k = 0; k < kn; ++k) {
                    const float w = __shfl_sync(0xffffffffu, wl, k);
                    if (w == 0.f) continue;
                    const float4 o = reinterpret_cast<const float4 *>(c.part_o + (base + (k0 + k) * step) * kDn)[lane];
                    acc.x = fmaf(w, o.x, acc.x);
                    acc.y = fmaf(w, o.y, acc.y);
                    acc.z = fmaf(w, o.z, acc.z);
                    acc.w = fmaf(w, o.w, acc.w);
                    wsum += w;
                }
            }
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        T *orow = reinterpret_cast<T *>(c.out) + (long long)(s.x + u0 + r) * c.out_st + (long long)h * c.out_sh;
        const uint32_t lo = DType<T>::pack(acc.x * inv, acc.y * inv), hi = DType<T>::pack(acc.z * inv, acc.w * inv);
        reinterpret_cast<uint2 *>(orow)[lane] = make_uint2(lo, hi);
    }
}

// ---------------------------------------------------------------------------
// Diagnostic: the pipeline's bounded wait on an mbarrier that nothing arrives at.
// It gives up after limit_ns, records kStatusTimeout in the status word and
// returns -- the path every role of the attention kernel takes when a wait runs
// out -- so that a test can check the timeout reporting without a real fault.
// ---------------------------------------------------------------------------
__global__ void mla_selftest_wait_kernel(int *status, unsigned long long limit_ns) {
    __shared__ Barriers b;
    if (threadIdx.x == 0) {
        ptx::mbar_init(ptx::smem_addr(&b.drain), 1);
        b.abort = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    // phase 0 of a fresh barrier completes only when someone arrives: nobody does
    wait_bar_warp(ptx::smem_addr(&b.drain), 0, &b, status, limit_ns);
}

}  // namespace mla
