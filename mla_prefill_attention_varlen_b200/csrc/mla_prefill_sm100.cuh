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
// Work unit: one 128-row query tile of one sequence for one query head.  Per
// unit the kernel walks 128-key tiles j = 0 .. n_kv-1 (tiles wholly above the
// causal diagonal are never visited):
//   MMA warp   S_j = [Qn|Qr] [Kn|Kr]_j^T   (12 MMAs 128x128x16 into TMEM, the
//              nope and rope k-steps accumulate into the same accumulator)
//              O  += P_{j-1} V_{j-1}        (8 MMAs, P read from TMEM)
//   softmax    rows of S_j -> mask -> running max / sum -> P_j (16-bit) in TMEM,
//              lazy rescale of O when the running max grows by more than 2^8
//   load warp  TMA tiles of Q (once per unit), K_j and V_j (2-deep rings)
// Tensor memory (512 columns): S double buffer [0,256), O [256,384),
// P double buffer [384,512) (16-bit pairs packed per 32-bit column).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace mla {

constexpr int kBM = 128;  // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;  // keys per tile
constexpr int kDn = 128;  // nope width of Q/K, width of V (embeddimV)
constexpr int kDr = 64;   // rope width

constexpr int kChunkBytes = 128 * 64 * 2;  // one [128 rows x 64 cols] 16-bit block, 128-B swizzled
constexpr int kQBytes = 3 * kChunkBytes;   // Qn cols 0-63, Qn cols 64-127, Qr
constexpr int kKBytes = 3 * kChunkBytes;   // Kn cols 0-63, Kn cols 64-127, Kr
constexpr int kVBytes = 2 * kChunkBytes;   // V cols 0-63, V cols 64-127
constexpr int kKStages = 2;
constexpr int kVStages = 2;

constexpr int kSmemQ = 0;
constexpr int kSmemK = kSmemQ + kQBytes;
constexpr int kSmemV = kSmemK + kKStages * kKBytes;
constexpr int kSmemBar = kSmemV + kVStages * kVBytes;
constexpr int kSmemBytes = kSmemBar + 256;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024 B

constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemO = 256;
constexpr uint32_t kTmemP = 384;
constexpr uint32_t kTmemCols = 512;

constexpr int kThreads = 192;  // warp 0: TMA, warp 1: MMA + TMEM owner, warps 2-5: softmax / epilogue

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // a pipeline wait gives up after 2 s

// Status codes the device writes (mirror mla_status in include/mla_prefill.h).
constexpr int kStatusSeqlen = 8;
constexpr int kStatusTimeout = 9;

struct Params {
    const int4 *seq_info;  // per sequence {cq, ck, lq, lk} after clamping
    const int2 *tiles;     // (sequence, query-tile) pairs, most key tiles first
    const int *num_tiles;  // number of valid entries in tiles
    int *status;           // sticky device status word
    void *out;
    long long out_st, out_sh;  // token / head strides of out, elements
    int head_num;
    int group;  // head_num / kv_head_num
    float scale_log2;  // qk_scale * log2(e)
};

struct Barriers {
    uint64_t q_full, q_empty;
    uint64_t k_full[kKStages], k_empty[kKStages];
    uint64_t v_full[kVStages], v_empty[kVStages];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2];
    uint64_t o_done, o_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Barriers) <= 256, "barrier block too large");

// Number of 128-key tiles a query tile touches: the keys visible to its last
// row (causal) or all keys.  0 when no row sees any key.
__host__ __device__ __forceinline__ int kv_tiles_for(int q0, int rows, int lq, int lk, bool causal) {
    const int kv_end = causal ? min(q0 + rows + (lk - lq), lk) : lk;
    return kv_end > 0 ? (kv_end + kBN - 1) / kBN : 0;
}

struct WorkItem {
    int h, kh;
    int q_tok0, k_tok0;  // first packed token of the query tile / of the sequence's keys
    int q0;              // first query row of the tile within its sequence
    int rows;            // valid query rows in the tile (<= 128)
    int off;             // Lk - Lq
    int lk;
    int n_kv;
};

__device__ __forceinline__ WorkItem decode_item(const Params &p, int it, bool causal) {
    const int tile = it / p.head_num;
    WorkItem x;
    x.h = it - tile * p.head_num;
    x.kh = x.h / p.group;
    const int2 bm = p.tiles[tile];
    const int4 s = p.seq_info[bm.x];
    x.q0 = bm.y * kBM;
    x.rows = min(kBM, s.z - x.q0);
    x.q_tok0 = s.x + x.q0;
    x.k_tok0 = s.y;
    x.off = s.w - s.z;
    x.lk = s.w;
    x.n_kv = kv_tiles_for(x.q0, x.rows, s.z, s.w, causal);
    return x;
}

// Bounded mbarrier wait.  Gives up (and makes every role give up) when another
// role has aborted or after kWaitLimitNs, recording kStatusTimeout.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, Barriers *bars, int *status) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (*reinterpret_cast<volatile int *>(&bars->abort)) return false;
            if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
                *reinterpret_cast<volatile int *>(&bars->abort) = 1;
                atomicCAS(status, 0, kStatusTimeout);
                return false;
            }
        }
    }
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

// ---------------------------------------------------------------------------
// Plan kernel: one block of 1024 threads.  Clamps the seqlens to the tensor
// extents (recording kStatusSeqlen on any inconsistency), writes per-sequence
// offsets, and writes the (sequence, query tile) list sorted by descending
// number of key tiles (a counting sort; ties in arbitrary order).
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

__global__ void __launch_bounds__(kPlanThreads) mla_plan_kernel(const int *__restrict__ q_seqlen,
                                                                const int *__restrict__ kv_seqlen, int batch,
                                                                long long t_q, long long t_k, int causal,
                                                                int4 *seq_info, int *tile_off, int *hist,
                                                                int hist_len, int2 *tiles, int *num_tiles,
                                                                int *status) {
    __shared__ long long warp_sums[32];
    __shared__ int bad;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();

    // 1. clamped prefix sums and query-tile counts, in chunks of blockDim.x sequences
    long long carry_q = 0, carry_k = 0, carry_t = 0;
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
        const long long ck = pk < t_k ? pk : t_k, ek = pk + lk < t_k ? pk + lk : t_k;
        if (b < batch && (eq - cq != lq || ek - ck != lk)) bad = 1;
        const int lqc = static_cast<int>(eq - cq), lkc = static_cast<int>(ek - ck);
        const long long nt = (b < batch) ? (lqc + kBM - 1) / kBM : 0;
        long long tot_t;
        const long long pt = carry_t + block_exclusive_scan(nt, tot_t, warp_sums);
        if (b < batch) {
            seq_info[b] = make_int4(static_cast<int>(cq), static_cast<int>(ck), lqc, lkc);
            tile_off[b] = static_cast<int>(pt);
        }
        carry_q += tot_q;
        carry_k += tot_k;
        carry_t += tot_t;
    }
    const int total_tiles = static_cast<int>(carry_t);
    if (threadIdx.x == 0) tile_off[batch] = total_tiles;
    for (int c = threadIdx.x; c < hist_len; c += blockDim.x) hist[c] = 0;
    __syncthreads();

    // 2. histogram of key-tile counts
    for (int t = threadIdx.x; t < total_tiles; t += blockDim.x) {
        int lo = 0, hi = batch - 1;  // last b with tile_off[b] <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tile_off[mid] <= t) lo = mid; else hi = mid - 1;
        }
        const int4 s = seq_info[lo];
        const int m = t - tile_off[lo];
        const int q0 = m * kBM;
        const int cost = kv_tiles_for(q0, min(kBM, s.z - q0), s.z, s.w, causal != 0);
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
    for (int t = threadIdx.x; t < total_tiles; t += blockDim.x) {
        int lo = 0, hi = batch - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (tile_off[mid] <= t) lo = mid; else hi = mid - 1;
        }
        const int4 s = seq_info[lo];
        const int m = t - tile_off[lo];
        const int q0 = m * kBM;
        const int cost = kv_tiles_for(q0, min(kBM, s.z - q0), s.z, s.w, causal != 0);
        const int pos = atomicAdd(&hist[min(cost, hist_len - 1)], 1);
        tiles[pos] = make_int2(lo, m);
    }
    if (threadIdx.x == 0) {
        *num_tiles = total_tiles;
        if (bad) atomicCAS(status, 0, kStatusSeqlen);
    }
}

// Max of a 128-element row as a balanced tree (short dependency chains).
__device__ __forceinline__ float row_max(const float (&s)[kBN]) {
    float m[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) m[i] = fmaxf(s[i], s[i + 16]);
#pragma unroll
    for (int c = 32; c < kBN; c += 16) {
#pragma unroll
        for (int i = 0; i < 16; ++i) m[i] = fmaxf(m[i], s[c + i]);
    }
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1) {
#pragma unroll
        for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
    }
    return m[0];
}

// ---------------------------------------------------------------------------
// Attention kernel
// ---------------------------------------------------------------------------
template <typename T, bool kCausal, bool kPositiveScale>
__global__ void __launch_bounds__(kThreads, 1)
    mla_prefill_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                             const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kr,
                             const __grid_constant__ CUtensorMap tm_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Barriers *bars = reinterpret_cast<Barriers *>(smem + kSmemBar);
    const uint32_t sQ = ptx::smem_addr(smem + kSmemQ);
    const uint32_t sK = ptx::smem_addr(smem + kSmemK);
    const uint32_t sV = ptx::smem_addr(smem + kSmemV);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    auto bar = [&](uint64_t &b) { return ptx::smem_addr(&b); };

    if (threadIdx.x == 0) {
        ptx::mbar_init(bar(bars->q_full), 1);
        ptx::mbar_init(bar(bars->q_empty), 1);
        for (int s = 0; s < kKStages; ++s) {
            ptx::mbar_init(bar(bars->k_full[s]), 1);
            ptx::mbar_init(bar(bars->k_empty[s]), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            ptx::mbar_init(bar(bars->v_full[s]), 1);
            ptx::mbar_init(bar(bars->v_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            ptx::mbar_init(bar(bars->s_full[s]), 1);
            ptx::mbar_init(bar(bars->s_empty[s]), kBM);
            ptx::mbar_init(bar(bars->p_full[s]), kBM);
        }
        ptx::mbar_init(bar(bars->o_done), 1);
        ptx::mbar_init(bar(bars->o_empty), kBM);
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

    const int n_items = *p.num_tiles * p.head_num;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tm_q);
            ptx::tma_prefetch_desc(&tm_qr);
            ptx::tma_prefetch_desc(&tm_k);
            ptx::tma_prefetch_desc(&tm_kr);
            ptx::tma_prefetch_desc(&tm_v);
            const uint64_t pol_q = ptx::policy_evict_first();
            const uint64_t pol_kv = ptx::policy_evict_last();
            uint32_t qc = 0, kc = 0, vc = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                const WorkItem x = decode_item(p, it, kCausal);
                if (x.n_kv == 0) continue;
                ok = wait_bar(bar(bars->q_empty), (qc & 1) ^ 1, bars, p.status);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(bar(bars->q_full), kQBytes);
                ptx::tma_load_3d(sQ, &tm_q, bar(bars->q_full), 0, x.h, x.q_tok0, pol_q);
                ptx::tma_load_3d(sQ + kChunkBytes, &tm_q, bar(bars->q_full), 64, x.h, x.q_tok0, pol_q);
                ptx::tma_load_3d(sQ + 2 * kChunkBytes, &tm_qr, bar(bars->q_full), 0, x.h, x.q_tok0, pol_q);
                ++qc;
                auto load_k = [&](int j) -> bool {
                    const int s = kc % kKStages;
                    if (!wait_bar(bar(bars->k_empty[s]), ((kc / kKStages) & 1) ^ 1, bars, p.status)) return false;
                    const uint32_t dst = sK + s * kKBytes;
                    const int tok = x.k_tok0 + j * kBN;
                    ptx::mbar_arrive_expect_tx(bar(bars->k_full[s]), kKBytes);
                    ptx::tma_load_3d(dst, &tm_k, bar(bars->k_full[s]), 0, x.kh, tok, pol_kv);
                    ptx::tma_load_3d(dst + kChunkBytes, &tm_k, bar(bars->k_full[s]), 64, x.kh, tok, pol_kv);
                    ptx::tma_load_3d(dst + 2 * kChunkBytes, &tm_kr, bar(bars->k_full[s]), 0, x.kh, tok, pol_kv);
                    ++kc;
                    return true;
                };
                auto load_v = [&](int j) -> bool {
                    const int s = vc % kVStages;
                    if (!wait_bar(bar(bars->v_empty[s]), ((vc / kVStages) & 1) ^ 1, bars, p.status)) return false;
                    const uint32_t dst = sV + s * kVBytes;
                    const int tok = x.k_tok0 + j * kBN;
                    ptx::mbar_arrive_expect_tx(bar(bars->v_full[s]), kVBytes);
                    ptx::tma_load_3d(dst, &tm_v, bar(bars->v_full[s]), 0, x.kh, tok, pol_kv);
                    ptx::tma_load_3d(dst + kChunkBytes, &tm_v, bar(bars->v_full[s]), 64, x.kh, tok, pol_kv);
                    ++vc;
                    return true;
                };
                ok = load_k(0);
                for (int j = 0; j < x.n_kv && ok; ++j) {
                    if (j + 1 < x.n_kv) ok = load_k(j + 1);
                    if (ok) ok = load_v(j);
                }
            }
            // Let every copy this thread started land before the block can exit.
            if (qc) wait_bar(bar(bars->q_full), (qc - 1) & 1, bars, p.status);
            for (uint32_t s = 0; s < kKStages; ++s) {
                const uint32_t n = kc / kKStages + (s < kc % kKStages ? 1 : 0);
                if (n) wait_bar(bar(bars->k_full[s]), (n - 1) & 1, bars, p.status);
            }
            for (uint32_t s = 0; s < kVStages; ++s) {
                const uint32_t n = vc / kVStages + (s < vc % kVStages ? 1 : 0);
                if (n) wait_bar(bar(bars->v_full[s]), (n - 1) & 1, bars, p.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr bool kBf16 = DType<T>::kBf16;
            constexpr uint32_t idesc_qk = ptx::instr_desc_f16(kBf16, kBM, kBN, false);
            constexpr uint32_t idesc_pv = ptx::instr_desc_f16(kBf16, kBM, kDn, true);
            uint32_t qc = 0, kc = 0, vc = 0, sc = 0, oe = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
                const WorkItem x = decode_item(p, it, kCausal);
                if (x.n_kv == 0) continue;
                ok = wait_bar(bar(bars->q_full), qc & 1, bars, p.status);
                if (!ok) break;
                ++qc;
                ptx::tc_fence_after();
                for (int j = 0; j <= x.n_kv && ok; ++j) {
                    if (j < x.n_kv) {
                        // S_j = Q K_j^T over 192 channels: 2 nope chunks + 1 rope chunk, 4 k-steps each
                        const int ks = kc % kKStages;
                        const uint32_t sidx = sc + j, sb = sidx & 1;
                        ok = wait_bar(bar(bars->k_full[ks]), (kc / kKStages) & 1, bars, p.status) &&
                             wait_bar(bar(bars->s_empty[sb]), ((sidx >> 1) & 1) ^ 1, bars, p.status);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        const uint32_t d = tmem + kTmemS + sb * kBN;
                        const uint32_t kbase = sK + ks * kKBytes;
#pragma unroll
                        for (int c = 0; c < 3; ++c) {
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const uint64_t a = ptx::smem_desc_sw128(sQ + c * kChunkBytes + k * 32, 16, 1024);
                                const uint64_t b = ptx::smem_desc_sw128(kbase + c * kChunkBytes + k * 32, 16, 1024);
                                ptx::mma_ss(d, a, b, idesc_qk, (c | k) != 0);
                            }
                        }
                        ptx::mma_commit(bar(bars->k_empty[ks]));
                        ++kc;
                        ptx::mma_commit(bar(bars->s_full[sb]));
                        if (j == x.n_kv - 1) ptx::mma_commit(bar(bars->q_empty));
                    }
                    if (j >= 1) {
                        // O += P_{j-1} V_{j-1}: P from TMEM (A operand), V from shared memory (MN-major B)
                        const int t = j - 1;
                        const uint32_t pidx = sc + t, pb = pidx & 1;
                        const int vs = vc % kVStages;
                        ok = wait_bar(bar(bars->p_full[pb]), (pidx >> 1) & 1, bars, p.status) &&
                             wait_bar(bar(bars->v_full[vs]), (vc / kVStages) & 1, bars, p.status);
                        if (ok && t == 0) {
                            ok = wait_bar(bar(bars->o_empty), (oe & 1) ^ 1, bars, p.status);
                            ++oe;
                        }
                        if (!ok) break;
                        ptx::tc_fence_after();
                        const uint32_t vbase = sV + vs * kVBytes;
#pragma unroll
                        for (int k = 0; k < kBN / 16; ++k) {
                            const uint64_t b = ptx::smem_desc_sw128(vbase + k * 16 * 128, kChunkBytes, 1024);
                            ptx::mma_ts(tmem + kTmemO, tmem + kTmemP + pb * (kBN / 2) + k * 8, b, idesc_pv,
                                        (t > 0 || k > 0) ? 1u : 0u);
                        }
                        ptx::mma_commit(bar(bars->v_empty[vs]));
                        ++vc;
                        ptx::mma_commit(bar(bars->o_done));
                    }
                }
                sc += x.n_kv;
            }
            // Drain: wait until every MMA this thread issued has completed.
            ptx::mma_commit(bar(bars->drain));
            wait_bar(bar(bars->drain), 0, bars, p.status);
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int wq = warp & 3;           // TMEM lane quarter this warp may access
        const int row = wq * 32 + lane;    // query row within the tile
        const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
        const float sl2 = p.scale_log2;
        uint32_t sc = 0, od = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            const WorkItem x = decode_item(p, it, kCausal);
            const bool row_valid = row < x.rows;
            T *orow = reinterpret_cast<T *>(p.out) + (long long)(x.q_tok0 + row) * p.out_st +
                      (long long)x.h * p.out_sh;
            if (x.n_kv == 0) {
                if (row_valid) {
                    uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int c = 0; c < kDn * 2 / 16; ++c) reinterpret_cast<uint4 *>(orow)[c] = z;
                }
                continue;
            }
            const int i = x.q0 + row;
            const int lim_row = kCausal ? min(i + x.off + 1, x.lk) : x.lk;  // keys [0, lim_row) visible
            float m_run = -INFINITY, l_run = 0.f;
            for (int j = 0; j < x.n_kv; ++j) {
                const uint32_t sidx = sc + j, sb = sidx & 1;
                ok = wait_bar(bar(bars->s_full[sb]), (sidx >> 1) & 1, bars, p.status);
                if (!ok) break;
                ptx::tc_fence_after();
                float s[kBN];
                {
                    uint32_t r0[32], r1[32], r2[32], r3[32];
                    const uint32_t sa = tmem + lane_addr + kTmemS + sb * kBN;
                    ptx::tmem_ld32(sa, r0);
                    ptx::tmem_ld32(sa + 32, r1);
                    ptx::tmem_ld32(sa + 64, r2);
                    ptx::tmem_ld32(sa + 96, r3);
                    ptx::tmem_wait_ld_dep(r0);
                    ptx::tmem_wait_ld_dep(r1);
                    ptx::tmem_wait_ld_dep(r2);
                    ptx::tmem_wait_ld_dep(r3);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        s[e] = __uint_as_float(r0[e]);
                        s[32 + e] = __uint_as_float(r1[e]);
                        s[64 + e] = __uint_as_float(r2[e]);
                        s[96 + e] = __uint_as_float(r3[e]);
                    }
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(bar(bars->s_empty[sb]));

                const int kv0 = j * kBN;
                const bool tile_masked =
                    (kv0 + kBN > x.lk) || (kCausal && kv0 + kBN - 1 > x.q0 + x.off);
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
                uint32_t pk[kBN / 2];
                float psum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // independent partial sums
#pragma unroll
                for (int c = 0; c < kBN; c += 2) {
                    float p0, p1;
                    if (kPositiveScale) {
                        p0 = ptx::ex2(fmaf(s[c], sl2, -m_use));
                        p1 = ptx::ex2(fmaf(s[c + 1], sl2, -m_use));
                    } else {
                        p0 = ptx::ex2(s[c] - m_use);
                        p1 = ptx::ex2(s[c + 1] - m_use);
                    }
                    psum[(c / 2) & 7] += p0 + p1;
                    pk[c / 2] = DType<T>::pack(p0, p1);
                }
                if (j > 0) {
                    // O holds P_{j-1} V_{j-1} once o_done completes; P buffer sb is free again.
                    ok = wait_bar(bar(bars->o_done), od & 1, bars, p.status);
                    ++od;
                    if (!ok) break;
                    ptx::tc_fence_after();
                    if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
                        for (int c = 0; c < kDn / 32; ++c) {
                            uint32_t r[32];
                            const uint32_t taddr = tmem + lane_addr + kTmemO + c * 32;
                            ptx::tmem_ld32(taddr, r);
                            ptx::tmem_wait_ld_dep(r);
#pragma unroll
                            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                            ptx::tmem_st32(taddr, r);
                        }
                    }
                }
                const float rowsum = ((psum[0] + psum[1]) + (psum[2] + psum[3])) +
                                     ((psum[4] + psum[5]) + (psum[6] + psum[7]));
                l_run = l_run * alpha + rowsum;
#pragma unroll
                for (int c = 0; c < kBN / 2 / 32; ++c) {
                    uint32_t r[32];
#pragma unroll
                    for (int e = 0; e < 32; ++e) r[e] = pk[c * 32 + e];
                    ptx::tmem_st32(tmem + lane_addr + kTmemP + sb * (kBN / 2) + c * 32, r);
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(bar(bars->p_full[sb]));
            }
            if (!ok) break;
            sc += x.n_kv;
            // Epilogue: O / l -> 16-bit, one 256-byte row per thread.
            ok = wait_bar(bar(bars->o_done), od & 1, bars, p.status);
            ++od;
            if (!ok) break;
            ptx::tc_fence_after();
            const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
            for (int c = 0; c < kDn / 32; ++c) {
                uint32_t r[32];
                ptx::tmem_ld32(tmem + lane_addr + kTmemO + c * 32, r);
                ptx::tmem_wait_ld_dep(r);
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = DType<T>::pack(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
                if (row_valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar(bars->o_empty));
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace mla
