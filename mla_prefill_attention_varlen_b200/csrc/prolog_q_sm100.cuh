// q projection of the MLA Prolog with its per-head RmsNorm and RoPE as the GEMM's epilogue (sm_100a,
// clusters of two CTAs).  The "MlaProlog" page of cann-recipes-infer (计算公式 section) defines, for
// each token row c of c^Q [t, r] and head h of wq_b [r, H*d]:
//   v        = c wq_b[:, h*d : (h+1)*d]                    (d channels, fp32 accumulation)
//   q[h]     = v / sqrt(mean(v^2) + eps)                   (RmsNorm, weight 1)
//   q[h, d-R+2i], q[h, d-R+2i+1] = the interleaved rotation of that pair by the token's cos / sin rows
//   rope_cos / rope_sin [t, R]:  y[2i] = v[2i] cos[2i] - v[2i+1] sin[2i],  y[2i+1] = v[2i+1] cos[2i+1] + v[2i] sin[2i+1]
// and q is written as bf16.  The norm needs the whole head row, so a tile is 256 tokens x one head:
// each CTA of the pair holds 128 token rows x d fp32 accumulators in its tensor memory (d <= 512
// columns), and the row never leaves the SM in fp32.
//
// Operands: A = c^Q rows (K-major: r contiguous), B = wq_b (MN-major: the head's d columns
// contiguous).  The MMAs are tcgen05 cta_group::2 with M = 256 (128 rows in each CTA) and N = nc
// (256 when d is a multiple of 256, else 128): B is split along N, so for N-chunk c each CTA loads
// its nc/2 columns c*nc + rank*nc/2 + [0, nc/2).  A stage is 64 channels of r for one N-chunk: per
// CTA 16 KB of A (128 rows x 128 B) and nc/128 blocks of 8 KB of B (64 rows of r x 64 columns,
// 128-byte swizzled); six stages in flight.  A tile runs chunk by chunk (A is read once per chunk),
// and the head's two channel halves have their own accumulated / read-back barriers, so the next
// tile's first chunk starts as soon as the epilogue has read the first half.  The epilogue writes q through shared memory: each 32-column block of a
// half (128 rows x 64 B, 64-byte swizzled; two buffers per half) is stored by a TMA tensor store,
// so the output leaves in whole 64-byte row segments, a store overlaps the next block's work, and
// rows past the last token are clipped by the store.
//
//   leader   warp 0: TMA loads of its A rows and B halves; warp 1: MMA issuer for the pair
//   follower warp 0: TMA loads of its halves; warp 1: relay of its full barriers to the leader's
//   both     warps 4-11: epilogue, two warps per tensor-memory lane quarter, each owning a quarter
//            of the head's d channels of its 32 rows (d/4 columns of each half).  Once half 0 is
//            accumulated the warp copies its columns into registers and hands the half back at
//            once, so the next tile's first N-chunk runs during the rest of the epilogue; once half
//            1 is accumulated it adds that half's squares, the two warps' sums meet through shared
//            memory (an mbarrier per lane quarter), and it scales (and rotates), converts and
//            stages 32-column blocks: half 0 from registers, half 1 from tensor memory (64 columns
//            per load), releasing half 1 after its last load
//            warps 2, 3: TMA stores of the staged blocks of warps 4-7 / 8-11
// Tiles are static (tile = cluster + i * clusters, head-major so that concurrent clusters share a
// head's wq_b columns in L2).  The kernel is instantiated per head size (d = 128, 256, 384, 512).
// Every wait is bounded; a timeout sets the status word and aborts both CTAs.
#pragma once

#include "mla_prefill_sm100.cuh"

namespace mla {
namespace prolog {

constexpr int kThreads = 384;
constexpr int kTileTokens = 256;   // rows of one pair MMA (128 per CTA)
constexpr int kStageK = 64;        // channels of r per stage (one 128-byte swizzle row of A)
constexpr int kStages = 6;
constexpr int kABytes = 128 * kStageK * 2;  // 16 KB: this CTA's 128 rows of the stage
constexpr int kBBlock = 64 * kStageK * 2;   // 8 KB: 64 columns of wq_b x the stage's 64 rows
constexpr int kMaxBBlocks = 2;              // one N-chunk per stage: nc / 128 blocks per CTA
constexpr int kStageBytes = kABytes + kMaxBBlocks * kBBlock;
constexpr int kOutCols = 32;                   // output block: 32 columns (64 B) x 128 rows
constexpr int kStageOut = 128 * kOutCols * 2;   // 8 KB
constexpr int kSmemStages = 0;
constexpr int kSmemOut = kSmemStages + kStages * kStageBytes;  // two output blocks per half
constexpr int kSmemBar = kSmemOut + 4 * kStageOut;
constexpr int kSmemXss = kSmemBar + 256;      // per-row partial sums of squares, one per half
constexpr int kSmemBytes = kSmemXss + 2 * 128 * 4;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024 B
static_assert(kSmemAlloc <= 232448, "shared memory per CTA");
constexpr int kEpiWarps = 8;
// warpgroup 0 (producer, MMA issuer / relay, store warps) gives registers to the two epilogue
// warpgroups, which hold their columns of half 0 (up to 128 per thread) across the second half's
// accumulation; the split stays within the 168 registers per thread the block is launched with
constexpr int kRegsLow = 72;
constexpr int kRegsEpi = 216;
static_assert(kRegsLow * 128 + kRegsEpi * 256 <= 65536 / kThreads / 8 * 8 * kThreads,
              "register split exceeds the launch's register file share");
constexpr int kHalfFreeArrivals = 2 * kEpiWarps;  // every epilogue warp of both CTAs reads part of each half
constexpr uint64_t kWaitLimitNs = 200000000ull;   // 200 ms

struct QParams {
    const __nv_bfloat16 *cos, *sin;  // [tokens, R] with row strides cos_tok / sin_tok
    long long cos_tok, sin_tok;
    int tokens;      // rows of this launch
    int heads;       // H
    int d;           // head_dim: a multiple of 128, <= 512
    int nc;          // MMA N per chunk: 256 or 128
    int rope;        // R (a multiple of 32, <= d)
    int k_stages;    // r / 64
    float eps;
    int *status;
};

struct Bars {
    uint64_t full[kStages], empty[kStages];
    uint64_t half_full[2], half_free[2];  // the head's channel halves: accumulated / read by the epilogue
    uint64_t xready[4];  // per lane quarter: both halves' sums of squares are in shared memory
    uint64_t st_full[2][2], st_empty[2][2];  // [half][buffer]: staged by the half's 4 warps / read by its store
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block too large");

// Bounded wait on a phase; on timeout records the status, raises both CTAs' abort flags.
__device__ __forceinline__ bool qwait(uint32_t bar, uint32_t parity, Bars *bars, uint32_t peer_abort, int *status) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (*reinterpret_cast<volatile int *>(&bars->abort)) return false;
            if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
                *reinterpret_cast<volatile int *>(&bars->abort) = 1;
                ptx::st_shared_cluster_u32(peer_abort, 1u);
                atomicCAS(status, 0, kStatusTimeout);
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool qwait_warp(uint32_t bar, uint32_t parity, Bars *bars, uint32_t peer_abort,
                                           int *status) {
    const bool ok = qwait(bar, parity, bars, peer_abort, status);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void qwait_landed(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity))
        if (ptx::globaltimer_ns() - t0 > 100000000ull) return;
}

// One 32-column output block of a row: scale by the row's norm (two lanes per multiply) and, for
// kRot, rotate the interleaved pairs by the row's cos / sin values (cs, sn: the block's 32 entries);
// pack to bf16.
template <bool kRot>
__device__ __forceinline__ void scale_block(const uint32_t *cur, float inv, const __nv_bfloat16 *cs,
                                            const __nv_bfloat16 *sn, uint32_t (&w)[16]) {
    const float2 inv2 = make_float2(inv, inv);
    if constexpr (kRot) {
        uint4 cv[4], sv[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            cv[v] = __ldg(reinterpret_cast<const uint4 *>(cs) + v);
            sv[v] = __ldg(reinterpret_cast<const uint4 *>(sn) + v);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float2 xy = ptx::fmul2(make_float2(__uint_as_float(cur[2 * e]), __uint_as_float(cur[2 * e + 1])), inv2);
            const uint32_t cw = reinterpret_cast<const uint32_t *>(&cv[e >> 2])[e & 3];
            const uint32_t sw = reinterpret_cast<const uint32_t *>(&sv[e >> 2])[e & 3];
            const float2 c2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&cw));
            const float2 s2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&sw));
            w[e] = DType<__nv_bfloat16>::pack(xy.x * c2.x - xy.y * s2.x, xy.y * c2.y + xy.x * s2.y);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float2 xy = ptx::fmul2(make_float2(__uint_as_float(cur[2 * e]), __uint_as_float(cur[2 * e + 1])), inv2);
            w[e] = DType<__nv_bfloat16>::pack(xy.x, xy.y);
        }
    }
}

template <int kD>
__global__ void __launch_bounds__(kThreads, 1)
    mla_prolog_q_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_o /* q_out {d, H, tokens} */, const QParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars *bars = reinterpret_cast<Bars *>(smem + kSmemBar);
    float *xss = reinterpret_cast<float *>(smem + kSmemXss);
    const uint32_t sStages = ptx::smem_addr(smem + kSmemStages);
    const uint32_t sOut = ptx::smem_addr(smem + kSmemOut);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t cta = ptx::cluster_ctarank();
    const bool leader = cta == 0;
    auto bar = [&](uint64_t &b) { return ptx::smem_addr(&b); };
    auto lead_bar = [&](uint64_t &b) { return ptx::mapa_shared(ptx::smem_addr(&b), 0); };
    const uint32_t peer_abort = ptx::mapa_shared(ptx::smem_addr(&bars->abort), cta ^ 1u);

    if (threadIdx.x == 32) {
        ptx::tma_prefetch_desc(&tm_a);
        ptx::tma_prefetch_desc(&tm_b);
        ptx::tma_prefetch_desc(&tm_o);
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar(bars->full[s]), leader ? 2 : 1);
            ptx::mbar_init(bar(bars->empty[s]), 1);
        }
        for (int hh = 0; hh < 2; ++hh) {
            ptx::mbar_init(bar(bars->half_full[hh]), 1);
            ptx::mbar_init(bar(bars->half_free[hh]), kHalfFreeArrivals);
        }
        for (int q = 0; q < 4; ++q) ptx::mbar_init(bar(bars->xready[q]), 2);
        for (int hh = 0; hh < 2; ++hh)
            for (int b = 0; b < 2; ++b) {
                ptx::mbar_init(bar(bars->st_full[hh][b]), 4);
                ptx::mbar_init(bar(bars->st_empty[hh][b]), 1);
            }
        bars->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(ptx::smem_addr(&bars->tmem_base), kTmemCols);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    ptx::cluster_sync_all();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    static_assert(kD % 128 == 0 && kD >= 128 && kD <= 512, "head_dim");
    constexpr int kNc = kD % 256 == 0 ? 256 : 128;  // MMA N per chunk
    constexpr int chunk_blocks = kNc / 128;          // this CTA's 8 KB B blocks per stage (one N-chunk)
    constexpr int chunks = kD / kNc;
    constexpr int hd = kD / 2;                       // channels per half of the head
    const int n_tblocks = (p.tokens + kTileTokens - 1) / kTileTokens;
    const int n_tiles = n_tblocks * p.heads;
    const int cluster_id = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    const uint32_t stage_tx = kABytes + chunk_blocks * kBBlock;
    // Per tile the stages run N-chunk by N-chunk (all of r for chunk 0, then chunk 1, ...), so the
    // columns of the head's first half are accumulated, and can be handed back by the epilogue,
    // before those of its second half.
    const int stages_per_tile = chunks * p.k_stages;

    if (warp < 4) ptx::regs_dec<kRegsLow>();
    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ TMA producer (both CTAs)
            const uint64_t pol_a = ptx::policy_evict_last();  // c^Q rows: read by every head
            const uint64_t pol_b = ptx::policy_evict_last();  // wq_b columns: read by every token block
            uint32_t it = 0;  // stages issued
            bool ok = true;
            for (int tile = cluster_id; tile < n_tiles && ok; tile += n_clusters) {
                const int h = tile / n_tblocks, tb = tile - h * n_tblocks;
                const int row0 = tb * kTileTokens + static_cast<int>(cta) * 128;
                for (int c = 0; c < chunks && ok; ++c)
                    for (int ks = 0; ks < p.k_stages && ok; ++ks, ++it) {
                        const uint32_t s = it % kStages;
                        if (it >= kStages && !(ok = qwait(bar(bars->empty[s]), ((it / kStages) & 1) ^ 1, bars,
                                                          peer_abort, p.status)))
                            break;
                        const uint32_t fb = bar(bars->full[s]);
                        const uint32_t dst = sStages + s * kStageBytes;
                        ptx::mbar_arrive_expect_tx(fb, stage_tx);
                        ptx::tma_load_2d(dst, &tm_a, fb, ks * kStageK, row0, pol_a);
                        for (int b = 0; b < chunk_blocks; ++b) {
                            const int col = h * kD + c * kNc + static_cast<int>(cta) * (kNc / 2) + 64 * b;
                            ptx::tma_load_2d(dst + kABytes + b * kBBlock, &tm_b, fb, col, ks * kStageK, pol_b);
                        }
                    }
            }
            // every copy into this CTA lands before it may exit
            for (uint32_t i = it > kStages ? it - kStages : 0; i < it; ++i)
                qwait_landed(bar(bars->full[i % kStages]), (i / kStages) & 1);
        }
    } else if (warp == 1 && !leader) {
        // ------------------------------------------------------------ relay (follower)
        uint32_t it = 0;
        bool ok = true;
        for (int tile = cluster_id; tile < n_tiles && ok; tile += n_clusters)
            for (int k = 0; k < stages_per_tile && ok; ++k, ++it) {
                const uint32_t s = it % kStages;
                ok = qwait_warp(bar(bars->full[s]), (it / kStages) & 1, bars, peer_abort, p.status);
                if (ok && lane == 0) ptx::mbar_arrive_remote(lead_bar(bars->full[s]));
                __syncwarp();
            }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        constexpr uint32_t kHi = ptx::desc_hi_sw128(1024);
        constexpr uint32_t kId256 = ptx::instr_desc_f16(true, kTileTokens, 256, true);
        constexpr uint32_t kId128 = ptx::instr_desc_f16(true, kTileTokens, 128, true);
        constexpr uint16_t kBoth = 3;
        const uint32_t a_lo = ptx::desc_lo(sStages, 16);
        const uint32_t b_lo = ptx::desc_lo(sStages + kABytes, kBBlock);  // LBO: the chunk's next 64 columns
        constexpr uint32_t kStageU = kStageBytes >> 4;
        uint32_t it = 0, tl = 0;
        bool ok = true;
        for (int tile = cluster_id; tile < n_tiles && ok; tile += n_clusters, ++tl) {
            int waited = 0;  // halves whose previous-tile release this tile has waited for
            for (int c = 0; c < chunks && ok; ++c) {
                // the halves chunk c writes must have been read by the previous tile's epilogue
                const int h_lo = (c * kNc) / hd, h_hi = ((c + 1) * kNc - 1) / hd;
                for (int hh = h_lo; hh <= h_hi && ok; ++hh)
                    if (!(waited & (1 << hh))) {
                        ok = qwait_warp(bar(bars->half_free[hh]), (tl & 1) ^ 1, bars, peer_abort, p.status);
                        waited |= 1 << hh;
                    }
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(c * kNc);
                for (int ks = 0; ks < p.k_stages && ok; ++ks, ++it) {
                    const uint32_t s = it % kStages;
                    ok = qwait_warp(bar(bars->full[s]), (it / kStages) & 1, bars, peer_abort, p.status);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    if (ptx::elect_one()) {
                        const uint32_t a = a_lo + s * kStageU, b = b_lo + s * kStageU;
#pragma unroll
                        for (int k = 0; k < kStageK / 16; ++k) {
                            // 16 channels of r per MMA: 32 B along A's swizzled rows, 16 rows (2 KB) of B
                            const bool acc = ks > 0 || k > 0;
                            if constexpr (kNc == 256) {
                                if (acc) ptx::mma2_ss_lo<kHi, kId256, 1>(d, a + 2 * k, b + 128 * k);
                                else ptx::mma2_ss_lo<kHi, kId256, 0>(d, a + 2 * k, b + 128 * k);
                            } else {
                                if (acc) ptx::mma2_ss_lo<kHi, kId128, 1>(d, a + 2 * k, b + 128 * k);
                                else ptx::mma2_ss_lo<kHi, kId128, 0>(d, a + 2 * k, b + 128 * k);
                            }
                        }
                        ptx::mma_commit_pair(bar(bars->empty[s]), kBoth);  // the stage's operands are read
                        if (ks == p.k_stages - 1)  // halves whose last chunk this is are complete
                            for (int hh = h_lo; hh <= h_hi; ++hh)
                                if ((hh + 1) * hd <= (c + 1) * kNc) ptx::mma_commit_pair(bar(bars->half_full[hh]), kBoth);
                    }
                    __syncwarp();
                }
            }
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        ptx::regs_inc<kRegsEpi>();
        constexpr int kQ = hd / 2;         // columns of each half this warp owns (32 .. 128)
        constexpr int kBlocks = kQ / 32;   // its 32-column output blocks per half
        const int wq = warp & 3;           // tensor-memory lane quarter
        const int part = (warp - 4) >> 2;  // which quarter of each half: columns part * kQ + [0, kQ)
        const int row = wq * 32 + lane;    // row within this CTA's 128
        const uint32_t tcol = tmem + (static_cast<uint32_t>(wq * 32) << 16) + static_cast<uint32_t>(part * kQ);
        const int rope0 = kD - p.rope;     // first rotated channel
        constexpr float inv_d = 1.f / static_cast<float>(kD);
        uint32_t tl = 0, kb = 0;           // tiles; output blocks staged by this warp's buffers
        bool ok = true;
        for (int tile = cluster_id; tile < n_tiles && ok; tile += n_clusters, ++tl) {
            const int tb = tile % n_tblocks;
            const int token = tb * kTileTokens + static_cast<int>(cta) * 128 + row;
            // half 0: this warp's columns into registers, and the half goes straight back to the MMA warp
            uint32_t keep[kQ];
            float ss = 0.f;
            ok = qwait_warp(bar(bars->half_full[0]), tl & 1, bars, peer_abort, p.status);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int j = 0; j < kQ; j += 32)
                ptx::tmem_ld32(tcol + static_cast<uint32_t>(j), *reinterpret_cast<uint32_t (*)[32]>(keep + j));
#pragma unroll
            for (int j = 0; j < kQ; j += 32) ptx::tmem_wait_ld_dep(*reinterpret_cast<uint32_t (*)[32]>(keep + j));
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_remote(lead_bar(bars->half_free[0]));
#pragma unroll
            for (int e = 0; e < kQ; ++e) ss = fmaf(__uint_as_float(keep[e]), __uint_as_float(keep[e]), ss);
            // half 1: the squares of this warp's columns, 32 per load (the held half leaves few registers)
            ok = qwait_warp(bar(bars->half_full[1]), tl & 1, bars, peer_abort, p.status);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int j = 0; j < kQ; j += 32) {
                uint32_t r[32];
                ptx::tmem_ld32(tcol + static_cast<uint32_t>(hd + j), r);
                ptx::tmem_wait_ld_dep(r);
#pragma unroll
                for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(r[e]), __uint_as_float(r[e]), ss);
            }
            // the partner warp (same lane quarter) holds the other two quarters of these rows
            xss[part * 128 + row] = ss;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(bars->xready[wq]));
            ok = qwait_warp(bar(bars->xready[wq]), tl & 1, bars, peer_abort, p.status);
            if (!ok) break;
            const float total = xss[row] + xss[128 + row];
            const float inv = rsqrtf(total * inv_d + p.eps);
            const int tok_c = token < p.tokens ? token : 0;  // rows past the end: any valid cos / sin row
            const __nv_bfloat16 *cs = p.cos + static_cast<long long>(tok_c) * p.cos_tok;
            const __nv_bfloat16 *sn = p.sin + static_cast<long long>(tok_c) * p.sin_tok;
            // one 32-column block at column cc: scale (and rotate), pack, stage for the store warp
            auto emit = [&](int cc, const uint32_t *cur) {
                uint32_t w[16];
                if (cc >= rope0) scale_block<true>(cur, inv, cs + (cc - rope0), sn + (cc - rope0), w);
                else scale_block<false>(cur, inv, cs, sn, w);
                const uint32_t b = kb & 1, use = kb >> 1;
                const uint32_t buf = sOut + static_cast<uint32_t>((part * 2 + b) * kStageOut);
                // the buffer is free once the store of its previous block has read it
                if (use > 0 &&
                    !(ok = qwait_warp(bar(bars->st_empty[part][b]), (use - 1) & 1, bars, peer_abort, p.status)))
                    return;
#pragma unroll
                for (int v = 0; v < 4; ++v) {  // 16-byte chunk v of the row's 64 bytes, swizzled by (row / 2) mod 4
                    const uint32_t chunk = static_cast<uint32_t>(v ^ ((row >> 1) & 3));
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + row * 64 + chunk * 16),
                                 "r"(w[4 * v]), "r"(w[4 * v + 1]), "r"(w[4 * v + 2]), "r"(w[4 * v + 3])
                                 : "memory");
                }
                ptx::fence_proxy_async_smem();  // visible to the TMA store
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(bar(bars->st_full[part][b]));
                ++kb;
            };
            // the warp's last tensor-memory read of half 1 has completed: hand the half back
            auto release1 = [&]() {
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_remote(lead_bar(bars->half_free[1]));
            };
            // half 0 from registers
#pragma unroll
            for (int j = 0; j < kBlocks; ++j)
                if (ok) emit(part * kQ + 32 * j, keep + 32 * j);
            // half 1 from tensor memory, 64 columns (two blocks) per load
            const int c1 = hd + part * kQ;
#pragma unroll
            for (int j = 0; j < kBlocks; j += 2) {
                if (!ok) break;
                if (j + 1 < kBlocks) {
                    uint32_t r[64];
                    ptx::tmem_ld64(tcol + static_cast<uint32_t>(hd + 32 * j), r);
                    ptx::tmem_wait_ld_dep64(r);
                    if (j + 2 >= kBlocks) release1();
                    emit(c1 + 32 * j, r);
                    if (ok) emit(c1 + 32 * (j + 1), r + 32);
                } else {
                    uint32_t r[32];
                    ptx::tmem_ld32(tcol + static_cast<uint32_t>(hd + 32 * j), r);
                    ptx::tmem_wait_ld_dep(r);
                    release1();
                    emit(c1 + 32 * j, r);
                }
            }
        }
        ptx::tmem_wait_ld();  // a load left in flight by an aborted tile lands before the columns are freed
    } else if (warp >= 2) {
        // ---------------------------------------------------------------- q stores (both CTAs)
        // Warp 2 stores the blocks of the epilogue warps 4-7, warp 3 those of warps 8-11, in their
        // order: once the four warps have staged a block, one TMA tensor store; once the store
        // before it has read its buffer, that buffer is released.
        const int half = warp - 2;
        constexpr int nb = kD / 64;
        uint32_t kb = 0;
        bool ok = true;
        for (int tile = cluster_id; tile < n_tiles && ok; tile += n_clusters) {
            const int h = tile / n_tblocks, tb = tile - h * n_tblocks;
            for (int k = 0; k < nb && ok; ++k, ++kb) {
                const uint32_t b = kb & 1, use = kb >> 1;
                ok = qwait_warp(bar(bars->st_full[half][b]), use & 1, bars, peer_abort, p.status);
                if (!ok) break;
                if (lane == 0) {
                    const int cc = (k < nb / 2 ? 0 : hd) + half * (hd / 2) + (k % (nb / 2)) * kOutCols;
                    ptx::tma_store_3d(&tm_o, sOut + static_cast<uint32_t>((half * 2 + b) * kStageOut), cc, h,
                                      tb * kTileTokens + static_cast<int>(cta) * 128);
                    ptx::bulk_commit_group();
                    ptx::bulk_wait_group_read1();  // the previous block's store has read its buffer
                    if (kb > 0) ptx::mbar_arrive(bar(bars->st_empty[half][b ^ 1]));
                }
                __syncwarp();
            }
        }
        if (lane == 0) ptx::bulk_wait_group0();  // this CTA's q stores have completed
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync_all();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace prolog
}  // namespace mla
