// CTA-pair variant of the varlen MLA prefill attention kernel (sm_100a, clusters of two CTAs).
//
// The operation is the one of mla_prefill_sm100.cuh (the "MLA Prefill" page of the Ascend
// Transformer Boost C API, AtbMLAPreFillGetWorkspaceSize members table): for sequence b, query
// head h, kv head kh = h / (headNum / kvHeadNum), row i and key j,
//   s_ij = qkScale * (Q_nope[i,h] . K_nope[j,kh] + Q_rope[i,h] . K_rope[j,kh]),
//   key j visible iff j <= i + (Lk - Lq) (causal, bottom-right),  O[i,h] = sum_j softmax_j(s_ij) V[j,kh].
//
// Two CTAs of a cluster (ranks 0 and 1, "leader" and "follower", on two SMs) share one work
// unit: 512 query rows of one sequence for one query head, in two groups t = 0, 1 of 256 rows
// (rows u0 + 256 t + [0, 128) in the leader, the next 128 in the follower).  The leader's MMA
// warp issues M = 256 tensor-core MMAs over the pair (tcgen05 cta_group::2): each CTA's tensor
// memory receives its own 128 rows, the A operand (Q or P) comes from each CTA's own shared or
// tensor memory, and the B operand (K for S, V for P V) is split along N: each CTA loads only
// its half of every key tile -- 64 of the 128 keys of K, 64 of the 128 columns of V.  Per CTA
// that halves the shared-memory bytes loaded per key tile and the B-operand bytes the tensor
// core reads per FLOP, and a single thread issues the MMAs of two SMs.
//
//   leader   warp 0: TMA loads of its halves; claims work items and hands them to both CTAs
//            warp 1: MMA issuer for the pair
//            warps 2, 3: helpers of groups 0, 1: for every step, once the group's S is ready,
//                    wait until the key tile's V and the next tile's K have landed in both CTAs
//                    and then arrive on the group's P-ready barrier, so that the MMA issuer waits
//                    for nothing but P-ready between its MMAs
//   follower warp 0: TMA loads of its halves (items received from the leader)
//            warp 1: relay: once each of its loads has landed (its own barrier), arrives on the
//                    leader's matching barrier, so the leader's MMAs see both halves
//   both     warps 4-7 / 8-11: softmax of group 0 / 1 over this CTA's 128 rows of the group,
//            P written to tensor memory, epilogue of this CTA's rows
//
// Every TMA load completes on a barrier of the CTA it writes to, so each CTA can wait for its
// own copies before it exits.  Commits of the pair MMAs arrive on the same barrier in both CTAs
// (multicast); P-ready and O-free arrivals of the follower's softmax warps go to the leader's
// barriers.  All waits are bounded; a timeout in either CTA aborts both.
#pragma once

#include "mla_prefill_sm100.cuh"

namespace mla {
namespace pair {

constexpr int kUnitRows = 512;          // query rows per work unit (two groups of 256)
constexpr int kGroupRows = 256;         // rows of one pair MMA (128 per CTA)
constexpr int kChunkBytes = 8192;       // one ring chunk: 64 rows x 128 B
constexpr int kRing = 16;               // ring chunks per CTA (128 KB)
constexpr int kKChunks = 3;             // this CTA's 64 keys: nope cols 0-63 | nope cols 64-127 | rope
constexpr int kVChunks = 2;             // keys 0-63 | keys 64-127, this CTA's 64 V columns each
constexpr int kTileChunks = kKChunks + kVChunks;
constexpr int kQTileBytes = 3 * 16384;  // this CTA's 128 rows of a group: nope lo | nope hi | rope
constexpr int kTileBars = 4;            // key-tile barrier sets
constexpr int kSched = 4;

constexpr int kSmemQ = 0;
constexpr int kSmemRing = kSmemQ + 2 * kQTileBytes;
constexpr int kSmemBar = kSmemRing + kRing * kChunkBytes;
constexpr int kSmemBytes = kSmemBar + 512;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024 B
static_assert(kSmemAlloc <= 232448, "shared memory per CTA");

// Arrivals the leader's sched_empty barrier collects per slot: its MMA warp, 2 helpers and 8
// softmax warps, the follower's producer, relay and 8 softmax warps.
constexpr int kSchedConsumers = 1 + 2 + 8 + 1 + 1 + 8;
constexpr int kSoftmaxWarpsPerPair = 8;  // per-warp O-free arrivals of one group, both CTAs
constexpr int kPReadyArrivals = kSoftmaxWarpsPerPair + 1;  // P_t(j) published by both CTAs, data seen by the helper

struct Barriers {
    // full barriers: the leader's count its own producer's arrival (with the bytes it loads) and
    // the follower relay's arrival; the follower's count its own producer's arrival only
    uint64_t q_full[2], q_empty[2];
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

// Bounded wait.  On timeout it records kStatusTimeout and raises the abort flag of both CTAs;
// every role of both gives up at its next wait.  kCluster: acquire at cluster scope, for the one
// phase whose guarded data is a plain shared-memory store from the peer CTA (the work item);
// every other phase guards tensor-memory or TMA data, ordered by the tcgen05 fences and the
// copies' completion mechanism, and is waited for at the default (CTA) scope.
template <bool kCluster = false>
__device__ __forceinline__ bool wait_pair(uint32_t bar, uint32_t parity, Barriers *bars, uint32_t peer_abort,
                                          int *status) {
    auto probe = [&]() { return kCluster ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity); };
    if (probe()) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (probe()) return true;
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

template <bool kCluster = false>
__device__ __forceinline__ bool wait_pair_warp(uint32_t bar, uint32_t parity, Barriers *bars, uint32_t peer_abort,
                                               int *status) {
    const bool ok = wait_pair<kCluster>(bar, parity, bars, peer_abort, status);
    return __all_sync(0xffffffffu, ok);
}

// Waits, up to 100 ms and whether or not the kernel is aborting, for a phase that copies
// already issued complete: used before exit so that no copy into this CTA is still in flight.
__device__ __forceinline__ void wait_landed(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity))
        if (ptx::globaltimer_ns() - t0 > 100000000ull) return;
}

struct Item {
    int h, kh;
    int u0;              // first query row of the unit within its sequence
    int q_tok0, k_tok0;  // first packed token of the unit / of the sequence's keys
    int lq, lk, off;     // off = Lk - Lq
    int rows[2];         // this CTA's valid rows in group 0 / 1
    int n[2];            // key tiles of group 0 / 1: the larger of its two halves' counts
    int n_max;
};

// Items are ordered as in the single-CTA kernel (kv-head-major, or unit-major when K/V fits in L2).
__device__ __forceinline__ Item decode(const Params &p, int it, int num_units, bool causal, uint32_t cta) {
    Item x;
    int e;
    item_unit_head(p, it, num_units, e, x.h);
    x.kh = x.h / p.group;
    const int2 bm = p.units[e];
    const int4 s = p.seq_info[bm.x];
    x.u0 = bm.y * kUnitRows;
    x.q_tok0 = s.x + x.u0;
    x.k_tok0 = s.y;
    x.lq = s.z;
    x.lk = s.w;
    x.off = s.w - s.z;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int r0 = x.u0 + t * kGroupRows, r1 = r0 + kBM;
        const int n0 = kv_tiles_for(r0, tile_rows(r0, s.z), s.z, s.w, causal);
        const int n1 = kv_tiles_for(r1, tile_rows(r1, s.z), s.z, s.w, causal);
        x.n[t] = max(n0, n1);
        x.rows[t] = tile_rows(cta ? r1 : r0, s.z);
    }
    x.n_max = max(x.n[0], x.n[1]);
    return x;
}

template <typename T, bool kCausal, bool kPositiveScale>
__global__ void __launch_bounds__(kThreads, 1)
    mla_prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                            const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kr,
                            const __grid_constant__ CUtensorMap tm_v, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Barriers *bars = reinterpret_cast<Barriers *>(smem + kSmemBar);
    const uint32_t sQ = ptx::smem_addr(smem + kSmemQ);
    const uint32_t sRing = ptx::smem_addr(smem + kSmemRing);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t cta = ptx::cluster_ctarank();
    const bool leader = cta == 0;

    auto bar = [&](uint64_t &b) { return ptx::smem_addr(&b); };
    // the same barrier in the leader CTA (shared::cluster address)
    auto lead_bar = [&](uint64_t &b) { return ptx::mapa_shared(ptx::smem_addr(&b), 0); };
    const uint32_t peer_abort = ptx::mapa_shared(ptx::smem_addr(&bars->abort), cta ^ 1u);

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
        const uint32_t full_count = leader ? 2 : 1;
        for (int t = 0; t < 2; ++t) {
            ptx::mbar_init(bar(bars->q_full[t]), full_count);
            ptx::mbar_init(bar(bars->q_empty[t]), 1);
            ptx::mbar_init(bar(bars->s_full[t]), 1);
            ptx::mbar_init(bar(bars->p_full[t]), kPReadyArrivals);
            ptx::mbar_init(bar(bars->o_full[t]), 1);
            ptx::mbar_init(bar(bars->o_empty[t]), kSoftmaxWarpsPerPair);
        }
        for (int c = 0; c < kTileBars; ++c) {
            ptx::mbar_init(bar(bars->k_full[c]), full_count);
            ptx::mbar_init(bar(bars->v_full[c]), full_count);
            ptx::mbar_init(bar(bars->k_empty[c]), 1);
            ptx::mbar_init(bar(bars->v_empty[c]), 1);
        }
        for (int i = 0; i < kSched; ++i) {
            ptx::mbar_init(bar(bars->sched_full[i]), 1);
            ptx::mbar_init(bar(bars->sched_empty[i]), kSchedConsumers);
        }
        ptx::mbar_init(bar(bars->drain), 1);
        bars->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(ptx::smem_addr(&bars->tmem_base), kTmemCols);
        ptx::tmem_relinquish_pair();
    }
    // both CTAs' barriers are initialised before either CTA arrives on the other's
    ptx::tc_fence_before();
    ptx::cluster_sync_all();
    ptx::tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    ptx::griddep_wait();  // the plan kernel's work list is complete and visible
    const int num_units = *p.num_units;
    const int n_items = num_units * p.head_num;
    const int cluster_id = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;

    // Work-item hand-off, consumer side: returns the item of ring slot sc (-1: no more work).
    auto receive = [&](uint32_t sc, bool &ok) -> int {
        const uint32_t slot = sc % kSched;
        ok = wait_pair_warp<true>(bar(bars->sched_full[slot]), (sc / kSched) & 1, bars, peer_abort, p.status);
        if (!ok) return -1;
        const int it = *reinterpret_cast<volatile int *>(&bars->sched_item[slot]);
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_remote(lead_bar(bars->sched_empty[slot]));
        __syncwarp();
        return it;
    };

    if (warp < 4) {
        ptx::regs_dec<kRegsLow>();
        if (warp == 0 && lane == 0) {
            // ------------------------------------------------------------ TMA producer (both CTAs)
            const uint64_t pol_q = ptx::policy_evict_first();
            const uint64_t pol_kv = ptx::policy_evict_last();
            auto wait = [&](uint32_t b, uint32_t parity) { return wait_pair(b, parity, bars, peer_abort, p.status); };
            auto chunk = [&](uint32_t c) { return sRing + (c % kRing) * kChunkBytes; };
            uint32_t tk = 0, tv = 0, ql0 = 0, ql1 = 0;
            bool ok = true;
            // Key tile g sits in ring chunks 5g .. 5g + 4 (mod 16).  K_g's chunks last held V_{g-4}'s
            // second chunk and K_{g-3}'s first two; V_g's chunks last held K_{g-3}'s third and
            // V_{g-3}'s first.  The commit releasing K_{g-3} follows every MMA reading V_{g-4}, so
            // K_g waits for K_{g-3}'s release and V_g for V_{g-3}'s.
            uint32_t sc = 0;
            int next = cluster_id < n_items ? cluster_id : -1;
            while (ok) {
                int it;
                const uint32_t slot = sc % kSched;
                if (leader) {
                    it = next;
                    ok = wait(bar(bars->sched_empty[slot]), ((sc / kSched) & 1) ^ 1);
                    if (!ok) break;
                    *reinterpret_cast<volatile int *>(&bars->sched_item[slot]) = it;
                    ptx::st_shared_cluster_u32(ptx::mapa_shared(ptx::smem_addr(&bars->sched_item[slot]), 1),
                                               static_cast<uint32_t>(it));
                    ptx::mbar_arrive(bar(bars->sched_full[slot]));
                    ptx::mbar_arrive_cluster(ptx::mapa_shared(bar(bars->sched_full[slot]), 1));
                    if (it >= 0) {
                        next = n_clusters + atomicAdd(p.work_counter, 1);
                        if (next >= n_items) next = -1;
                    }
                } else {
                    ok = wait_pair<true>(bar(bars->sched_full[slot]), (sc / kSched) & 1, bars, peer_abort, p.status);
                    if (!ok) break;
                    it = *reinterpret_cast<volatile int *>(&bars->sched_item[slot]);
                    ptx::mbar_arrive_remote(lead_bar(bars->sched_empty[slot]));
                }
                ++sc;
                if (it < 0) break;
                const Item x = decode(p, it, num_units, kCausal, cta);
                if (x.n_max == 0) continue;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (!ok || x.n[t] == 0) continue;
                    uint32_t &ql = t ? ql1 : ql0;
                    ok = wait(bar(bars->q_empty[t]), (ql & 1) ^ 1);  // the last S_t of the previous unit is done
                    if (!ok) continue;
                    const uint32_t fb = bar(bars->q_full[t]);
                    const uint32_t dst = sQ + t * kQTileBytes;
                    const int tok = x.q_tok0 + t * kGroupRows + static_cast<int>(cta) * kBM;
                    ptx::mbar_arrive_expect_tx(fb, kQTileBytes);
                    ptx::tma_load_3d(dst, &tm_q, fb, 0, x.h, tok, pol_q);
                    ptx::tma_load_3d(dst + 16384, &tm_q, fb, 64, x.h, tok, pol_q);
                    ptx::tma_load_3d(dst + 32768, &tm_qr, fb, 0, x.h, tok, pol_q);
                    ++ql;
                }
                for (int j = 0; j < x.n_max && ok; ++j) {
                    const int tok = x.k_tok0 + j * kBN;
                    const uint32_t g = tk, c0 = kTileChunks * g;
                    // K_j: this CTA's 64 keys, nope cols 0-63 | nope cols 64-127 | rope
                    if (g >= 3 && !(ok = wait(bar(bars->k_empty[(g - 3) % kTileBars]), ((g - 3) / kTileBars) & 1)))
                        break;
                    uint32_t fb = bar(bars->k_full[g % kTileBars]);
                    ptx::mbar_arrive_expect_tx(fb, kKChunks * kChunkBytes);
                    const int ktok = tok + static_cast<int>(cta) * 64;
                    ptx::tma_load_3d(chunk(c0), &tm_k, fb, 0, x.kh, ktok, pol_kv);
                    ptx::tma_load_3d(chunk(c0 + 1), &tm_k, fb, 64, x.kh, ktok, pol_kv);
                    ptx::tma_load_3d(chunk(c0 + 2), &tm_kr, fb, 0, x.kh, ktok, pol_kv);
                    ++tk;
                    // V_j: keys 0-63 | keys 64-127, this CTA's 64 columns
                    if (g >= 3 && !(ok = wait(bar(bars->v_empty[(g - 3) % kTileBars]), ((g - 3) / kTileBars) & 1)))
                        break;
                    fb = bar(bars->v_full[g % kTileBars]);
                    ptx::mbar_arrive_expect_tx(fb, kVChunks * kChunkBytes);
                    const int vcol = static_cast<int>(cta) * 64;
                    ptx::tma_load_3d(chunk(c0 + 3), &tm_v, fb, vcol, x.kh, tok, pol_kv);
                    ptx::tma_load_3d(chunk(c0 + 4), &tm_v, fb, vcol, x.kh, tok + 64, pol_kv);
                    ++tv;
                }
            }
            // Let every copy this CTA started land before it can exit, also when aborting.  The
            // follower's barriers count its own loads only; the leader's also need the relay's
            // arrival, which may never come after an abort: the wait is bounded either way.
            if (ql0) wait_landed(bar(bars->q_full[0]), (ql0 - 1) & 1);
            if (ql1) wait_landed(bar(bars->q_full[1]), (ql1 - 1) & 1);
            for (uint32_t g = tk > kTileBars ? tk - kTileBars : 0; g < tk; ++g)
                wait_landed(bar(bars->k_full[g % kTileBars]), (g / kTileBars) & 1);
            for (uint32_t g = tv > kTileBars ? tv - kTileBars : 0; g < tv; ++g)
                wait_landed(bar(bars->v_full[g % kTileBars]), (g / kTileBars) & 1);
        } else if (warp == 1 && !leader) {
            // ------------------------------------------------------------ relay (follower)
            // Follows the producer's order of loads: each time one of this CTA's loads has landed,
            // arrives on the leader's barrier for the same data.
            uint32_t ss = 0, tg = 0, qf0 = 0, qf1 = 0;
            bool ok = true;
            auto fwd = [&](uint64_t &b, uint32_t parity) -> bool {
                if (!wait_pair_warp(bar(b), parity, bars, peer_abort, p.status)) return false;
                if (lane == 0) ptx::mbar_arrive_remote(lead_bar(b));
                __syncwarp();
                return true;
            };
            while (ok) {
                const int it = receive(ss++, ok);
                if (!ok || it < 0) break;
                const Item x = decode(p, it, num_units, kCausal, cta);
                if (x.n_max == 0) continue;
                if (x.n[0]) ok = fwd(bars->q_full[0], qf0++ & 1);
                if (ok && x.n[1]) ok = fwd(bars->q_full[1], qf1++ & 1);
                for (int j = 0; j < x.n_max && ok; ++j) {
                    const uint32_t g = tg + j;
                    ok = fwd(bars->k_full[g % kTileBars], (g / kTileBars) & 1);
                    if (ok) ok = fwd(bars->v_full[g % kTileBars], (g / kTileBars) & 1);
                }
                tg += x.n_max;
            }
        } else if (warp >= 2 && leader) {
            // ------------------------------------------------------------ helpers (leader)
            // Warp 2 serves group 0, warp 3 group 1.  For every step j < n_t of a unit: once S_t(j)
            // is ready (the MMA warp then has consumed the group's previous P-ready phase, so this
            // arrival cannot fall into it), waits until key tile j's V and, if the group has a next
            // tile, tile j + 1's K have landed in both CTAs (the leader's full barriers count the
            // relay's arrivals), then arrives on the group's P-ready barrier.  All of this overlaps
            // the group's softmax of step j.
            const int t = warp - 2;
            uint32_t ss = 0, tg = 0, sf = 0;
            bool ok = true;
            auto waitw = [&](uint32_t b, uint32_t parity) {
                return wait_pair_warp(b, parity, bars, peer_abort, p.status);
            };
            while (ok) {
                const int it = receive(ss++, ok);
                if (!ok || it < 0) break;
                const Item x = decode(p, it, num_units, kCausal, cta);
                const int n_t = x.n[t];
                for (int j = 0; j < n_t && ok; ++j) {
                    const uint32_t g = tg + j;
                    ok = waitw(bar(bars->s_full[t]), sf++ & 1);
                    if (ok) ok = waitw(bar(bars->v_full[g % kTileBars]), (g / kTileBars) & 1);
                    if (ok && j + 1 < n_t) ok = waitw(bar(bars->k_full[(g + 1) % kTileBars]), ((g + 1) / kTileBars) & 1);
                    if (ok && lane == 0) ptx::mbar_arrive(bar(bars->p_full[t]));
                    __syncwarp();
                }
                tg += x.n_max;
            }
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer (leader)
            constexpr bool kBf16 = DType<T>::kBf16;
            constexpr uint32_t kIdQK = ptx::instr_desc_f16(kBf16, kGroupRows, kBN, false);
            constexpr uint32_t kIdPV = ptx::instr_desc_f16(kBf16, kGroupRows, kDn, true);
            constexpr uint32_t kHi = ptx::desc_hi_sw128(1024);
            constexpr uint16_t kBoth = 3;  // commits arrive in both CTAs
            const uint32_t q_lo = ptx::desc_lo(sQ, 16);
            const uint32_t ring_k_lo = ptx::desc_lo(sRing, 16);
            const uint32_t ring_v_lo = ptx::desc_lo(sRing, kChunkBytes);
            constexpr uint32_t kC = kChunkBytes >> 4;  // one ring chunk in descriptor units
            uint32_t tg = 0, qf0 = 0, qf1 = 0, pf0 = 0, pf1 = 0, oe0 = 0, oe1 = 0;
            bool ok = true;
            auto waitw = [&](uint32_t b, uint32_t parity) {
                return wait_pair_warp(b, parity, bars, peer_abort, p.status);
            };
            auto commit = [&](uint64_t &b) {
                if (ptx::elect_one()) ptx::mma_commit_pair(bar(b), kBoth);
                __syncwarp();
            };
            // S_t = [Qn|Qr]_t [Kn|Kr]^T over the pair: 12 k-steps of 16 channels
            auto issue_s = [&](int t, uint32_t kc) {
                const uint32_t d = tmem + kTmemS + t * kBN;
                const uint32_t a0 = q_lo + ((t * kQTileBytes) >> 4);
                const uint32_t b0 = ring_k_lo + ((kc + 0) % kRing) * kC;
                const uint32_t b1 = ring_k_lo + ((kc + 1) % kRing) * kC;
                const uint32_t b2 = ring_k_lo + ((kc + 2) % kRing) * kC;
                if (ptx::elect_one()) {
                    constexpr uint32_t kQC = 16384 >> 4;  // one Q chunk (128 rows x 128 B)
                    ptx::mma2_ss_lo<kHi, kIdQK, 0>(d, a0 + 0, b0 + 0);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + 2, b0 + 2);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + 4, b0 + 4);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + 6, b0 + 6);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + kQC + 0, b1 + 0);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + kQC + 2, b1 + 2);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + kQC + 4, b1 + 4);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + kQC + 6, b1 + 6);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + 2 * kQC + 0, b2 + 0);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + 2 * kQC + 2, b2 + 2);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + 2 * kQC + 4, b2 + 4);
                    ptx::mma2_ss_lo<kHi, kIdQK, 1>(d, a0 + 2 * kQC + 6, b2 + 6);
                    ptx::mma_commit_pair(bar(bars->s_full[t]), kBoth);
                }
                __syncwarp();
            };
            // O_t (+)= P_t V over the pair: 8 k-steps of 16 keys, P from tensor memory
            auto issue_pv = [&](int t, uint32_t vc, bool accumulate) {
                const uint32_t d = tmem + kTmemO + t * kDn;
                const uint32_t pa = tmem + kTmemS + t * kBN + kTmemPOff;
                const uint32_t v0 = ring_v_lo + ((vc + 0) % kRing) * kC;
                const uint32_t v1 = ring_v_lo + ((vc + 1) % kRing) * kC;
                if (ptx::elect_one()) {
                    // 16 keys x 128 B = 2048 B = 128 units per k-step; P advances 8 columns per k-step
                    if (accumulate) ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa, v0);
                    else ptx::mma2_ts_lo<kHi, kIdPV, 0>(d, pa, v0);
                    ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa + 8, v0 + 128);
                    ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa + 16, v0 + 256);
                    ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa + 24, v0 + 384);
                    ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa + 32, v1);
                    ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa + 40, v1 + 128);
                    ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa + 48, v1 + 256);
                    ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa + 56, v1 + 384);
                }
                __syncwarp();
            };
            uint32_t ss = 0;
            while (ok) {
                const int it = receive(ss++, ok);
                if (!ok || it < 0) break;
                const Item x = decode(p, it, num_units, kCausal, cta);
                if (x.n_max == 0) continue;
                if (x.n[0]) ok = waitw(bar(bars->q_full[0]), qf0++ & 1);
                if (ok && x.n[1]) ok = waitw(bar(bars->q_full[1]), qf1++ & 1);
                if (!ok) break;
                // key tile g = tg + j: K_g in ring chunks 5g + {0,1,2}, V_g in 5g + {3,4}.  The last MMA
                // reading a key tile is group 1's when group 1 reads it (issued after group 0's).
                ok = waitw(bar(bars->k_full[tg % kTileBars]), (tg / kTileBars) & 1);
                if (!ok) break;
                ptx::tc_fence_after();
                if (x.n[0] > 0) {
                    issue_s(0, kTileChunks * tg);
                    if (x.n[0] == 1) commit(bars->q_empty[0]);
                }
                if (x.n[1] > 0) {
                    issue_s(1, kTileChunks * tg);
                    if (x.n[1] == 1) commit(bars->q_empty[1]);
                }
                commit(bars->k_empty[tg % kTileBars]);
                // Inside the unit the issuer waits for P-ready only: the helper has seen V_j and
                // K_{j+1} land before its own arrival on the step's P-ready barriers.
                for (int j = 0; j < x.n_max && ok; ++j) {
                    const uint32_t g = tg + j, kc = kTileChunks * g, vc = kc + kKChunks, kn = kc + kTileChunks;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        if (ok && j < x.n[t]) {
                            uint32_t &pf = t ? pf1 : pf0;
                            uint32_t &oe = t ? oe1 : oe0;
                            ok = waitw(bar(bars->p_full[t]), pf++ & 1);
                            if (ok && j == 0) ok = waitw(bar(bars->o_empty[t]), (oe++ & 1) ^ 1);
                            if (ok) {
                                ptx::tc_fence_after();
                                issue_pv(t, vc, j > 0);
                                if (j == x.n[t] - 1) commit(bars->o_full[t]);
                                if (t == 1 || j >= x.n[1]) commit(bars->v_empty[g % kTileBars]);  // last P V_g
                            }
                        }
                        if (ok && j + 1 < x.n[t]) {
                            issue_s(t, kn);
                            if (j + 2 == x.n[t]) commit(bars->q_empty[t]);  // last S_t of the unit
                            if (t == 1 || j + 1 >= x.n[1]) commit(bars->k_empty[(g + 1) % kTileBars]);
                        }
                    }
                }
                if (!ok) break;
                tg += x.n_max;
            }
            // Drain: wait until every MMA issued here has completed (commit to the leader only).
            if (ptx::elect_one()) ptx::mma_commit_pair(bar(bars->drain), 1);
            __syncwarp();
            wait_pair_warp(bar(bars->drain), 0, bars, peer_abort, p.status);
        }
    } else {
        ptx::regs_inc<kRegsHigh>();
        // ---------------------------------------------------------------- softmax + epilogue (both CTAs)
        const int t = (warp >> 2) - 1;   // group of this warpgroup
        const int wq = warp & 3;         // TMEM lane quarter this warp may access
        const int row = wq * 32 + lane;  // row within this CTA's 128 rows of the group
        const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_addr + kTmemS + t * kBN;
        const uint32_t tO = tmem + lane_addr + kTmemO + t * kDn;
        const uint32_t p_ready = lead_bar(bars->p_full[t]);
        const uint32_t o_free = lead_bar(bars->o_empty[t]);
        const float sl2 = p.scale_log2;
        uint32_t sf = 0, of = 0, ss = 0;
        bool ok = true;
        // One arrival per warp on the leader's barrier, after this warp's tensor-memory accesses.
        auto arrive_warp = [&](uint32_t lead_addr) {
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_remote(lead_addr);
        };
        while (ok) {
            const int it = receive(ss++, ok);
            if (!ok || it < 0) break;
            const Item x = decode(p, it, num_units, kCausal, cta);
            const int n_t = x.n[t];
            const bool row_valid = row < x.rows[t];
            const int tile_q0 = x.u0 + t * kGroupRows + static_cast<int>(cta) * kBM;
            const int i = tile_q0 + row;  // query row within the sequence
            T *orow = reinterpret_cast<T *>(p.out) + (long long)(x.q_tok0 + t * kGroupRows +
                                                                 static_cast<int>(cta) * kBM + row) * p.out_st +
                      (long long)x.h * p.out_sh;
            if (n_t == 0) {  // no key visible to any row of the group: no MMA runs for it
                if (row_valid) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int c = 0; c < kDn * 2 / 16; ++c) reinterpret_cast<uint4 *>(orow)[c] = z;
                }
                continue;
            }
            const int lim_row = kCausal ? min(i + x.off + 1, x.lk) : x.lk;  // keys [0, lim_row) visible
            float m_run = -INFINITY, l_run = 0.f;
            for (int j = 0; j < n_t; ++j) {
                ok = wait_pair_warp(bar(bars->s_full[t]), sf & 1, bars, peer_abort, p.status);
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
                const int kv0 = j * kBN;
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
                const float2 sc2 = kPositiveScale ? make_float2(sl2, sl2) : make_float2(1.f, 1.f);
                const float2 nm2 = make_float2(-m_use, -m_use);
                uint32_t pk[64];
                const float rowsum = exp_pack_sum<T>(s, sc2, nm2, pk);
                ptx::tmem_st64(tS + kTmemPOff, pk);
                // O_t holds P(j-1) V(j-1) already (the MMAs behind S_t(j) have completed);
                // rescale it before P V(j) may start.
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
                arrive_warp(p_ready);
                l_run = l_run * alpha + rowsum;
            }
            if (!ok) break;
            // Epilogue: O / l -> 16-bit, one 256-byte row per thread.
            ok = wait_pair_warp(bar(bars->o_full[t]), of & 1, bars, peer_abort, p.status);
            ++of;
            if (!ok) break;
            ptx::tc_fence_after();
            const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
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
            arrive_warp(o_free);
        }
    }

    // Neither CTA leaves while the other may still arrive on its barriers or while pair MMAs may
    // still write its tensor memory (the leader's MMA warp has drained before it gets here).
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync_all();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace pair
}  // namespace mla
