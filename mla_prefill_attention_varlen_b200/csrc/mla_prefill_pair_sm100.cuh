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
// (rows u0 + 256 t + [0, 128) in the leader, the next 128 in the follower); or, when every kv
// head serves an even number of query heads, 256 rows for two query heads h, h + 1 of one kv head,
// group t taking head h + t over the same rows (head pairs: both groups walk the same key tiles,
// where the two halves of a 512-row unit differ by four, and the last unit of a sequence may leave
// its second group empty).  The leader's MMA
// warp issues M = 256 tensor-core MMAs over the pair (tcgen05 cta_group::2): each CTA's tensor
// memory receives its own 128 rows, the A operand (Q or P) comes from each CTA's own shared or
// tensor memory, and the B operand (K for S, V for P V) is split along N: each CTA loads only
// its half of every key tile -- 32 of the 64 keys of K, 64 of the 128 columns of V.
//
// Key tiles are 64 keys, and each group has two S buffers in tensor memory: S of the group's
// g-th tile (counted across units) goes to buffer g mod 2, and the softmax writes P over the
// buffer it has just read.  The MMA warp issues S_t(j + 2) right after P V_t(j) -- into the
// buffer P V_t(j) reads, which the in-order tensor pipe empties first -- so S of the next tile
// is computed while the softmax still works on the current one: the softmax runs tile after
// tile without waiting for P V and the next S, and the tensor pipe has the other group's work
// and this group's next S to fill its time.  The S-full, P-ready and P V-done barriers come in
// pairs by tile parity: a barrier's next phase then needs the group's next-but-one tile, so no
// role can fall two phases behind one it waits for, and the softmax waits for P V only when it
// has to rescale O.
//
//   leader   warp 0: TMA loads of its halves; claims work items and hands them to both CTAs
//            warp 1: MMA issuer for the pair
//            warps 2, 3: helpers of groups 0, 1: for every tile, wait until the key tile's V
//                    and the K of the group's tile two ahead have landed in both CTAs, then
//                    arrive on the group's P-ready barrier, so that the MMA issuer waits for
//                    nothing but P-ready between its MMAs
//   follower warp 0: TMA loads of its halves (items received from the leader)
//            warp 1: relay: once each of its loads has landed (its own barrier), arrives on the
//                    leader's matching barrier, so the leader's MMAs see both halves
//   both     warps 4-7 / 8-11: softmax of group 0 / 1 over this CTA's 128 rows of the group,
//            P written to tensor memory, epilogue of this CTA's rows
//
// Every TMA load completes on a barrier of the CTA it writes to, so each CTA can wait for its
// own copies before it exits.  Commits of the pair MMAs arrive on the same barrier in both CTAs
// (multicast); P-ready arrivals of the follower's softmax warps go to the leader's barriers.
// All waits are bounded; a timeout in either CTA aborts both.
#pragma once

#include "mla_prefill_sm100.cuh"

namespace mla {
namespace pair {

constexpr int kUnitRows = 512;           // query rows per work unit (two groups of 256)
constexpr int kGroupRows = 256;          // rows of one pair MMA (128 per CTA)
constexpr int kKeys = 64;                // keys per key tile
constexpr int kSlots = 6;                // key-tile slots in each CTA's ring
constexpr int kKPart = 4096;             // this CTA's 32 keys x 64 channels (128 B rows)
constexpr int kVBytes = 8192;            // 64 keys x this CTA's 64 V columns (128 B rows)
constexpr int kSlotBytes = 3 * kKPart + kVBytes;  // K: nope 0-63 | nope 64-127 | rope, then V
constexpr int kQTileBytes = 3 * 16384;   // this CTA's 128 rows of a group: nope lo | nope hi | rope
constexpr int kSched = 4;

constexpr int kSmemQ = 0;
constexpr int kSmemRing = kSmemQ + 2 * kQTileBytes;
constexpr int kSmemBar = kSmemRing + kSlots * kSlotBytes;
constexpr int kSmemBytes = kSmemBar + 512;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack to align the base to 1024 B
static_assert(kSmemAlloc <= 232448, "shared memory per CTA");
static_assert(kSlotBytes % 1024 == 0 && kKPart % 1024 == 0, "128-byte-swizzle atoms stay 1024-byte aligned");

// Tensor memory (512 columns): O_t at 128 t; S_t buffer b at 256 + 128 t + 64 b, P_t of that
// buffer's tile over its first 32 columns (64 16-bit values per row).
constexpr uint32_t kTmemOBase = 0;
constexpr uint32_t kTmemSBase = 256;

// Arrivals the leader's sched_empty barrier collects per slot: its MMA warp, 2 helpers and 8
// softmax warps, the follower's producer, relay and 8 softmax warps.
constexpr int kSchedConsumers = 1 + 2 + 8 + 1 + 1 + 8;
constexpr int kSoftmaxWarpsPerPair = 8;  // per-warp arrivals of one group, both CTAs
constexpr int kPReadyArrivals = kSoftmaxWarpsPerPair + 1;  // P_t(g) published by both CTAs, data seen by the helper

struct Barriers {
    // full barriers: the leader's count its own producer's arrival (with the bytes it loads) and
    // the follower relay's arrival; the follower's count its own producer's arrival only
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[kSlots], v_full[kSlots], k_empty[kSlots], v_empty[kSlots];
    // [group][tile parity]: S buffer full, P-ready, P V done of the group's tiles of that parity
    uint64_t s_full[2][2], p_full[2][2], pv_done[2][2];
    uint64_t o_full[2];
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
    int h, kh;           // query head of group 0 (group t runs head h + t * dh) and its kv head
    int dh, drow;        // head and row steps from group 0 to group 1: (0, 256), or (1, 0) for head pairs
    int u0;              // first query row of the unit within its sequence
    int q_tok0, k_tok0;  // first packed token of the unit / of the sequence's keys
    int lq, lk, off;     // off = Lk - Lq
    int rows[2];         // this CTA's valid rows in group 0 / 1
    int n[2];            // 64-key tiles of group 0 / 1: the larger of its two halves' counts
    int n_max;
};

// 64-key tiles a 128-row query tile touches: the keys visible to its last row (causal) or all
// keys; 0 when the tile has no rows or sees no key.
__device__ __forceinline__ int key_tiles(int q0, int rows, int lq, int lk, bool causal) {
    if (rows <= 0) return 0;
    const int kv_end = causal ? min(q0 + rows + (lk - lq), lk) : lk;
    return kv_end > 0 ? (kv_end + kKeys - 1) / kKeys : 0;
}

// Items are ordered as in the single-CTA kernel (kv-head-major, or unit-major when K/V fits in L2),
// over heads or, with p.head_pair, over pairs of heads (2j, 2j + 1) of one kv head.
__device__ __forceinline__ Item decode(const Params &p, int it, int num_units, bool causal, uint32_t cta) {
    Item x;
    const int hp = p.head_pair;
    const int hn = p.head_num >> hp, gr = p.group >> hp;  // heads (pairs) in all and per kv head
    int e, h;
    if (p.lpt) {
        e = it / hn;
        h = it - e * hn;
    } else {
        const int per_kh = num_units * gr;
        const int kh = it / per_kh;
        const int rem = it - kh * per_kh;
        e = rem / gr;
        h = kh * gr + (rem - e * gr);
    }
    x.h = h << hp;
    x.kh = x.h / p.group;
    x.dh = hp;
    x.drow = hp ? 0 : kGroupRows;
    const int2 bm = p.units[e];
    const int4 s = p.seq_info[bm.x];
    x.u0 = bm.y * (hp ? kGroupRows : kUnitRows);
    x.q_tok0 = s.x + x.u0;
    x.k_tok0 = s.y;
    x.lq = s.z;
    x.lk = s.w;
    x.off = s.w - s.z;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int r0 = x.u0 + t * x.drow, r1 = r0 + kBM;
        const int n0 = key_tiles(r0, tile_rows(r0, s.z), s.z, s.w, causal);
        const int n1 = key_tiles(r1, tile_rows(r1, s.z), s.z, s.w, causal);
        x.n[t] = max(n0, n1);
        x.rows[t] = tile_rows(cta ? r1 : r0, s.z);
    }
    x.n_max = max(x.n[0], x.n[1]);
    return x;
}

// Max of a 64-element row: eight independent chains of three-input max, then a short tree.
__device__ __forceinline__ float row_max64(const float (&s)[kKeys]) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = ptx::fmax3(s[i], s[i + 8], s[i + 16]);  // s[0..23]
#pragma unroll
    for (int c = 24; c + 16 <= kKeys; c += 16) {                               // s[24..55]
#pragma unroll
        for (int i = 0; i < 8; ++i) m[i] = ptx::fmax3(m[i], s[c + i], s[c + 8 + i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(m[i], s[56 + i]);                 // s[56..63]
    return ptx::fmax3(ptx::fmax3(m[0], m[1], m[2]), ptx::fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// Exponentials of one row of a key tile: p = 2^(s * sc - m) for the 64 scores, packed to the
// 16-bit P operand (pk) and summed in fp32 (returned): one packed FMA per pair, one MUFU ex2 per
// element, four packed partial sums, one 16-bit pair conversion per pair.
template <typename T>
__device__ __forceinline__ float exp_pack_sum64(const float (&s)[kKeys], float2 sc2, float2 nm2,
                                                uint32_t (&pk)[kKeys / 2]) {
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int e = 0; e < kKeys / 2; ++e) {
        const float2 x2 = ptx::ffma2(make_float2(s[2 * e], s[2 * e + 1]), sc2, nm2);
        const float2 p2 = make_float2(ptx::ex2(x2.x), ptx::ex2(x2.y));
        acc[e & 3] = ptx::fadd2(acc[e & 3], p2);
        pk[e] = DType<T>::pack(p2.x, p2.y);
    }
    const float2 acc01 = ptx::fadd2(acc[0], acc[1]), acc23 = ptx::fadd2(acc[2], acc[3]);
    const float2 acc2 = ptx::fadd2(acc01, acc23);
    return acc2.x + acc2.y;
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
            for (int b = 0; b < 2; ++b) {
                ptx::mbar_init(bar(bars->s_full[t][b]), 1);
                ptx::mbar_init(bar(bars->p_full[t][b]), kPReadyArrivals);
                ptx::mbar_init(bar(bars->pv_done[t][b]), 1);
            }
            ptx::mbar_init(bar(bars->o_full[t]), 1);
        }
        for (int c = 0; c < kSlots; ++c) {
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
    const int n_items = num_units * (p.head_num >> p.head_pair);
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
            uint32_t tk = 0, tv = 0, ql0 = 0, ql1 = 0;
            bool ok = true;
            // Key tile g (counted across units) sits in slot g mod 6; its K waits for the release of
            // tile g - 6's K, its V for that of tile g - 6's V.
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
                } else {
                    ok = wait_pair<true>(bar(bars->sched_full[slot]), (sc / kSched) & 1, bars, peer_abort, p.status);
                    if (!ok) break;
                    it = *reinterpret_cast<volatile int *>(&bars->sched_item[slot]);
                    ptx::mbar_arrive_remote(lead_bar(bars->sched_empty[slot]));
                }
                ++sc;
                if (it < 0) break;
                // The leader claims the next item when the loads of this one's last key tile are
                // about to be issued (claimed at an item's start, a pair that drew a long item would
                // also take the next item of the longest-first list from pairs that free up sooner).
                auto claim = [&]() {
                    if (leader) {
                        next = n_clusters + atomicAdd(p.work_counter, 1);
                        if (next >= n_items) next = -1;
                    }
                };
                const Item x = decode(p, it, num_units, kCausal, cta);
                if (x.n_max == 0) {
                    claim();
                    continue;
                }
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (!ok || x.n[t] == 0) continue;
                    uint32_t &ql = t ? ql1 : ql0;
                    ok = wait(bar(bars->q_empty[t]), (ql & 1) ^ 1);  // the last S_t of the previous unit is done
                    if (!ok) continue;
                    const uint32_t fb = bar(bars->q_full[t]);
                    const uint32_t dst = sQ + t * kQTileBytes;
                    const int tok = x.q_tok0 + t * x.drow + static_cast<int>(cta) * kBM;
                    const int qh = x.h + t * x.dh;
                    ptx::mbar_arrive_expect_tx(fb, kQTileBytes);
                    ptx::tma_load_3d(dst, &tm_q, fb, 0, qh, tok, pol_q);
                    ptx::tma_load_3d(dst + 16384, &tm_q, fb, 64, qh, tok, pol_q);
                    ptx::tma_load_3d(dst + 32768, &tm_qr, fb, 0, qh, tok, pol_q);
                    ++ql;
                }
                for (int j = 0; j < x.n_max && ok; ++j) {
                    if (j == x.n_max - 1) claim();
                    const int tok = x.k_tok0 + j * kKeys;
                    const uint32_t g = tk, slot = g % kSlots, phase = ((g / kSlots) & 1) ^ 1;
                    const uint32_t dst = sRing + slot * kSlotBytes;
                    // K_g: this CTA's 32 keys, nope cols 0-63 | nope cols 64-127 | rope
                    if (g >= kSlots && !(ok = wait(bar(bars->k_empty[slot]), phase))) break;
                    uint32_t fb = bar(bars->k_full[slot]);
                    ptx::mbar_arrive_expect_tx(fb, 3 * kKPart);
                    const int ktok = tok + static_cast<int>(cta) * (kKeys / 2);
                    ptx::tma_load_3d(dst, &tm_k, fb, 0, x.kh, ktok, pol_kv);
                    ptx::tma_load_3d(dst + kKPart, &tm_k, fb, 64, x.kh, ktok, pol_kv);
                    ptx::tma_load_3d(dst + 2 * kKPart, &tm_kr, fb, 0, x.kh, ktok, pol_kv);
                    ++tk;
                    // V_g: the 64 keys, this CTA's 64 columns
                    if (g >= kSlots && !(ok = wait(bar(bars->v_empty[slot]), phase))) break;
                    fb = bar(bars->v_full[slot]);
                    ptx::mbar_arrive_expect_tx(fb, kVBytes);
                    ptx::tma_load_3d(dst + 3 * kKPart, &tm_v, fb, static_cast<int>(cta) * 64, x.kh, tok, pol_kv);
                    ++tv;
                }
            }
            // Let every copy this CTA started land before it can exit, also when aborting.  The
            // follower's barriers count its own loads only; the leader's also need the relay's
            // arrival, which may never come after an abort: the wait is bounded either way.
            if (ql0) wait_landed(bar(bars->q_full[0]), (ql0 - 1) & 1);
            if (ql1) wait_landed(bar(bars->q_full[1]), (ql1 - 1) & 1);
            for (uint32_t g = tk > kSlots ? tk - kSlots : 0; g < tk; ++g)
                wait_landed(bar(bars->k_full[g % kSlots]), (g / kSlots) & 1);
            for (uint32_t g = tv > kSlots ? tv - kSlots : 0; g < tv; ++g)
                wait_landed(bar(bars->v_full[g % kSlots]), (g / kSlots) & 1);
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
                    ok = fwd(bars->k_full[g % kSlots], (g / kSlots) & 1);
                    if (ok) ok = fwd(bars->v_full[g % kSlots], (g / kSlots) & 1);
                }
                tg += x.n_max;
            }
        } else if (warp >= 2 && leader) {
            // ------------------------------------------------------------ helpers (leader)
            // Warp 2 serves group 0, warp 3 group 1.  For the group's g-th tile (step j of a unit):
            // waits until S_t(g) has completed -- it was issued after P V_t(g - 2), so the P-ready
            // phase of tile g - 2 (the same barrier's previous one) is complete and this arrival
            // cannot fall into it, and every slot checked next is within one phase of the tile
            // asked for -- then until the tile's V and, if the group has a tile j + 2, that tile's
            // K have landed in both CTAs (the leader's full barriers count the relay's arrivals),
            // and arrives on the group's P-ready barrier of the tile's parity.  All of this
            // overlaps the group's softmax of the tile.
            const int t = warp - 2;
            uint32_t ss = 0, tg = 0, gt = 0;
            bool ok = true;
            auto waitw = [&](uint32_t b, uint32_t parity) {
                return wait_pair_warp(b, parity, bars, peer_abort, p.status);
            };
            while (ok) {
                const int it = receive(ss++, ok);
                if (!ok || it < 0) break;
                const Item x = decode(p, it, num_units, kCausal, cta);
                const int n_t = x.n[t];
                for (int j = 0; j < n_t && ok; ++j, ++gt) {
                    const uint32_t kg = tg + j;
                    ok = waitw(bar(bars->s_full[t][gt & 1]), (gt >> 1) & 1);
                    if (ok) ok = waitw(bar(bars->v_full[kg % kSlots]), (kg / kSlots) & 1);
                    if (ok && j + 2 < n_t)
                        ok = waitw(bar(bars->k_full[(kg + 2) % kSlots]), ((kg + 2) / kSlots) & 1);
                    if (ok && lane == 0) ptx::mbar_arrive(bar(bars->p_full[t][gt & 1]));
                    __syncwarp();
                }
                tg += x.n_max;
            }
        } else if (warp == 1) {
            // ------------------------------------------------------------ MMA issuer (leader)
            constexpr bool kBf16 = DType<T>::kBf16;
            constexpr uint32_t kIdQK = ptx::instr_desc_f16(kBf16, kGroupRows, kKeys, false);
            constexpr uint32_t kIdPV = ptx::instr_desc_f16(kBf16, kGroupRows, kDn, true);
            constexpr uint32_t kHi = ptx::desc_hi_sw128(1024);
            constexpr uint16_t kBoth = 3;  // commits arrive in both CTAs
            const uint32_t q_lo = ptx::desc_lo(sQ, 16);
            const uint32_t ring_k_lo = ptx::desc_lo(sRing, 16);
            const uint32_t ring_v_lo = ptx::desc_lo(sRing + 3 * kKPart, kVBytes);
            constexpr uint32_t kSlotU = kSlotBytes >> 4;  // one slot in descriptor units
            constexpr uint32_t kPartU = kKPart >> 4;
            uint32_t tg = 0, qf0 = 0, qf1 = 0, gs0 = 0, gs1 = 0;
            bool ok = true;
            auto waitw = [&](uint32_t b, uint32_t parity) {
                return wait_pair_warp(b, parity, bars, peer_abort, p.status);
            };
            auto commit = [&](uint64_t &b) {
                if (ptx::elect_one()) ptx::mma_commit_pair(bar(b), kBoth);
                __syncwarp();
            };
            // S_t = [Qn|Qr]_t [Kn|Kr]^T of key tile kg into S buffer sb: 12 k-steps of 16 channels
            auto issue_s = [&](int t, uint32_t kg, uint32_t sb) {
                const uint32_t d = tmem + kTmemSBase + t * 128 + sb * kKeys;
                const uint32_t a0 = q_lo + ((t * kQTileBytes) >> 4);
                const uint32_t b0 = ring_k_lo + (kg % kSlots) * kSlotU;
                const uint32_t b1 = b0 + kPartU, b2 = b0 + 2 * kPartU;
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
                    ptx::mma_commit_pair(bar(bars->s_full[t][sb]), kBoth);
                }
                __syncwarp();
            };
            // O_t (+)= P_t V of key tile kg over the pair: 4 k-steps of 16 keys, P from S buffer sb
            auto issue_pv = [&](int t, uint32_t kg, uint32_t sb, bool accumulate) {
                const uint32_t d = tmem + kTmemOBase + t * kDn;
                const uint32_t pa = tmem + kTmemSBase + t * 128 + sb * kKeys;
                const uint32_t v0 = ring_v_lo + (kg % kSlots) * kSlotU;
                if (ptx::elect_one()) {
                    // 16 keys x 128 B = 2048 B = 128 units per k-step; P advances 8 columns per k-step
                    if (accumulate) ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa, v0);
                    else ptx::mma2_ts_lo<kHi, kIdPV, 0>(d, pa, v0);
                    ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa + 8, v0 + 128);
                    ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa + 16, v0 + 256);
                    ptx::mma2_ts_lo<kHi, kIdPV, 1>(d, pa + 24, v0 + 384);
                    ptx::mma_commit_pair(bar(bars->pv_done[t][sb]), kBoth);
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
                // S of the unit's first two key tiles.  Every release (k_empty, v_empty) is committed
                // after the last MMA reading the tile: group 1's when group 1 reads it (its MMAs are
                // issued after group 0's), else group 0's.
                for (int j = 0; j < 2 && j < x.n_max && ok; ++j) {
                    ok = waitw(bar(bars->k_full[(tg + j) % kSlots]), ((tg + j) / kSlots) & 1);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    if (j < x.n[0]) {
                        issue_s(0, tg + j, (gs0 + j) & 1);
                        if (j == x.n[0] - 1) commit(bars->q_empty[0]);
                    }
                    if (j < x.n[1]) {
                        issue_s(1, tg + j, (gs1 + j) & 1);
                        if (j == x.n[1] - 1) commit(bars->q_empty[1]);
                    }
                    commit(bars->k_empty[(tg + j) % kSlots]);
                }
                // Per step: P V_t(j) once P_t(j) is ready (the helper has seen V_j and K_{j+2} land
                // before its own arrival), then S_t(j + 2) into the buffer P V_t(j) reads.
                for (int j = 0; j < x.n_max && ok; ++j) {
                    const uint32_t kg = tg + j;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const uint32_t g = (t ? gs1 : gs0) + j, sb = g & 1;  // the group's g-th tile
                        if (ok && j < x.n[t]) {
                            ok = waitw(bar(bars->p_full[t][sb]), (g >> 1) & 1);
                            if (ok) {
                                ptx::tc_fence_after();
                                issue_pv(t, kg, sb, j > 0);
                                if (j == x.n[t] - 1) commit(bars->o_full[t]);
                                if (t == 1 || j >= x.n[1]) commit(bars->v_empty[kg % kSlots]);
                            }
                        }
                        if (ok && j + 2 < x.n[t]) {
                            issue_s(t, kg + 2, sb);
                            if (j + 3 == x.n[t]) commit(bars->q_empty[t]);  // last S_t of the unit
                            if (t == 1 || j + 2 >= x.n[1]) commit(bars->k_empty[(kg + 2) % kSlots]);
                        }
                    }
                }
                if (!ok) break;
                gs0 += x.n[0];
                gs1 += x.n[1];
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
        const uint32_t tS0 = tmem + lane_addr + kTmemSBase + t * 128;
        const uint32_t tO = tmem + lane_addr + kTmemOBase + t * kDn;
        const float sl2 = p.scale_log2;
        uint32_t gt = 0, of = 0, ss = 0;
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
            const int tile_q0 = x.u0 + t * x.drow + static_cast<int>(cta) * kBM;
            const int i = tile_q0 + row;  // query row within the sequence
            T *orow = reinterpret_cast<T *>(p.out) + (long long)(x.q_tok0 + t * x.drow +
                                                                 static_cast<int>(cta) * kBM + row) * p.out_st +
                      (long long)(x.h + t * x.dh) * p.out_sh;
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
            for (int j = 0; j < n_t; ++j, ++gt) {
                const uint32_t sb = gt & 1;
                ok = wait_pair_warp(bar(bars->s_full[t][sb]), (gt >> 1) & 1, bars, peer_abort, p.status);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t tS = tS0 + sb * kKeys;
                float s[kKeys];
                {
                    uint32_t r[64];
                    ptx::tmem_ld64(tS, r);
                    ptx::tmem_wait_ld_dep64(r);
#pragma unroll
                    for (int e = 0; e < 64; ++e) s[e] = __uint_as_float(r[e]);
                }
                const int kv0 = j * kKeys;
                const bool tile_masked = (kv0 + kKeys > x.lk) || (kCausal && kv0 + kKeys - 1 > tile_q0 + x.off);
                float m_tile;
                if (kPositiveScale) {
                    if (tile_masked) {
                        const int lim = lim_row - kv0;
#pragma unroll
                        for (int c = 0; c < kKeys; ++c) s[c] = c < lim ? s[c] : -INFINITY;
                    }
                    m_tile = row_max64(s) * sl2;
                } else {
                    const int lim = tile_masked ? lim_row - kv0 : kKeys;
#pragma unroll
                    for (int c = 0; c < kKeys; ++c) s[c] = c < lim ? s[c] * sl2 : -INFINITY;
                    m_tile = row_max64(s);
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
                uint32_t pk[kKeys / 2];
                const float rowsum = exp_pack_sum64<T>(s, sc2, nm2, pk);
                ptx::tmem_st32(tS, pk);  // P over the S values just read
                // The running max moved: once P V_t of the group's previous tile has completed
                // (O_t holds it), rescale O_t before P V of this tile may start.  That barrier's
                // next phase needs this group's next tile's P-ready, so it is never two phases
                // ahead of the one waited for, also when most tiles skip this wait.
                if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
                    const uint32_t gp = gt - 1;
                    ok = wait_pair_warp(bar(bars->pv_done[t][gp & 1]), (gp >> 1) & 1, bars, peer_abort, p.status);
                    if (!ok) break;
                    ptx::tc_fence_after();
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
                arrive_warp(lead_bar(bars->p_full[t][sb]));
                l_run = l_run * alpha + rowsum;
            }
            if (!ok) break;
            // Epilogue: O / l -> 16-bit, one 256-byte row per thread.  The next unit's first P V_t,
            // which overwrites O_t, waits for P-ready of that unit: every warp of the group arrives
            // on it only after this read.
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
