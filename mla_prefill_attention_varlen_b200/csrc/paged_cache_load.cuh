// Paged KV-cache gather (the "PagedCacheLoadOperation" page of the Ascend
// Transformer Boost C API, ND cache format): copies each batch entry's cached
// tokens out of a block-paged key / value cache into packed key / value
// tensors -- the packed [tokens, heads, dim] layout the prefill kernel reads.
//
// For batch entry b with length len_b, start s_b and packed offset
// o_b = len_0 + ... + len_{b-1}, token t < len_b sits at logical position
// p = s_b + t, i.e. in slot p mod block_size of physical block
// blockTables[b][p / block_size], and is copied to row o_b + t.
//
// Byte movement only: one warp copies one token row (heads x dim elements,
// contiguous in cache and output) with 16-byte vector loads and stores.  The
// kernel is HBM-bound; its roofline is the copy bandwidth.
#pragma once

#include <cstdint>

namespace mla {

constexpr int kGatherThreads = 256;
constexpr int kPagedPlanThreads = 1024;

// Lengths (plain or running sums) -> packed offsets, clamped to the output's
// token count (kStatusSeqlen on any inconsistency).  offs[batch] = total rows.
__global__ void __launch_bounds__(kPagedPlanThreads)
    paged_plan_kernel(const int *__restrict__ context_lens, int batch, int cumsum, long long num_tokens, int *offs,
                      int *status) {
    __shared__ long long warp_sums[32];
    __shared__ int bad;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    long long carry = 0;
    for (int base = 0; base < batch; base += blockDim.x) {
        const int b = base + threadIdx.x;
        long long len = 0;
        if (b < batch) {
            len = cumsum ? (long long)context_lens[b + 1] - context_lens[b] : context_lens[b];
            if (len < 0) {
                bad = 1;
                len = 0;
            }
        }
        long long tot;
        const long long pre = carry + block_exclusive_scan(len, tot, warp_sums);
        if (b < batch) {
            const long long o = pre < num_tokens ? pre : num_tokens;
            const long long e = pre + len < num_tokens ? pre + len : num_tokens;
            if (e - o != len) bad = 1;
            offs[b] = static_cast<int>(o);
        }
        carry += tot;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        offs[batch] = static_cast<int>(carry < num_tokens ? carry : num_tokens);
        if (bad) atomicCAS(status, 0, kStatusSeqlen);
    }
}

struct GatherParams {
    const uint8_t *key_cache, *value_cache;
    long long kc_block, kc_slot, vc_block, vc_slot;  // byte strides of a block / a slot
    int key_row, value_row;                          // bytes per token row (multiples of 16)
    uint8_t *key, *value;
    long long key_tok, value_tok;                    // byte strides of an output token
    const int *tables;
    long long table_stride;  // elements between batch rows of the block table
    int width;               // logical blocks per batch row of the table
    int num_blocks, block_size;
    const int *starts;  // nullable: every entry starts at position 0
    const int *offs;    // [batch + 1] packed offsets (offs[batch] = rows to write)
    int batch;
    int *status;
};

// Copies `bytes` (a multiple of 16) from src to dst with the 32 lanes of a warp,
// four 16-byte vectors in flight per lane.
__device__ __forceinline__ void warp_copy_row(uint8_t *dst, const uint8_t *src, int bytes, int lane) {
    const int n = bytes >> 4;
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
    uint4 *d = reinterpret_cast<uint4 *>(dst);
    int i = lane;
    for (; i + 96 < n; i += 128) {
        const uint4 a = __ldg(s + i), b = __ldg(s + i + 32), c = __ldg(s + i + 64), e = __ldg(s + i + 96);
        d[i] = a;
        d[i + 32] = b;
        d[i + 64] = c;
        d[i + 96] = e;
    }
    for (; i < n; i += 32) d[i] = __ldg(s + i);
}

__device__ __forceinline__ void warp_zero_row(uint8_t *dst, int bytes, int lane) {
    uint4 *d = reinterpret_cast<uint4 *>(dst);
    for (int i = lane; i < (bytes >> 4); i += 32) d[i] = make_uint4(0, 0, 0, 0);
}

__global__ void __launch_bounds__(kGatherThreads) paged_gather_kernel(const GatherParams p) {
    const int lane = threadIdx.x & 31;
    const int warps_per_block = kGatherThreads / 32;
    const int total = p.offs[p.batch];
    const int nwarps = gridDim.x * warps_per_block;
    for (int g = blockIdx.x * warps_per_block + (threadIdx.x >> 5); g < total; g += nwarps) {
        int lo = 0, hi = p.batch - 1;  // last entry with offs[b] <= g (empty entries are skipped)
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.offs[mid] <= g) lo = mid; else hi = mid - 1;
        }
        const long long pos = (long long)(p.starts ? p.starts[lo] : 0) + (g - p.offs[lo]);
        const long long lb = pos >= 0 ? pos / p.block_size : -1;
        const int within = pos >= 0 ? static_cast<int>(pos % p.block_size) : 0;
        const int blk = (lb >= 0 && lb < p.width) ? p.tables[(long long)lo * p.table_stride + lb] : -1;
        uint8_t *kd = p.key + (long long)g * p.key_tok;
        uint8_t *vd = p.value + (long long)g * p.value_tok;
        if (blk >= 0 && blk < p.num_blocks) {
            warp_copy_row(kd, p.key_cache + blk * p.kc_block + within * p.kc_slot, p.key_row, lane);
            warp_copy_row(vd, p.value_cache + blk * p.vc_block + within * p.vc_slot, p.value_row, lane);
        } else {
            warp_zero_row(kd, p.key_row, lane);
            warp_zero_row(vd, p.value_row, lane);
            if (lane == 0) atomicCAS(p.status, 0, kStatusIndex);
        }
    }
}

}  // namespace mla
