// RmsNorm + interleaved RoPE rows of the MLA Prolog (the "MlaProlog" page of
// cann-recipes-infer, 计算公式 section).  The three projections of the page
// (x wq_a, c^Q wq_b, x wkv) are plain GEMMs with fp32 results; this kernel turns
// their rows into the page's outputs:
//   c^Q row      = RmsNorm(row) * gamma_cq                         -> bf16
//   kv row       = RmsNorm(row) * gamma_ckv, rope on the last R    -> bf16
//   q row (head) = RmsNorm(row) (weight 1),  rope on the last R    -> bf16
// with RmsNorm(v) = v / sqrt(mean(v^2) + eps) and the interleaved rope
//   y[2i]   = v[2i]   cos[2i]   - v[2i+1] sin[2i]
//   y[2i+1] = v[2i+1] cos[2i+1] + v[2i]   sin[2i+1]
// where cos / sin are the token's rows of rope_cos / rope_sin [t, R].
//
// HBM-bound: one warp per row, 16-byte loads of the fp32 row kept in registers
// for rows up to 1024 channels (eight adjacent channels per lane and group), a
// warp-shuffle sum of squares, then scale, rotate and store 16-byte groups of
// eight bf16 values.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace mla {

constexpr int kNormThreads = 256;  // 8 warps, one row each at a time

struct NormJob {
    const float *in;      // fp32 rows: row r starts at in + token * in_tok + head * width
    long long in_tok;     // elements between tokens of `in`
    __nv_bfloat16 *out;   // row r starts at out + token * out_tok + head * out_head
    long long out_tok, out_head;
    const __nv_bfloat16 *gamma;  // [width], or null for weight 1
    const __nv_bfloat16 *cos, *sin;  // [tokens, rope] rows with strides cos_tok / sin_tok (rope > 0)
    long long cos_tok, sin_tok;
    int width;  // channels per row (multiple of 4)
    int rope;   // rotated trailing channels (multiple of 4, <= width), 0 for none
    int heads;  // rows per token
    long long rows;  // tokens * heads
};

struct NormParams {
    NormJob job[2];
    int njobs;
    float eps;
};

__device__ __forceinline__ uint2 pack_bf16x4(float a, float b, float c, float d) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
    return make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
}

__device__ __forceinline__ float4 load_bf16x4(const __nv_bfloat16 *p) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// Scales, weights and rotates the four channels c .. c+3 of a row; returns them as bf16.
__device__ __forceinline__ uint2 norm4(const NormJob &j, long long token, int c, float4 v, float inv) {
    v.x *= inv;
    v.y *= inv;
    v.z *= inv;
    v.w *= inv;
    if (j.gamma) {
        const float4 g4 = load_bf16x4(j.gamma + c);
        v.x *= g4.x;
        v.y *= g4.y;
        v.z *= g4.z;
        v.w *= g4.w;
    }
    const int rope0 = j.width - j.rope;  // first rotated channel
    if (c >= rope0) {
        const float4 cs = load_bf16x4(j.cos + token * j.cos_tok + (c - rope0));
        const float4 sn = load_bf16x4(j.sin + token * j.sin_tok + (c - rope0));
        const float y0 = v.x * cs.x - v.y * sn.x, y1 = v.y * cs.y + v.x * sn.y;
        const float y2 = v.z * cs.z - v.w * sn.z, y3 = v.w * cs.w + v.z * sn.w;
        v = make_float4(y0, y1, y2, y3);
    }
    return pack_bf16x4(v.x, v.y, v.z, v.w);
}

__device__ __forceinline__ float sumsq4(float4 v, float ss) {
    return fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
}

__device__ __forceinline__ float warp_sum(float ss) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    return ss;
}

constexpr int kNormRegGroups = 4;  // rows of up to 32 lanes x 4 groups x 8 = 1024 channels stay in registers

__global__ void __launch_bounds__(kNormThreads) rms_norm_rope_kernel(const NormParams p) {
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (kNormThreads / 32);
    const long long total = p.job[0].rows + (p.njobs > 1 ? p.job[1].rows : 0);
    for (long long g = (long long)blockIdx.x * (kNormThreads / 32) + (threadIdx.x >> 5); g < total; g += warps) {
        const bool second = g >= p.job[0].rows;
        const NormJob &j = second ? p.job[1] : p.job[0];
        const long long r = second ? g - p.job[0].rows : g;
        const long long token = r / j.heads;
        const int head = static_cast<int>(r - token * j.heads);
        const float4 *in = reinterpret_cast<const float4 *>(j.in + token * j.in_tok + (long long)head * j.width);
        __nv_bfloat16 *out = j.out + token * j.out_tok + (long long)head * j.out_head;
        const float rw = 1.f / static_cast<float>(j.width);
        if ((j.width & 7) == 0 && j.width <= 256 * kNormRegGroups) {
            // the whole row in registers, eight adjacent channels per lane and group: every load of
            // the row in flight at once, one pass over HBM, 16-byte stores of eight bf16 values
            const int n8 = j.width >> 3;
            float4 lo[kNormRegGroups], hi[kNormRegGroups];
            float ss = 0.f;
#pragma unroll
            for (int k = 0; k < kNormRegGroups; ++k) {
                const int i = lane + 32 * k;
                lo[k] = i < n8 ? __ldg(in + 2 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
                hi[k] = i < n8 ? __ldg(in + 2 * i + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < kNormRegGroups; ++k) ss = sumsq4(hi[k], sumsq4(lo[k], ss));
            const float inv = rsqrtf(warp_sum(ss) * rw + p.eps);
#pragma unroll
            for (int k = 0; k < kNormRegGroups; ++k) {
                const int i = lane + 32 * k;
                if (i < n8) {
                    const uint2 a = norm4(j, token, 8 * i, lo[k], inv), b = norm4(j, token, 8 * i + 4, hi[k], inv);
                    reinterpret_cast<uint4 *>(out)[i] = make_uint4(a.x, a.y, b.x, b.y);
                }
            }
        } else {
            // other rows: sum of squares, then a second pass over the row (an L1 / L2 hit)
            const int n4 = j.width >> 2;
            float ss = 0.f;
#pragma unroll 4
            for (int i = lane; i < n4; i += 32) ss = sumsq4(__ldg(in + i), ss);
            const float inv = rsqrtf(warp_sum(ss) * rw + p.eps);
            for (int i = lane; i < n4; i += 32)
                reinterpret_cast<uint2 *>(out)[i] = norm4(j, token, 4 * i, __ldg(in + i), inv);
        }
    }
}

}  // namespace mla
