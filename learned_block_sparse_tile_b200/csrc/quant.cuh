// Per-tile FP8 (e4m3) quantisation of tile-ordered Q or K for the FP8 attention variant.
// Not on the pages (their kernel quantises to INT8 by an unpublished recipe). Reading adopted: for each
// (head, 128-row tile) the scale is s = amax(|x|) over the tile's real rows / 448 (1 when that is 0), kept
// as fp32; each code is x / s rounded to nearest-even e4m3 with saturation at +-448. Padding rows
// are zero and stay zero. HBM bound: reads 2 bytes and writes 1 byte per element.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace veda {

struct QuantArgs {
    const __nv_bfloat16* x_t;    // [n_heads, n_slots, D]
    const int32_t* valid_count;  // [n_tiles]
    uint8_t* codes;              // [n_heads, n_slots, D]
    float* scales;               // [n_heads, n_tiles]
    int64_t n_slots;
    int32_t n_tiles;
};

// x / s rounded once to e4m3. The quotient is formed in double and narrowed to fp32 with round-to-odd
// (truncate, then set the last bit when anything was cut off), so the final round-to-nearest-even into
// e4m3 (3 mantissa bits, far fewer than fp32's 23) equals rounding the double quotient directly. A plain
// fp32 division would round twice: quotients of bf16 values by amax / 448 often land within a few ulps of
// an e4m3 midpoint (for example 42.0000014 between 40 and 44) and the first rounding would move them
// onto it.
__device__ __forceinline__ float quotient_round_odd(float x, float s) {
    const double q = double(x) / double(s);
    float r = __double2float_rz(q);
    if (double(r) != q) r = __int_as_float(__float_as_int(r) | 1);
    return r;
}

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// One CTA per (tile, head), 256 threads; D / 8 threads cover a row (16 bytes each) and each thread keeps its
// 8 values of 128 / (256 / (D / 8)) rows in registers between the amax pass and the conversion pass.
template <int D>
__global__ void __launch_bounds__(256) quantize_fp8_kernel(const QuantArgs a) {
    constexpr int kTpr = D / 8;
    constexpr int kRpp = 256 / kTpr;
    constexpr int kPasses = 128 / kRpp;
    __shared__ float red[8];
    const int tile = blockIdx.x, hh = blockIdx.y, tid = threadIdx.x;
    const int c = tid % kTpr, r0 = tid / kTpr;
    const int vc = __ldg(a.valid_count + tile);
    const int64_t base = (int64_t(hh) * a.n_slots + int64_t(tile) * 128) * D + c * 8;
    uint4 v[kPasses];
    float amax = 0.f;
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        const int r = r0 + p * kRpp;
        v[p] = *reinterpret_cast<const uint4*>(a.x_t + base + int64_t(r) * D);
        if (r < vc) {
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[p]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    float m = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
    const float s = m > 0.f ? m / 448.f : 1.f;
    if (tid == 0) a.scales[int64_t(hh) * a.n_tiles + tile] = s;
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        const int r = r0 + p * kRpp;
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[p]);
        uint32_t w[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float2 f0 = __bfloat1622float2(h2[2 * e]), f1 = __bfloat1622float2(h2[2 * e + 1]);
            w[e] = uint32_t(e4m3x2(quotient_round_odd(f0.x, s), quotient_round_odd(f0.y, s))) |
                   (uint32_t(e4m3x2(quotient_round_odd(f1.x, s), quotient_round_odd(f1.y, s))) << 16);
        }
        *reinterpret_cast<uint2*>(a.codes + base + int64_t(r) * D) = make_uint2(w[0], w[1]);
    }
}

}  // namespace veda
