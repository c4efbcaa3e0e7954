// Per-tile quantisation of tile-ordered Q or K for the 8-bit attention variants.
// The pages' own kernel computes Q K^T in INT8 by a recipe they do not print. Readings adopted, per
// (head, 128-row tile), with the scale kept as fp32 (1 when the amax is 0):
//  e4m3: s = amax(|x| over the tile's real rows) / 448; code = x / s rounded to nearest-even e4m3,
//        saturating at +-448;
//  int8: s = amax / 127; code = x / s rounded to the nearest integer, ties to even, within +-127.
// Padding rows are zero and stay zero. HBM bound in principle: reads 2 bytes and writes 1 byte per element.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace veda {

struct QuantArgs {
    const __nv_bfloat16* x_t;    // [n_heads, n_slots, D]
    const int32_t* valid_count;  // [n_tiles]
    uint8_t* codes;              // [n_heads, n_slots, D]
    float* scales;               // [n_heads, n_tiles]
    int64_t n_slots;
    int32_t n_tiles;
};

// x / s rounded once to e4m3. The quotient is narrowed to fp32 with round-to-odd (the truncated quotient,
// with its last bit set when anything was cut off), so the final round-to-nearest-even into e4m3 (3
// mantissa bits, far fewer than fp32's 23) equals rounding the exact quotient directly. A plain fp32
// division would round twice: quotients of bf16 values by amax / 448 often land within a few ulps of an
// e4m3 midpoint (for example 42.0000014 between 40 and 44) and the first rounding would move them onto it.
//
// Round-to-odd needs only a faithful quotient q (one of the two fp32 neighbours of x / s) and the side of
// q on which x / s lies. q: x times the tile's reciprocal inv = 1/s, refined once by the FMA residual
// (q0 + (x - q0 s) inv is within one unit of x / s). The side: the sign of x - q s, formed exactly inside
// one FMA and rounded once, which keeps its sign and its being zero (s > 0). When |x / s| > |q| the
// truncation is q, otherwise q one unit lower in magnitude; the inexact result is that value with its
// last bit set. Quotients small enough to underflow round to 0 in e4m3 whatever happens here.
// The last step on the bits: when x / s lies on the zero side of q (r and q of opposite signs) the
// magnitude drops by one unit, which never borrows into the sign since |q| >= one unit.
__device__ __forceinline__ float round_odd_bits(float q, float r) {
    const uint32_t b = __float_as_uint(q);
    if (r == 0.f || q == 0.f) return q;
    return __uint_as_float((b - ((__float_as_uint(r) ^ b) >> 31)) | 1u);
}

// Two quotients at once on the packed f32x2 pipe; s2 = (s, s), ms2 = (-s, -s), inv2 = (1/s, 1/s).
__device__ __forceinline__ void quotient_round_odd2(float x0, float x1, uint64_t ms2, uint64_t inv2, float& q0_odd,
                                                    float& q1_odd) {
    const uint64_t x = ptx::f2_pack(x0, x1);
    const uint64_t q0 = ptx::f2_mul(x, inv2);
    const uint64_t q = ptx::f2_fma(ptx::f2_fma(q0, ms2, x), inv2, q0);
    const uint64_t r = ptx::f2_fma(q, ms2, x);
    float qa, qb, ra, rb;
    ptx::f2_unpack(q, qa, qb);
    ptx::f2_unpack(r, ra, rb);
    q0_odd = round_odd_bits(qa, ra);
    q1_odd = round_odd_bits(qb, rb);
}

__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Code formats of the 8-bit variants.
enum TileCode : int { kCodeE4M3 = 1, kCodeI8 = 2 };

// Round-to-odd quotient to an int8 code: nearest integer, ties to even (the fp32 round-to-odd value
// carries enough bits for that rounding to equal rounding the exact quotient), within +-127.
__device__ __forceinline__ uint32_t i8_code(float q_odd) {
    const int c = __float2int_rn(q_odd);
    return uint32_t(max(-127, min(127, c))) & 0xFFu;
}

// Quantises one (head, 128-row tile) held by a 256-thread CTA: D / 8 threads cover a row (8 bf16 = 16
// bytes each), thread tid holds rows r0 + p * kRpp (r0 = tid / (D / 8)) of its 8 columns in v[p]. Rows
// from vc on are padding (zero, and left out of the amax). Writes the tile's scale (thread 0) and the
// codes of all 128 rows to codes (this thread's column chunk of row 0; rows are D bytes apart). Contains a
// block barrier: every thread of the CTA must call it.
template <int D, int kCode>
__device__ __forceinline__ void quantize_tile(const uint4* v, int r0, int vc, float* red8, uint8_t* codes,
                                              float* scale) {
    constexpr int kTpr = D / 8;
    constexpr int kRpp = 256 / kTpr;
    constexpr int kPasses = 128 / kRpp;
    float amax = 0.f;
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        if (r0 + p * kRpp < vc) {
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
    if ((threadIdx.x & 31) == 0) red8[threadIdx.x >> 5] = amax;
    __syncthreads();
    float m = red8[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red8[w]);
    const float s = m > 0.f ? m / (kCode == kCodeI8 ? 127.f : 448.f) : 1.f;
    const float inv = 1.f / s;
    const uint64_t inv2 = ptx::f2_pack(inv, inv), ms2 = ptx::f2_pack(-s, -s);
    if (threadIdx.x == 0) *scale = s;
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[p]);
        uint32_t w[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float2 f0 = __bfloat1622float2(h2[2 * e]), f1 = __bfloat1622float2(h2[2 * e + 1]);
            float q0, q1, q2, q3;
            quotient_round_odd2(f0.x, f0.y, ms2, inv2, q0, q1);
            quotient_round_odd2(f1.x, f1.y, ms2, inv2, q2, q3);
            if constexpr (kCode == kCodeI8)
                w[e] = i8_code(q0) | (i8_code(q1) << 8) | (i8_code(q2) << 16) | (i8_code(q3) << 24);
            else
                w[e] = uint32_t(e4m3x2(q0, q1)) | (uint32_t(e4m3x2(q2, q3)) << 16);
        }
        *reinterpret_cast<uint2*>(codes + int64_t(r0 + p * kRpp) * D) = make_uint2(w[0], w[1]);
    }
}

// One CTA per (tile, head), 256 threads, over a tile-ordered bf16 tensor. HBM bound: reads 2 bytes and
// writes 1 byte per element.
template <int D, int kCode>
__global__ void __launch_bounds__(256) quantize_kernel(const QuantArgs a) {
    constexpr int kTpr = D / 8;
    constexpr int kRpp = 256 / kTpr;
    constexpr int kPasses = 128 / kRpp;
    __shared__ float red[8];
    const int tile = blockIdx.x, hh = blockIdx.y, tid = threadIdx.x;
    const int c = tid % kTpr, r0 = tid / kTpr;
    const int vc = __ldg(a.valid_count + tile);
    const int64_t base = (int64_t(hh) * a.n_slots + int64_t(tile) * 128) * D + c * 8;
    uint4 v[kPasses];
#pragma unroll
    for (int p = 0; p < kPasses; ++p) v[p] = *reinterpret_cast<const uint4*>(a.x_t + base + int64_t(r0 + p * kRpp) * D);
    quantize_tile<D, kCode>(v, r0, vc, red, a.codes + base, a.scales + int64_t(hh) * a.n_tiles + tile);
}

}  // namespace veda
