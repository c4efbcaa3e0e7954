// Tile-order gather of one [S, H, D] bf16 tensor with the per-tile [mean | max | min] pooling fused in.
// veda_core.py (ComfyUI-FunPack): "tiles", gather (x[perm, heads], zero on padding slots) and
// "predictor", pool (mean = fp32 sum of the tile's real rows / their count; max and min over the real
// rows only; zero for a tile with no real row).
//
// One CTA per (tile, head): 256 threads move the tile's 128 rows of D bf16 with 16-byte loads (each
// row is one contiguous 2*D-byte run of the source), keep them in registers, write them to the
// head-major tile-ordered output and reduce them column-wise in the same pass. HBM bound.
// kCode != 0 writes the tile as 8-bit codes (e4m3 or int8) with its per-tile scale (the 8-bit Q/K
// variants' quantisation, quant.cuh) instead of bf16, from the same registers.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"
#include "quant.cuh"

namespace veda {

struct GatherArgs {
    const __nv_bfloat16* x;
    int64_t s0, s1;               // element strides of x on S and H (D stride is 1)
    const int32_t* heads;         // [n_heads]
    const int32_t* perm;          // [n_slots]
    const int32_t* valid_count;   // [n_tiles]
    __nv_bfloat16* x_t;           // [n_heads, n_slots, D] (bf16 form), or null: pooled features only
    uint8_t* codes;               // [n_heads, n_slots, D] 8-bit codes (kCode != 0)
    float* scales;                // [n_heads, n_tiles] (kCode != 0)
    int32_t n_tiles;
    float* feats;                 // [n_heads, n_video, 3D] or null
    int64_t n_slots;
    int32_t n_video;
    int32_t h_total;
    int* err;                     // latched error bits; bit 4 = head index out of range
    // squared row norms for the attend's bound on its logits (either may be null):
    float* row_sq;                // [n_heads, seq_len] ||x||^2 of every real row, at its packed row
    unsigned* max_sq;             // [n_heads] largest ||x||^2 of the head's real rows (float bits; starts at 0)
    int64_t seq_len;
};

// CTAs of the pool-only launch (kPoolOnly: no tile copy, veda_pool) resident per SM, which its registers
// are held to: a pass that only reads keeps more bytes in flight with more CTAs resident.
constexpr int kPoolCtasPerSm = 4;

template <int D, int kCode = 0, bool kPoolOnly = false>
__global__ void __launch_bounds__(256, kPoolOnly ? kPoolCtasPerSm : 0) gather_pool_kernel(const GatherArgs a) {
    static_assert(!(kPoolOnly && kCode != 0), "the 8-bit gathers write codes");
    constexpr int kTpr = D / 8;          // threads per row (8 bf16 = 16 bytes each)
    constexpr int kRpp = 256 / kTpr;     // rows per pass
    constexpr int kPasses = 128 / kRpp;  // passes over the tile
    constexpr int kWarps = 8;
    __shared__ float red[3][kWarps][D];
    __shared__ unsigned warp_max[kWarps];  // each warp's largest row norm (float bits)

    const int tile = blockIdx.x, hh = blockIdx.y;
    const int tid = threadIdx.x, c = tid % kTpr, r0 = tid / kTpr;
    const int64_t head = __ldg(a.heads + hh);
    if (head < 0 || head >= a.h_total) {  // uniform across the CTA
        if (threadIdx.x == 0) atomicOr(a.err, 4);
        return;
    }
    const int vc = __ldg(a.valid_count + tile);
    const __nv_bfloat16* src = a.x + head * a.s1 + c * 8;

    uint4 v[kPasses];
    int pr[kPasses];  // packed row of each pass's row (-1: padding)
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        const int r = r0 + p * kRpp;
        pr[p] = __ldg(a.perm + int64_t(tile) * 128 + r);
        v[p] = pr[p] >= 0 ? __ldg(reinterpret_cast<const uint4*>(src + int64_t(pr[p]) * a.s0)) : make_uint4(0, 0, 0, 0);
    }
    const bool norms = a.row_sq != nullptr || a.max_sq != nullptr;
    const int warp = tid >> 5, lane = tid & 31;
    if (norms) {
        // ||x||^2 per row. Each thread squares its 8 columns of each of its kPasses rows; the kTpr threads
        // of a row then add up with a transposed butterfly: at every step a thread keeps half of its rows
        // and hands the other half to its partner, so the kPasses rows cost kPasses - 1 + log2(kTpr /
        // kPasses) shuffles (when kTpr >= kPasses) instead of kPasses log2(kTpr)
        static_assert(kTpr >= kPasses, "one row per thread pair after the butterfly");
        float ss[kPasses];
#pragma unroll
        for (int p = 0; p < kPasses; ++p) {
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[p]);
            uint64_t acc = ptx::f2_pack(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                const uint64_t f2 = ptx::f2_pack(f.x, f.y);
                acc = ptx::f2_fma(f2, f2, acc);
            }
            float lo, hi;
            ptx::f2_unpack(acc, lo, hi);
            ss[p] = lo + hi;
        }
        // after the step with distance d (kPasses / 2, ..., 1 in units of rows) a thread holds the partial
        // sums of the rows whose index bits match its own lane bits at those positions
#pragma unroll
        for (int d = kPasses / 2, bit = kPasses / 2; d >= 1; d >>= 1, bit >>= 1) {
            const bool upper = (c & bit) != 0;
#pragma unroll
            for (int i = 0; i < d; ++i) {
                // keep rows i + (upper ? d : 0), send the other
                const float send = upper ? ss[i] : ss[i + d];
                const float got = __shfl_xor_sync(0xffffffffu, send, bit);
                ss[i] = (upper ? ss[i + d] : ss[i]) + got;
            }
        }
        // ss[0] is now the partial sum of row p = c % kPasses over the threads c' == c (mod kPasses)
#pragma unroll
        for (int off = kPasses; off < kTpr; off <<= 1) ss[0] += __shfl_xor_sync(0xffffffffu, ss[0], off);
        const int pm = c % kPasses;
        int my_pr = pr[0];
#pragma unroll
        for (int p = 1; p < kPasses; ++p) my_pr = pm == p ? pr[p] : my_pr;
        const bool mine = c < kPasses && my_pr >= 0;
        if (mine && a.row_sq != nullptr) a.row_sq[int64_t(hh) * a.seq_len + my_pr] = ss[0];
        // non-negative floats order as their bit patterns; the warps' maxima meet after the next barrier
        const unsigned wm = __reduce_max_sync(0xffffffffu, mine ? __float_as_uint(ss[0]) : 0u);
        if (lane == 0) warp_max[warp] = wm;
    }
    // the CTA's largest row norm into max_sq (after a barrier that follows the warp_max writes)
    auto raise_max = [&]() {
        if (a.max_sq != nullptr && tid == 0) {
            unsigned m = 0u;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) m = max(m, warp_max[w]);
            atomicMax(a.max_sq + hh, m);
        }
    };
    const int64_t base = (int64_t(hh) * a.n_slots + int64_t(tile) * 128) * D + c * 8;
    if constexpr (kCode != 0) {
        __shared__ float red8[8];
        quantize_tile<D, kCode>(v, r0, vc, red8, a.codes + base, a.scales + int64_t(hh) * a.n_tiles + tile);
    } else if (!kPoolOnly && a.x_t != nullptr) {
        __nv_bfloat16* dst = a.x_t + base;
#pragma unroll
        for (int p = 0; p < kPasses; ++p) *reinterpret_cast<uint4*>(dst + int64_t(r0 + p * kRpp) * D) = v[p];
    }

    if (a.feats == nullptr || tile >= a.n_video) {
        if (norms) {
            __syncthreads();
            raise_max();
        }
        return;
    }

    // column sums in fp32 (packed pairs), maxima and minima on the bf16 pairs themselves (exact either way)
    uint64_t sum2[4];
    __nv_bfloat162 mx2[4], mn2[4];
    const __nv_bfloat162 ninf = __floats2bfloat162_rn(-INFINITY, -INFINITY), pinf = __floats2bfloat162_rn(INFINITY, INFINITY);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        sum2[e] = ptx::f2_pack(0.f, 0.f);
        mx2[e] = ninf;
        mn2[e] = pinf;
    }
#pragma unroll
    for (int p = 0; p < kPasses; ++p) {
        if (r0 + p * kRpp < vc) {
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[p]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                sum2[e] = ptx::f2_add(sum2[e], ptx::f2_pack(f.x, f.y));
                mx2[e] = __hmax2(mx2[e], h2[e]);
                mn2[e] = __hmin2(mn2[e], h2[e]);
            }
        }
    }
    float sum[8], mx[8], mn[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        ptx::f2_unpack(sum2[e], sum[2 * e], sum[2 * e + 1]);
        const float2 hi = __bfloat1622float2(mx2[e]), lo = __bfloat1622float2(mn2[e]);
        mx[2 * e] = hi.x;
        mx[2 * e + 1] = hi.y;
        mn[2 * e] = lo.x;
        mn[2 * e + 1] = lo.y;
    }
    // lanes that hold the same columns differ in the bits above log2(kTpr)
#pragma unroll
    for (int off = kTpr; off < 32; off <<= 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sum[e] += __shfl_xor_sync(0xffffffffu, sum[e], off);
            mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], off));
            mn[e] = fminf(mn[e], __shfl_xor_sync(0xffffffffu, mn[e], off));
        }
    }
    if (lane < kTpr) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            red[0][warp][c * 8 + e] = sum[e];
            red[1][warp][c * 8 + e] = mx[e];
            red[2][warp][c * 8 + e] = mn[e];
        }
    }
    __syncthreads();
    if (norms) raise_max();
    if (tid < D) {
        float s = 0.f, hi = -INFINITY, lo = INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            s += red[0][w][tid];
            hi = fmaxf(hi, red[1][w][tid]);
            lo = fminf(lo, red[2][w][tid]);
        }
        float* f = a.feats + (int64_t(hh) * a.n_video + tile) * (3 * D);
        if (vc > 0) {
            f[tid] = s / float(vc);
            f[D + tid] = hi;
            f[2 * D + tid] = lo;
        } else {
            f[tid] = 0.f;
            f[D + tid] = 0.f;
            f[2 * D + tid] = 0.f;
        }
    }
}

}  // namespace veda
