// Tile-pair logits of the predictor, fp32 on the CUDA cores.
// veda_core.py (ComfyUI-FunPack), "predictor", logits: per head, x_hat = feats @ P + feats[:, :D]
// (P is [3D, D]) for the query and the key side, then scores = q_hat @ k_hat^T / sqrt(D).
//
// Both steps run one batched fp32 GEMM kernel with two epilogues: "add the first N columns of A" for the
// projection and "divide by sqrt(D)" for the scores. A CTA of 256 threads computes a (16 TM) x (16 TN)
// output tile, TM x TN outputs per thread held as packed f32x2 pairs (fma.rn.f32x2: two independent
// fp32 FMAs, each rounded once), over 16-deep k slices that are double-buffered in shared memory (the next
// slice is read from global memory into registers while the current one is multiplied). Every output is
// accumulated over k in increasing order with one rounding per FMA, the order of a plain dot product.
// The query and key projections share one launch (blockIdx.z runs over both sides' heads).
#pragma once

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "ptx.cuh"

namespace veda {

struct GemmArgs {
    const float* A;  // [batch][M][K] row-major (lda = K)
    const float* B;  // kBT: [batch][N][K]; else [batch][K][N]
    float* C;        // [batch][M][N]
    // optional second operand set for blockIdx.z >= nb (same shapes and strides)
    const float* A2;
    const float* B2;
    float* C2;
    int nb;          // batches of the first set
    int M, N, K;     // K a multiple of 16; without kBT, N a multiple of 4
    int64_t sA, sB, sC;  // batch strides in elements
    float div;           // epilogue divisor (scores)
};

// kBT: C = A B^T / div (scores). !kBT: C = A B + A[:, :N] (projection with the mean part added back).
template <bool kBT, int TM, int TN>
__global__ void __launch_bounds__(256, 2) gemm_f32_kernel(const GemmArgs a) {
    static_assert(TM % 4 == 0 && TN % 4 == 0, "per-thread tile in multiples of 4");
    constexpr int BM = 16 * TM, BN = 16 * TN, BK = 16;
    constexpr int LA = BM / 64, LB = BN / 64;  // float4 loads per thread per k slice
    __shared__ __align__(16) float As[2][BK][BM + 4];
    __shared__ __align__(16) float Bs[2][BK][BN + 4];
    int bz = blockIdx.z;
    const bool second = bz >= a.nb;
    if (second) bz -= a.nb;
    const float* A = (second ? a.A2 : a.A) + bz * a.sA;
    const float* B = (second ? a.B2 : a.B) + bz * a.sB;
    float* C = (second ? a.C2 : a.C) + bz * a.sC;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;

    float4 ra[LA], rb[LB];
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    // global -> registers: A as BM rows x 16 k (row = f / 4, k = 4 (f % 4)); B likewise for kBT, else as
    // 16 k x BN columns (k = f / (BN / 4), n = 4 (f % (BN / 4)))
    auto load = [&](int k0) {
#pragma unroll
        for (int r = 0; r < LA; ++r) {
            const int f = tid + 256 * r, m = m0 + (f >> 2);
            ra[r] = m < a.M ? *reinterpret_cast<const float4*>(A + int64_t(m) * a.K + k0 + (f & 3) * 4) : zero;
        }
#pragma unroll
        for (int r = 0; r < LB; ++r) {
            const int f = tid + 256 * r;
            if (kBT) {
                const int n = n0 + (f >> 2);
                rb[r] = n < a.N ? *reinterpret_cast<const float4*>(B + int64_t(n) * a.K + k0 + (f & 3) * 4) : zero;
            } else {
                const int kk = f / (BN / 4), n = n0 + (f % (BN / 4)) * 4;
                rb[r] = n < a.N ? *reinterpret_cast<const float4*>(B + int64_t(k0 + kk) * a.N + n) : zero;
            }
        }
    };
    // registers -> shared memory, k-major ([k][m] and [k][n])
    auto store = [&](int buf) {
#pragma unroll
        for (int r = 0; r < LA; ++r) {
            const int f = tid + 256 * r, row = f >> 2, k4 = (f & 3) * 4;
            As[buf][k4 + 0][row] = ra[r].x;
            As[buf][k4 + 1][row] = ra[r].y;
            As[buf][k4 + 2][row] = ra[r].z;
            As[buf][k4 + 3][row] = ra[r].w;
        }
#pragma unroll
        for (int r = 0; r < LB; ++r) {
            const int f = tid + 256 * r;
            if (kBT) {
                const int row = f >> 2, k4 = (f & 3) * 4;
                Bs[buf][k4 + 0][row] = rb[r].x;
                Bs[buf][k4 + 1][row] = rb[r].y;
                Bs[buf][k4 + 2][row] = rb[r].z;
                Bs[buf][k4 + 3][row] = rb[r].w;
            } else {
                *reinterpret_cast<float4*>(&Bs[buf][f / (BN / 4)][(f % (BN / 4)) * 4]) = rb[r];
            }
        }
    };

    // thread (tx, ty) owns rows (i / 4) 64 + 4 ty + i % 4 and columns (j / 4) 64 + 4 tx + j % 4
    uint64_t acc[TM][TN / 2];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN / 2; ++j) acc[i][j] = 0;

    const int nk = a.K / BK;
    load(0);
    store(0);
    __syncthreads();
    for (int kt = 0; kt < nk; ++kt) {
        const int cur = kt & 1;
        if (kt + 1 < nk) load((kt + 1) * BK);
#pragma unroll
        for (int k = 0; k < BK; ++k) {
            float av[TM], bv[TN];
#pragma unroll
            for (int h = 0; h < TM / 4; ++h)
                *reinterpret_cast<float4*>(av + 4 * h) = *reinterpret_cast<const float4*>(&As[cur][k][64 * h + 4 * ty]);
#pragma unroll
            for (int h = 0; h < TN / 4; ++h)
                *reinterpret_cast<float4*>(bv + 4 * h) = *reinterpret_cast<const float4*>(&Bs[cur][k][64 * h + 4 * tx]);
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const uint64_t ai = ptx::f2_pack(av[i], av[i]);
#pragma unroll
                for (int j = 0; j < TN / 2; ++j) acc[i][j] = ptx::f2_fma(ai, ptx::f2_pack(bv[2 * j], bv[2 * j + 1]), acc[i][j]);
            }
        }
        // the other buffer was last read before the barrier that ended the previous slice
        if (kt + 1 < nk) store(cur ^ 1);
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const int m = m0 + (i >> 2) * 64 + 4 * ty + (i & 3);
        if (m >= a.M) continue;
#pragma unroll
        for (int j = 0; j < TN / 2; ++j) {
            float v[2];
            ptx::f2_unpack(acc[i][j], v[0], v[1]);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int n = n0 + ((2 * j) >> 2) * 64 + 4 * tx + ((2 * j) & 3) + u;
                if (n >= a.N) continue;
                C[int64_t(m) * a.N + n] = kBT ? v[u] / a.div : v[u] + A[int64_t(m) * a.K + n];
            }
        }
    }
}

// The three products of the predictor for n_heads heads: q_hat and k_hat ([n_heads][nv][dim] each, in
// one launch) and the scores [n_heads][nv][nv]. dim is 64 or 128 (checked by the callers).
inline void launch_score_gemms(const float* feats_q, const float* feats_k, const float* proj_q, const float* proj_k,
                               float* qh, float* kh, float* scores, int nv, int dim, int n_heads, cudaStream_t s) {
    GemmArgs g{};
    g.A = feats_q;
    g.B = proj_q;
    g.C = qh;
    g.A2 = feats_k;
    g.B2 = proj_k;
    g.C2 = kh;
    g.nb = n_heads;
    g.M = nv;
    g.N = dim;
    g.K = 3 * dim;
    g.sA = int64_t(nv) * 3 * dim;
    g.sB = int64_t(3) * dim * dim;
    g.sC = int64_t(nv) * dim;
    g.div = 1.f;
    // 64-row x (dim)-column tiles: with one output tile across the projection's columns the feature rows
    // are read once, and the 819-row heads of the 104k grid give 13 tiles per head and side
    if (dim == 128)
        gemm_f32_kernel<false, 4, 8><<<dim3(1, unsigned((nv + 63) / 64), unsigned(2 * n_heads)), 256, 0, s>>>(g);
    else
        gemm_f32_kernel<false, 4, 4><<<dim3(1, unsigned((nv + 63) / 64), unsigned(2 * n_heads)), 256, 0, s>>>(g);
    GemmArgs h{};
    h.A = qh;
    h.B = kh;
    h.C = scores;
    h.nb = n_heads;
    h.M = nv;
    h.N = nv;
    h.K = dim;
    h.sA = int64_t(nv) * dim;
    h.sB = int64_t(nv) * dim;
    h.sC = int64_t(nv) * nv;
    h.div = float(std::sqrt(double(dim)));
    gemm_f32_kernel<true, 8, 8><<<dim3(unsigned((nv + 127) / 128), unsigned((nv + 127) / 128), unsigned(n_heads)), 256, 0, s>>>(h);
}

}  // namespace veda
