// Tile-pair logits of the predictor, fp32 on the CUDA cores.
// veda_core.py (ComfyUI-FunPack), "predictor", logits: per head, x_hat = feats @ P + feats[:, :D]
// (P is [3D, D]) for the query and the key side, then scores = q_hat @ k_hat^T / sqrt(D).
//
// Both steps run one batched fp32 GEMM kernel (64x64 output tile per CTA, 16-deep k slices staged in
// shared memory, 4x4 outputs per thread) with two epilogues: "add the first N columns of A" for the
// projection and "divide by sqrt(D)" for the scores. 8 GFLOP at the 104k-token size: tens of us.
#pragma once

#include <cstdint>

namespace veda {

struct GemmArgs {
    const float* A;  // [batch][M][K] row-major (lda = K)
    const float* B;  // kBT: [batch][N][K]; else [batch][K][N]
    float* C;        // [batch][M][N]
    int M, N, K;
    int64_t sA, sB, sC;  // batch strides in elements
    float div;           // epilogue divisor (scores)
};

// kBT: C = A B^T / div (scores). !kBT: C = A B + A[:, :N] (projection with the mean part added back).
template <bool kBT>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const GemmArgs a) {
    constexpr int BM = 64, BN = 64, BK = 16;
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    const int bz = blockIdx.z;
    const float* A = a.A + bz * a.sA;
    const float* B = a.B + bz * a.sB;
    float* C = a.C + bz * a.sC;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    float acc[4][4] = {};

    // loaders: 64 rows x 16 k as 256 float4 (row = tid / 4, k4 = tid % 4)
    const int lr = tid >> 2, lk = (tid & 3) * 4;
    for (int k0 = 0; k0 < a.K; k0 += BK) {
        {
            const int m = m0 + lr;
            float4 va = make_float4(0.f, 0.f, 0.f, 0.f);
            if (m < a.M) va = *reinterpret_cast<const float4*>(A + int64_t(m) * a.K + k0 + lk);
            As[lk + 0][lr] = va.x;
            As[lk + 1][lr] = va.y;
            As[lk + 2][lr] = va.z;
            As[lk + 3][lr] = va.w;
        }
        if (kBT) {
            const int n = n0 + lr;
            float4 vb = make_float4(0.f, 0.f, 0.f, 0.f);
            if (n < a.N) vb = *reinterpret_cast<const float4*>(B + int64_t(n) * a.K + k0 + lk);
            Bs[lk + 0][lr] = vb.x;
            Bs[lk + 1][lr] = vb.y;
            Bs[lk + 2][lr] = vb.z;
            Bs[lk + 3][lr] = vb.w;
        } else {
            // 16 k x 64 n as 256 float4 (k = tid / 16, n4 = tid % 16)
            const int kk = tid >> 4, nn = (tid & 15) * 4;
            float4 vb = make_float4(0.f, 0.f, 0.f, 0.f);
            if (n0 + nn < a.N) vb = *reinterpret_cast<const float4*>(B + int64_t(k0 + kk) * a.N + n0 + nn);
            *reinterpret_cast<float4*>(&Bs[kk][nn]) = vb;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < BK; ++k) {
            const float4 av = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
            const float4 bv = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
            const float ar[4] = {av.x, av.y, av.z, av.w}, br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= a.M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= a.N) continue;
            float v = acc[i][j];
            if (kBT)
                v = v / a.div;
            else
                v = v + A[int64_t(m) * a.K + n];
            C[int64_t(m) * a.N + n] = v;
        }
    }
}

}  // namespace veda
