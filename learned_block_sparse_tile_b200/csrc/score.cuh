// Tile-pair logits of the predictor on the tensor cores, at fp32-level accuracy.
// veda_core.py (ComfyUI-FunPack), "predictor", logits: per head, x_hat = feats @ P + feats[:, :D] (P is
// [3D, D]) for the query and the key side, then scores = q_hat @ k_hat^T / sqrt(D).
//
// Split tf32. A tf32 operand keeps 10 explicit mantissa bits, too few for fp32 scores on its own, so every
// operand x is split into hi = x rounded to tf32 and lo = x - hi (exact in fp32, |lo| <= 2^-11 |x|), and
// a b is taken as hi_a hi_b + hi_a lo_b + lo_a hi_b: three kind::tf32 products into one fp32 accumulator.
// What is left out, lo_a lo_b (under 2^-22 |a b|) and the bits of the lo parts below tf32 (each under
// 2^-21 |a b| even if the MMA truncates them), is under 1.25 x 2^-20 |a b| per product: the order of the
// rounding of an fp32 dot product itself.
//
// Both products are C[batch] = scale A[batch] B[batch]^T with A [M][K] and B [N][K] K-major fp32. The
// projection's B is (P + E)^T, written first by transpose_kernel, where E is the identity in P's first D
// rows: feats @ (P + E) = feats @ P + feats[:, :D], so the residual costs nothing in the epilogue. The
// scores take scale = 1 / sqrt(D) (rounded to fp32). One persistent CTA per SM walks
// 128 x 128 output tiles; K runs in 32-deep slices (one 128-byte swizzled row per operand row) through a
// ring of kStages stages, each holding the hi and lo parts of an A and a B slice:
//   warp 0      TMA producer: the raw fp32 slices of A and B into the stage's hi parts;
//   warp 1      TMEM owner and MMA issuer: 12 MMAs per slice (4 k-steps x 3 products); the accumulator is
//               double-buffered in TMEM (2 x 128 columns), so a tile's epilogue overlaps the next tile's
//               products;
//   warps 2-5   the split: hi in place, lo into the stage's lo part at the same offset (the split is
//               elementwise, so the swizzled layout carries over), then a proxy fence and an arrival;
//   warps 6-9   epilogue: TMEM -> registers -> (x scale) -> global memory, each 32 x 32 block
//               transposed through shared memory so that a warp writes 32 consecutive columns of a row.
// Every wait is bounded: on expiry the CTA lets its copies and MMAs finish, frees its TMEM and returns
// (error bit kScoreTimeout).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace veda {
namespace tf32x3 {

constexpr int kBM = 128, kBN = 128, kBK = 32;
constexpr int kPart = kBM * kBK * 4;        // 16 KB: one 128-row slice of one operand part
constexpr int kStages = 3;
constexpr int kStageBytes = 4 * kPart;      // A hi, A lo, B hi, B lo
constexpr int kOffEpi = kStages * kStageBytes;
constexpr int kEpiBytes = 4 * 32 * 33 * 4;  // a 32 x 33 transpose block per epilogue warp
constexpr int kOffBar = kOffEpi + kEpiBytes;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 2 * kBN;
constexpr int kScoreTimeout = 1;               // error bit, as the attend's bounded waits use
constexpr uint64_t kDrainNs = 200000000ull;    // bound of the waits that let issued work finish

struct Bars {
    uint64_t full[kStages];   // TMA -> split (transaction bytes)
    uint64_t split[kStages];  // split (128 arrivals) -> MMA
    uint64_t empty[kStages];  // MMA commit -> producer
    uint64_t acc_full[2];     // MMA commit -> epilogue
    uint64_t acc_empty[2];    // epilogue (128 arrivals) -> MMA
    uint64_t drain;           // MMA commit at the end: every product complete
};
// dynamic shared memory: 1024 bytes of alignment slack, the stages, the epilogue blocks, the barriers,
// the TMEM address and the abort flag
constexpr size_t kSmem = 1024 + size_t(kOffBar) + sizeof(Bars) + 16;

// A [batch][M][K] and B [batch][N][K] fp32 per operand set, boxes of 32 x 128 with the 128-byte swizzle
struct Maps {
    CUtensorMap a[2], b[2];
};

struct Args {
    int n_sets, nb;         // operand sets (1 or 2), batches in each
    int M, N, K;            // K a multiple of kBK
    int tiles_m, tiles_n;   // output tiles per batch
    int n_tiles;            // n_sets * nb * tiles_m * tiles_n
    float* C[2];            // per set: [batch][M][N]
    float scale;            // C = acc * scale
    uint64_t timeout_ns;
    int* err;               // latched error bits
};

// kind::tf32 instruction descriptor: fp32 D (bit 4), tf32 A and B (format code 2), both K-major
__host__ __device__ constexpr uint32_t idesc(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::tf32, issued by one elected lane of a converged warp
__device__ __forceinline__ void mma_ss_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t id,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(id), "r"(accumulate)
        : "memory");
}

// x rounded to the nearest tf32 value (ties away from zero), as an fp32 with the low 13 bits clear
__device__ __forceinline__ float round_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

// makes this thread's generic-proxy shared-memory writes visible to later async-proxy reads (the MMAs)
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void decode(const Args& a, int t, int& set, int& batch, int& m0, int& n0) {
    const int per_batch = a.tiles_m * a.tiles_n;
    const int bt = t / per_batch, r = t - bt * per_batch;
    set = bt / a.nb;
    batch = bt - set * a.nb;
    m0 = (r / a.tiles_n) * kBM;
    n0 = (r % a.tiles_n) * kBN;
}

// dst[b][c][r] = src[b][r][c] + (r == c) for rows x cols matrices (both multiples of 32): the projection
// transposed, with the identity block added; batches blockIdx.z < nb come from src0 / go to dst0, the
// rest from src1 / to dst1
__global__ void __launch_bounds__(256) transpose_kernel(const float* src0, const float* src1, float* dst0,
                                                        float* dst1, int nb, int rows, int cols) {
    __shared__ float t[32][33];
    int bz = blockIdx.z;
    const bool second = bz >= nb;
    if (second) bz -= nb;
    const int64_t off = int64_t(bz) * rows * cols;
    const float* src = (second ? src1 : src0) + off;
    float* dst = (second ? dst1 : dst0) + off;
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
        const int r = r0 + ty + i, c = c0 + tx;
        t[ty + i][tx] = src[int64_t(r) * cols + c] + (r == c ? 1.f : 0.f);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 32; i += 8) dst[int64_t(c0 + ty + i) * rows + r0 + tx] = t[tx][ty + i];
}

__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ Maps maps, const Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars& B = *reinterpret_cast<Bars*>(smem + kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&B + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = a.K / kBK;
    const uint64_t tmo = a.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&B.full[s], 1);
            ptx::mbar_init(&B.split[s], 128);
            ptx::mbar_init(&B.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&B.acc_full[b], 1);
            ptx::mbar_init(&B.acc_empty[b], 128);
        }
        ptx::mbar_init(&B.drain, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < a.n_sets; ++s) {
            ptx::tma_prefetch_desc(&maps.a[s]);
            ptx::tma_prefetch_desc(&maps.b[s]);
        }
    }
    if (warp == 1) ptx::tmem_alloc(tmem_slot, kTmemCols);
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------------------- TMA producer
        const uint64_t keep = ptx::policy_evict_last();  // operand rows are read by several tiles
        int g = 0;  // slices issued (warp-uniform)
        bool stop = false;
        for (int t = blockIdx.x; t < a.n_tiles && !stop; t += gridDim.x) {
            int set, batch, m0, n0;
            decode(a, t, set, batch, m0, n0);
            for (int kk = 0; kk < nk; ++kk) {
                const int s = g % kStages, ph = g / kStages;
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(&B.empty[s], (ph & 1) ^ 1, abort_flag, tmo))) {
                    stop = true;
                    break;
                }
                if (ptx::elect_one()) {
                    uint8_t* st = smem + s * kStageBytes;
                    ptx::mbar_arrive_expect_tx(&B.full[s], 2 * kPart);
                    ptx::tma_load_3d_hint(st, set ? &maps.a[1] : &maps.a[0], kk * kBK, m0, batch, &B.full[s], keep);
                    ptx::tma_load_3d_hint(st + 2 * kPart, set ? &maps.b[1] : &maps.b[0], kk * kBK, n0, batch, &B.full[s],
                                          keep);
                }
                __syncwarp();
                ++g;
            }
        }
        if (*abort_flag && lane == 0) {
            // every copy already issued must land before the CTA releases its shared memory
            volatile int never = 0;
            for (int k = (g > kStages ? g - kStages : 0); k < g; ++k)
                ptx::mbar_wait(&B.full[k % kStages], (k / kStages) & 1, &never, kDrainNs);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------------------- MMA issuer
        constexpr uint32_t kId = idesc(kBM, kBN);
        int g = 0, lt = 0;  // slices and tiles consumed
        for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++lt) {
            const int b = lt & 1;
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(&B.acc_empty[b], ((lt >> 1) & 1) ^ 1, abort_flag, tmo))) break;
            ptx::tc_fence_after();
            const uint32_t d = tmem + uint32_t(b * kBN);
            bool stop = false;
            for (int kk = 0; kk < nk; ++kk) {
                const int s = g % kStages, ph = g / kStages;
                if (!__all_sync(0xffffffffu, ptx::mbar_wait(&B.split[s], ph & 1, abort_flag, tmo))) {
                    stop = true;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t base = ptx::smem_addr(smem + s * kStageBytes);
                const uint64_t ah = ptx::smem_desc_sw128(base, 16, 1024);
                const uint64_t al = ptx::smem_desc_sw128(base + kPart, 16, 1024);
                const uint64_t bh = ptx::smem_desc_sw128(base + 2 * kPart, 16, 1024);
                const uint64_t bl = ptx::smem_desc_sw128(base + 3 * kPart, 16, 1024);
#pragma unroll
                for (int k8 = 0; k8 < kBK / 8; ++k8) {
                    const uint64_t o = uint64_t(k8 * 2);  // 8 tf32 = 32 bytes per k-step, in 16-byte units
                    mma_ss_w(d, al + o, bh + o, kId, (kk > 0 || k8 > 0) ? 1u : 0u);
                    mma_ss_w(d, ah + o, bl + o, kId, 1u);
                    mma_ss_w(d, ah + o, bh + o, kId, 1u);
                }
                ptx::mma_commit_w(&B.empty[s]);
                ++g;
            }
            if (stop) break;
            ptx::mma_commit_w(&B.acc_full[b]);
        }
        // every product issued must be complete before the TMEM is released
        volatile int never = 0;
        ptx::mma_commit_w(&B.drain);
        ptx::mbar_wait(&B.drain, 0, &never, kDrainNs);
    } else if (warp < 6) {
        // ---------------------------------------------------------------------------- split into hi / lo
        const int i = threadIdx.x - 64;
        int g = 0;
        bool stop = false;
        for (int t = blockIdx.x; t < a.n_tiles && !stop; t += gridDim.x) {
            for (int kk = 0; kk < nk; ++kk) {
                const int s = g % kStages, ph = g / kStages;
                if (!ptx::mbar_wait(&B.full[s], ph & 1, abort_flag, tmo)) {
                    stop = true;
                    break;
                }
                uint8_t* st = smem + s * kStageBytes;
#pragma unroll
                for (int op = 0; op < 2; ++op) {
                    float4* hi = reinterpret_cast<float4*>(st + op * 2 * kPart);
                    float4* lo = reinterpret_cast<float4*>(st + op * 2 * kPart + kPart);
#pragma unroll
                    for (int j = 0; j < kPart / 16 / 128; ++j) {
                        const int e = i + 128 * j;
                        const float4 x = hi[e];
                        float4 h, l;
                        h.x = round_tf32(x.x);
                        h.y = round_tf32(x.y);
                        h.z = round_tf32(x.z);
                        h.w = round_tf32(x.w);
                        l.x = x.x - h.x;
                        l.y = x.y - h.y;
                        l.z = x.z - h.z;
                        l.w = x.w - h.w;
                        hi[e] = h;
                        lo[e] = l;
                    }
                }
                fence_async_smem();
                ptx::mbar_arrive(&B.split[s]);
                ++g;
            }
        }
    } else {
        // ---------------------------------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may read: rows 32 q .. 32 q + 31 of a tile
        float* tr = reinterpret_cast<float*>(smem + kOffEpi) + (warp - 6) * 32 * 33;
        int lt = 0;
        for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++lt) {
            const int b = lt & 1;
            if (!ptx::mbar_wait(&B.acc_full[b], (lt >> 1) & 1, abort_flag, tmo)) break;
            ptx::tc_fence_after();
            int set, batch, m0, n0;
            decode(a, t, set, batch, m0, n0);
            // (a select, not a.C[set]: a runtime index into the kernel arguments would copy them to the stack)
            float* C = (set ? a.C[1] : a.C[0]) + int64_t(batch) * a.M * a.N;
            const uint32_t taddr = tmem + (uint32_t(32 * q) << 16) + uint32_t(b * kBN);
#pragma unroll 1
            for (int j = 0; j < kBN / 32; ++j) {
                uint32_t v[32];
                ptx::tmem_ld32(taddr + 32 * j, v);
                ptx::tmem_wait_ld();
                if (j == kBN / 32 - 1) {
                    // the accumulator is read: the next tile's products may overwrite it
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(&B.acc_empty[b]);
                }
#pragma unroll
                for (int e = 0; e < 32; ++e) tr[lane * 33 + e] = __uint_as_float(v[e]);
                __syncwarp();
                const int n = n0 + 32 * j + lane;
#pragma unroll 8
                for (int rr = 0; rr < 32; ++rr) {
                    const int m = m0 + 32 * q + rr;
                    if (m < a.M && n < a.N) C[int64_t(m) * a.N + n] = tr[rr * 33 + lane] * a.scale;
                }
                __syncwarp();
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(a.err, kScoreTimeout);
}

}  // namespace tf32x3
}  // namespace veda
