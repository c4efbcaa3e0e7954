// Block-sparse flash attention over kept 128x128 tiles, sm_100a (tcgen05 + TMA), with the scatter
// back to packed rows fused into the epilogue.
//
// What it computes: veda_core.py (ComfyUI-FunPack), "selection", reference_attend - for query tile i of
// head h, softmax(q k^T * D^-0.5) v over the key slots of the kept tiles that hold a real row (a tile's
// real rows are a prefix, so slot j of tile t is live iff j < valid_count[t]); a row that sees no key
// gives 0. Then "tiles", scatter_: each real query slot goes to its packed row of the output.
//
// Design (one persistent CTA per SM, 192 threads, work items = (head, query tile)):
//   warp 0      TMA producer: Q tile once per item, then K and V tiles of the item's kept list into a
//               ring of STAGES stages (each TMA box is 128 rows x 128 bytes, 128-byte swizzle).
//   warp 1      TMEM allocator and MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM S buffers
//               (128 fp32 columns each), O += P_j V_j into the TMEM O accumulator (D fp32 columns).
//   warps 2-5   softmax: one thread per query row (its TMEM lane). Reads S_j, applies the key-slot mask,
//               keeps a running max (rescaling O only when the max grows by more than 2^8, which keeps
//               every P value below 256), writes P_j as bf16 into swizzled shared memory, and at the end
//               of the item normalises O by the row sum and stores it to the packed output row.
// Every wait is bounded (see ptx::mbar_wait); on expiry the CTA drains its in-flight copies and MMAs,
// frees its TMEM and returns, and the host reads VEDA_ERR_TIMEOUT.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace veda {

constexpr int kErrTimeout = 1;
constexpr int kErrBadList = 2;

struct AttendArgs {
    const int32_t* kept_idx;     // [n_heads, n_video, max_kept]
    const int32_t* kept_cnt;     // [n_heads, n_video]
    const int32_t* ok_list;      // [n_ok] non-empty tiles (the dense list of a global query tile)
    const int32_t* valid_count;  // [n_tiles]
    const int32_t* perm;         // [n_slots]
    const int32_t* heads;        // [n_heads]
    __nv_bfloat16* out;          // [S, H_total, D] strided
    int64_t out_s0, out_s1;
    int64_t n_slots;
    int32_t max_kept, n_ok, n_tiles, n_video, n_global, n_heads, h_total;
    int32_t n_items;
    float scale_log2;  // D^-0.5 * log2(e)
    uint64_t timeout_ns;
    int* err;
};

template <int D>
struct AttendCfg {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr int kThreads = 192;
    static constexpr int kTileBytes = 128 * D * 2;     // one Q, K or V tile (bf16)
    static constexpr int kBoxes = D / 64;              // 64-column TMA boxes per tile
    static constexpr int kPBytes = 128 * 128 * 2;      // P tile (bf16)
    static constexpr int kStages = D == 128 ? 2 : 4;   // K/V ring depth
    static constexpr int kOffQ = 0;
    static constexpr int kOffP = kOffQ + kTileBytes;
    static constexpr int kOffKV = kOffP + kPBytes;     // stage s: K at kOffKV + 2s*tile, V right after
    static constexpr int kOffBar = kOffKV + kStages * 2 * kTileBytes;
    static constexpr int kBarBytes = 512;
    static constexpr int kSmem = kOffBar + kBarBytes + 1024;  // + slack to align the base to 1024
    static constexpr uint32_t kTmemCols = 512;         // S0 [0,128) S1 [128,256) O [256, 256 + D)
    static constexpr uint32_t kColO = 256;
    static constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 128, false, false);
    static constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, D, false, true);
};

// Number of kept tiles of an item and its list. Warp-collective (all 32 lanes, same result in each).
// A video query tile's list is checked: count within [0, max_kept], ids in [0, n_tiles) and strictly
// ascending; the list is cut before the first bad entry and *bad is set.
__device__ __forceinline__ int item_tiles(const AttendArgs& a, int hh, int qt, const int32_t** list, bool* bad) {
    const int lane = threadIdx.x & 31;
    if (qt >= a.n_video) {
        *list = a.ok_list;
        *bad = false;
        return a.n_ok;
    }
    const int64_t rowid = int64_t(hh) * a.n_video + qt;
    const int32_t* l = a.kept_idx + rowid * a.max_kept;
    *list = l;
    int cnt = __ldg(a.kept_cnt + rowid);
    bool b = false;
    if (cnt < 0 || cnt > a.max_kept) {
        b = true;
        cnt = cnt < 0 ? 0 : a.max_kept;
    }
    int n = cnt, prev_last = -1;
    for (int base = 0; base < cnt; base += 32) {
        const int j = base + lane;
        const int v = j < cnt ? __ldg(l + j) : 0x7fffffff;
        int prev = __shfl_up_sync(0xffffffffu, v, 1);
        if (lane == 0) prev = prev_last;
        const bool ok = j >= cnt || (v >= 0 && v < a.n_tiles && v > prev);
        const unsigned badmask = __ballot_sync(0xffffffffu, !ok);
        if (badmask) {
            n = base + __ffs(badmask) - 1;
            b = true;
            break;
        }
        prev_last = __shfl_sync(0xffffffffu, v, 31);
    }
    *bad = b;
    return n;
}

__device__ __forceinline__ void decode_item(const AttendArgs& a, int item, int* hh, int* qt) {
    const int n_glob_items = a.n_heads * a.n_global;  // dense global rows first: they are the longest
    if (item < n_glob_items) {
        *hh = item / a.n_global;
        *qt = a.n_video + item % a.n_global;
    } else {
        const int v = item - n_glob_items;
        *hh = v / a.n_video;
        *qt = v % a.n_video;
    }
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const AttendArgs a) {
    using C = AttendCfg<D>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* q_full = bars + 0;
    uint64_t* q_empty = bars + 1;
    uint64_t* k_full = bars + 2;
    uint64_t* v_full = k_full + S;
    uint64_t* kv_empty = v_full + S;
    uint64_t* s_full = kv_empty + S;   // [2]
    uint64_t* s_empty = s_full + 2;    // [2]
    uint64_t* p_full = s_empty + 2;
    uint64_t* o_done = p_full + 1;
    uint64_t* o_empty = o_done + 1;
    uint64_t* drain = o_empty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* kvalid = const_cast<int*>(abort_flag) + 1;  // [S]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        ptx::mbar_init(q_full, 1);
        ptx::mbar_init(q_empty, 1);
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(k_full + s, 1);
            ptx::mbar_init(v_full + s, 1);
            ptx::mbar_init(kv_empty + s, 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(s_full + b, 1);
            ptx::mbar_init(s_empty + b, 128);
        }
        ptx::mbar_init(p_full, 128);
        ptx::mbar_init(o_done, 1);
        ptx::mbar_init(o_empty, 128);
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::tma_prefetch_desc(&tm_q);
        ptx::tma_prefetch_desc(&tm_k);
        ptx::tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t tmo = a.timeout_ns;

    const uint32_t sm_q = ptx::smem_addr(smem + C::kOffQ);
    const uint32_t sm_p = ptx::smem_addr(smem + C::kOffP);
    const uint32_t sm_kv = ptx::smem_addr(smem + C::kOffKV);

    if (warp == 0) {
        // ------------------------------------------------------------------------------ producer
        int g = 0, it_local = 0;
        int last_use[S];
        for (int s = 0; s < S; ++s) last_use[s] = -1;
        int last_q = -1;
        const uint64_t keep = ptx::policy_evict_last();
        for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
            int hh, qt;
            decode_item(a, item, &hh, &qt);
            const int32_t* list;
            bool bad;
            const int n = item_tiles(a, hh, qt, &list, &bad);
            if (bad && lane == 0) atomicOr(a.err, kErrBadList);
            if (n == 0) continue;
            const int32_t row0 = int32_t(int64_t(hh) * a.n_slots);
            if (lane == 0) {
                if (ptx::mbar_wait(q_empty, (it_local & 1) ^ 1, abort_flag, tmo)) {
                    ptx::mbar_arrive_expect_tx(q_full, C::kTileBytes);
                    for (int b = 0; b < C::kBoxes; ++b)
                        ptx::tma_load_2d(smem + C::kOffQ + b * 16384, &tm_q, b * 64, row0 + qt * 128, q_full);
                    last_q = it_local;
                }
            }
            ++it_local;
            __syncwarp();
            if (*abort_flag) break;
            int mine = 0;
            for (int j = 0; j < n; ++j, ++g) {
                if ((j & 31) == 0) mine = (j + lane < n) ? __ldg(list + j + lane) : 0;
                const int tile = __shfl_sync(0xffffffffu, mine, j & 31);
                if (lane == 0) {
                    const int st = g % S, u = g / S;
                    if (ptx::mbar_wait(kv_empty + st, (u & 1) ^ 1, abort_flag, tmo)) {
                        kvalid[st] = __ldg(a.valid_count + tile);
                        uint8_t* kd = smem + C::kOffKV + st * 2 * C::kTileBytes;
                        ptx::mbar_arrive_expect_tx(k_full + st, C::kTileBytes);
                        for (int b = 0; b < C::kBoxes; ++b)
                            ptx::tma_load_2d_hint(kd + b * 16384, &tm_k, b * 64, row0 + tile * 128, k_full + st, keep);
                        ptx::mbar_arrive_expect_tx(v_full + st, C::kTileBytes);
                        for (int b = 0; b < C::kBoxes; ++b)
                            ptx::tma_load_2d_hint(kd + C::kTileBytes + b * 16384, &tm_v, b * 64, row0 + tile * 128,
                                                  v_full + st, keep);
                        last_use[st] = u;
                    }
                }
                __syncwarp();
                if (*abort_flag) break;
            }
            if (*abort_flag) break;
        }
        if (*abort_flag && lane == 0) {
            // let every copy already issued land before the CTA releases its shared memory
            volatile int never = 0;
            for (int s = 0; s < S; ++s)
                if (last_use[s] >= 0) {
                    ptx::mbar_wait(k_full + s, last_use[s] & 1, &never, tmo);
                    ptx::mbar_wait(v_full + s, last_use[s] & 1, &never, tmo);
                }
            if (last_q >= 0) ptx::mbar_wait(q_full, last_q & 1, &never, tmo);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------------------ MMA issuer
        int g = 0, sc = 0, pc = 0, it_local = 0, o_uses = 0;
        for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
            int hh, qt;
            decode_item(a, item, &hh, &qt);
            const int32_t* list;
            bool bad;
            const int n = item_tiles(a, hh, qt, &list, &bad);
            if (n == 0) continue;
            if (lane == 0) {
                bool ok = ptx::mbar_wait(q_full, it_local & 1, abort_flag, tmo);
                ptx::tc_fence_after();
                for (int j = 0; ok && j <= n; ++j) {
                    if (j < n) {
                        const int st = (g + j) % S, u = (g + j) / S, b = sc & 1;
                        ok = ptx::mbar_wait(k_full + st, u & 1, abort_flag, tmo) &&
                             ptx::mbar_wait(s_empty + b, ((sc >> 1) & 1) ^ 1, abort_flag, tmo);
                        if (!ok) break;
                        ptx::tc_fence_after();
                        const uint32_t kbase = sm_kv + st * 2 * C::kTileBytes;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                            ptx::mma_bf16_ss(tmem + b * 128, ptx::smem_desc_sw128(sm_q + off, 16, 1024),
                                             ptx::smem_desc_sw128(kbase + off, 16, 1024), C::kIdescS, kk > 0);
                        }
                        ptx::mma_commit(s_full + b);
                        ++sc;
                        if (j == n - 1) ptx::mma_commit(q_empty);
                    }
                    if (j >= 1) {
                        const int jj = j - 1, st = (g + jj) % S, u = (g + jj) / S;
                        ok = ptx::mbar_wait(v_full + st, u & 1, abort_flag, tmo) &&
                             ptx::mbar_wait(p_full, pc & 1, abort_flag, tmo);
                        if (ok && jj == 0) {
                            ok = ptx::mbar_wait(o_empty, (o_uses & 1) ^ 1, abort_flag, tmo);
                            ++o_uses;
                        }
                        if (!ok) break;
                        ptx::tc_fence_after();
                        const uint32_t vbase = sm_kv + st * 2 * C::kTileBytes + C::kTileBytes;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t poff = (kk >> 2) * 16384 + (kk & 3) * 32;
                            ptx::mma_bf16_ss(tmem + C::kColO, ptx::smem_desc_sw128(sm_p + poff, 16, 1024),
                                             ptx::smem_desc_sw128(vbase + kk * 2048, 16384, 1024), C::kIdescPV,
                                             (jj > 0 || kk > 0) ? 1u : 0u);
                        }
                        ptx::mma_commit(o_done);
                        ptx::mma_commit(kv_empty + st);
                        ++pc;
                    }
                }
            }
            g += n;
            ++it_local;
            __syncwarp();
            if (*abort_flag) break;
        }
        if (lane == 0) {
            // every MMA issued so far must finish before the TMEM is released
            volatile int never = 0;
            ptx::mma_commit(drain);
            ptx::mbar_wait(drain, 0, &never, tmo);
        }
    } else {
        // ------------------------------------------------------------------------------ softmax
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const uint32_t lane_base = uint32_t(q4 * 32) << 16;
        const float sl2 = a.scale_log2;
        int g = 0, sc = 0, pc = 0;
        for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
            int hh, qt;
            decode_item(a, item, &hh, &qt);
            const int32_t* list;
            bool bad;
            const int n = item_tiles(a, hh, qt, &list, &bad);
            const int head = __ldg(a.heads + hh);
            const bool head_ok = head >= 0 && head < a.h_total;
            if (!head_ok && threadIdx.x == 64) atomicOr(a.err, 4);
            const int prow = head_ok ? __ldg(a.perm + int64_t(qt) * 128 + row) : -1;
            __nv_bfloat16* dst = a.out + int64_t(prow < 0 ? 0 : prow) * a.out_s0 + int64_t(head_ok ? head : 0) * a.out_s1;
            if (n == 0) {
                if (prow >= 0) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(dst)[c] = z;
                }
                continue;
            }
            float m_ref = -INFINITY, l = 0.f;
            bool ok = true;
            for (int j = 0; j < n; ++j) {
                const int b = sc & 1;
                ok = ptx::mbar_wait(s_full + b, (sc >> 1) & 1, abort_flag, tmo);
                if (!ok) break;
                ptx::tc_fence_after();
                uint32_t s[128];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(s + 32 * i);
                    ptx::tmem_ld32(tmem + lane_base + b * 128 + 32 * i, chunk);
                }
                ptx::tmem_wait_ld();
                ptx::tc_fence_before();
                ptx::mbar_arrive(s_empty + b);
                ++sc;
                const int st = (g + j) % S, u = (g + j) / S;
                ok = ptx::mbar_wait(k_full + st, u & 1, abort_flag, tmo);  // already complete: orders kvalid
                if (!ok) break;
                const int vc = kvalid[st];
                float mx = -INFINITY;
                if (vc >= 128) {
#pragma unroll
                    for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(s[c]));
                } else {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c < vc) mx = fmaxf(mx, __uint_as_float(s[c]));
                }
                const float m_new = mx * sl2;
                const bool resc = m_new > m_ref + 8.0f;
                float alpha = 1.f;
                if (resc) {
                    alpha = ptx::ex2(m_ref - m_new);
                    l *= alpha;
                    m_ref = m_new;
                }
                const float neg = -m_ref;
                float rs = 0.f;
#pragma unroll
                for (int c = 0; c < 128; c += 2) {
                    float p0 = ptx::ex2(fmaf(__uint_as_float(s[c]), sl2, neg));
                    float p1 = ptx::ex2(fmaf(__uint_as_float(s[c + 1]), sl2, neg));
                    if (vc < 128) {
                        p0 = c < vc ? p0 : 0.f;
                        p1 = c + 1 < vc ? p1 : 0.f;
                    }
                    rs += p0 + p1;
                    s[c >> 1] = ptx::pack_bf16(p0, p1);
                }
                l += rs;
                if (j > 0) {
                    ok = ptx::mbar_wait(o_done, pc & 1, abort_flag, tmo);
                    ++pc;
                    if (!ok) break;
                    ptx::tc_fence_after();
                    if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
                        for (int i = 0; i < D / 32; ++i) {
                            uint32_t o[32];
                            ptx::tmem_ld32(tmem + lane_base + C::kColO + 32 * i, o);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                            ptx::tmem_st32(tmem + lane_base + C::kColO + 32 * i, o);
                        }
                        ptx::tmem_wait_st();
                    }
                }
                // P row -> two 64-key swizzle atoms (128 rows x 128 bytes each), K-major
                const uint32_t rbase = sm_p + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
                for (int c16 = 0; c16 < 16; ++c16) {
                    const uint32_t addr = rbase + (c16 >> 3) * 16384 + (((c16 & 7) ^ (row & 7)) << 4);
                    ptx::st_shared_v4(addr, s[c16 * 4 + 0], s[c16 * 4 + 1], s[c16 * 4 + 2], s[c16 * 4 + 3]);
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                ptx::mbar_arrive(p_full);
            }
            g += n;
            if (!ok) break;
            // epilogue: O / l -> bf16 -> packed output row
            ok = ptx::mbar_wait(o_done, pc & 1, abort_flag, tmo);
            ++pc;
            if (!ok) break;
            ptx::tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int i = 0; i < D / 32; ++i) {
                uint32_t o[32];
                ptx::tmem_ld32(tmem + lane_base + C::kColO + 32 * i, o);
                ptx::tmem_wait_ld();
                if (i == D / 32 - 1) {
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(o_empty);
                }
                if (prow >= 0) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * i);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint4 w;
                        w.x = ptx::pack_bf16(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
                        w.y = ptx::pack_bf16(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
                        w.z = ptx::pack_bf16(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
                        w.w = ptx::pack_bf16(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
                        d4[c] = w;
                    }
                }
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, C::kTmemCols);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(a.err, kErrTimeout);
}

}  // namespace veda
