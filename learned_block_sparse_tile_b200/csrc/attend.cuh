// Block-sparse flash attention over kept 128x128 tiles, sm_100a (tcgen05 + TMA), with the scatter
// back to packed rows fused into the epilogue.
//
// What it computes: veda_core.py (ComfyUI-FunPack), "selection", reference_attend - for query tile i of
// head h, softmax(q k^T * D^-0.5) v over the key slots of the kept tiles that hold a real row (a tile's
// real rows are a prefix, so slot j of tile t is live iff j < valid_count[t]); a row that sees no key
// gives 0. Then "tiles", scatter_: each real query slot goes to its packed row of the output.
//
// Design: one persistent CTA per SM, 640 threads, work items = (head, query tile), one item at a time.
// The item's kept key tiles are split between two softmax groups by parity, each with its own online
// softmax state and its own O accumulator in TMEM; the two partial results are merged at the end of the
// item. While one group computes its softmax the tensor core works on the other group's tiles.
//   warp 0       TMA producer of Q (one buffer) and K (ring); warp 2: TMA producer of V (ring). Every box
//                is 128 rows x 128 bytes with the 128-byte swizzle.
//   warp 1       TMEM owner and MMA issuer: the whole warp runs the issue loop (its waits, descriptors and
//                ring positions are warp-uniform) and elect.sync lets one lane issue each tcgen05 instruction,
//                which keeps the issuer's instruction count low next to the softmax warps sharing its
//                sub-partition. S_j = Q K_j^T (both operands in shared memory) into
//                the S columns of group j%2, then O_(j%2) += P_j V_j with P read from TMEM where the group
//                left it (the "TS" form) and V from shared memory. Issue order per item: S_0, S_1, then per
//                tile PV_j followed by S_(j+2).
//   warps 4-11   softmax group 0 (tiles 0, 2, 4, ...); warps 12-19 group 1 (tiles 1, 3, 5, ...). Each query
//                row (its TMEM lane) has two threads in its group, in warps four apart: one takes key
//                columns 0-63 of each S tile, the other 64-127, so a tile's softmax is split over eight
//                warps. Each masks key slots past the tile's real rows, exponentiates its half against the
//                row's running reference m (O is rescaled only when the max grows by more than 2^8, which
//                bounds P by 256; with the logit bound, an item's later tiles keep the first tile's m), and
//                writes P as bf16 over its own S columns. The two halves of a row exchange partial maxima
//                whenever a tile takes the row max. exp2 runs partly on the MUFU and partly as a polynomial
//                on the FMA pipe. At the end of the item the four threads of a row exchange (max, sum)
//                and each writes a quarter of the output columns:
//                (O_0 2^(m_0 - m) + O_1 2^(m_1 - m)) / sum.
// TMEM columns: S of group 0 [0,128), group 1 [128,256), P of a group over its S columns [0,32) (keys 0-63)
// and [64,96) (keys 64-127); O of group 0 [256, 256 + D), group 1 [384, 384 + D).
// Loads (kDirect): the tile-order variant reads head-major tile copies through 2D maps (tile t of head h
// at rows (h N + 128 t) of [H' N, D]). The gather-free variant reads the packed [S, H, D] tensors: a span
// tile is one 5D box (st, sh, sw, 1, 64) of its span's grid at the tile's origin, a global tile one 3D box
// of 128 consecutive rows; a partial box keeps its padding in place, so its keys are masked by the tile's
// 128-bit position mask instead of by count, and query rows scatter through the box-order row table.
// Every wait is bounded: on expiry the CTA drains its in-flight copies and MMAs, frees its TMEM and
// returns, and the host reads VEDA_ERR_TIMEOUT.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"

namespace veda {

// Of every 8 column pairs of a row, this many take exp2 on the FMA pipe (polynomial) and the rest on the
// MUFU: 128 MUFU exp2 per row would cost 1024 cycles of one SMSP's MUFU per tile, more than the MMAs,
// while each polynomial pair costs about ten issue slots. 2 measured fastest (1, 3, 4 and 5 slower).
constexpr int kPolyPairs = 2;

constexpr int kErrTimeout = 1;
constexpr int kErrBadList = 2;
constexpr int kErrLayout = 8;  // shared memory base not 1024-byte aligned: the kernel did nothing

// Upper bound of the waits that let in-flight copies and MMAs finish before a CTA that gave up exits;
// independent of the (possibly short) wait limit, since those operations complete in microseconds.
constexpr uint64_t kDrainNs = 200000000ull;

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
    int hold_q;  // test hook: the producer withholds every Q load, so every wait on Q expires
    const float* scales_q;  // FP8 variant: [n_heads, n_tiles] per-tile scales of the e4m3 Q and K codes
    const float* scales_k;
    // gather-free variant: per tile its box origin ({span, w0, h0, t0}, or {-1, row0, 0, 0} for a global
    // tile) and the 128-bit mask of box positions that hold one of its rows; perm is then the box-order
    // table (packed row per box position)
    const int4* tile_coord;
    const uint4* tile_mask;
    int32_t n_map_spans;  // span map sets in use (the global set is used when n_global > 0)
    // logit bound (bf16 Q/K; both null: none): ||q||^2 of every packed row and the largest ||k||^2 of each
    // head, so that q . k <= sqrt(||q||^2 max ||k||^2) for every key the row can see (Cauchy-Schwarz)
    const float* q_row_sq;  // [n_heads, seq_len]
    const float* k_max_sq;  // [n_heads]
    int64_t seq_len;
    // redo pass after the paired kernel (attend_pair.cuh): when set, the kernel processes only the items
    // redo_items[0, *redo_count) (device memory, written by the kernel before it) instead of all n_items
    const int32_t* redo_items;
    const int32_t* redo_count;
};

// With the logit bound, a softmax group takes its reference m from the exact row maxima of its first tile
// and keeps it for the rest of the item when every row of the warp has bound - m <= kSkipLimit (log2
// units): every later P = 2^(s - m) then stays below 2^kSkipLimit, so the row max and the rescale of O
// are skipped without any risk of overflow (fp32 and bf16 reach 2^127; O sums at most 2^18 keys of
// P |v|). The result is the same softmax, only the common scale of P, O and the row sum differs.
constexpr float kSkipLimit = 48.f;

// TMA maps of one launch. The tile-ordered variant uses set 0 only (2D maps over [n_heads * N, D]). The
// gather-free variant has one set of 5D maps per tiled span over the packed tensors viewed as
// [T, H, W, heads, D] (box (st, sh, sw, 1, 64)) and a set of 3D maps over [rows, heads, D] for the global
// tiles (box (128, 1, 64)), whose row extent ends after the last global row so that a partial last tile
// reads zeros past its rows.
constexpr int kMapSets = 5;
constexpr int kGlobalMapSet = kMapSets - 1;
struct AttendMaps {
    CUtensorMap q[kMapSets], k[kMapSets], v[kMapSets];
};

// Q/K formats: bf16, or 8-bit codes with per-tile scales: e4m3 (S = Q K^T on the kind::f8f6f4 path) or
// int8 (kind::i8, S in int32). V stays bf16 in every format.
enum QKFormat : int { kQKBf16 = 0, kQKE4M3 = 1, kQKI8 = 2 };

template <int D, int kQK = kQKBf16>
struct AttendCfg {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr bool kFp8 = kQK != kQKBf16;  // Q and K are 8-bit codes (1 byte per element)
    static_assert(!kFp8 || D == 128, "the 8-bit Q/K variants are built for head_dim 128");
    static constexpr int kWarps = 20;  // copy/MMA warpgroup (warps 0-3) + two softmax groups of eight warps
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kQKBytes = 128 * D * (kFp8 ? 1 : 2);  // one Q or K tile
    static constexpr int kTileBytes = 128 * D * 2;             // one V tile (bf16)
    static constexpr int kBoxesQK = kFp8 ? 1 : D / 64;         // 128-byte-wide TMA boxes per Q/K tile
    static constexpr int kBoxes = D / 64;                      // 64-column (128-byte) TMA boxes per V tile
    static constexpr int kKStages = kFp8 ? 4 : (D == 128 ? 2 : 3);  // K ring depth
    static constexpr int kVStages = kFp8 ? 4 : 3;                    // V ring depth
    // header first: barriers; the end-of-item (max, partial sum) of each [group][half][row]; the
    // [parity][group][half][row] partial row maxima the two halves of a row exchange. Then the 1024-aligned
    // tiles (at head_dim 128: 201 KB of the 227 KB a CTA may use)
    static constexpr int kOffBar = 0;
    static constexpr int kOffStats = 512;
    static constexpr int kOffXch = kOffStats + 2 * 2 * 128 * 8;
    static constexpr int kHeader = 9216;
    static_assert(kOffXch + 2 * 2 * 2 * 128 * 4 <= kHeader, "header layout");
    static constexpr int kOffQ = kHeader;
    static constexpr int kOffK = kOffQ + kQKBytes;
    static constexpr int kOffV = kOffK + kKStages * kQKBytes;
    static constexpr int kSmem = kOffV + kVStages * kTileBytes;
    static constexpr uint32_t kTmemCols = 512;  // S/P of group 0, S/P of group 1, O of group 0, O of group 1
    static constexpr uint32_t kIdescS = kQK == kQKI8    ? ptx::idesc_s8_s32(128, 128)
                                        : kQK == kQKE4M3 ? ptx::idesc_e4m3_f32(128, 128)
                                                         : ptx::idesc_bf16_f32(128, 128, false, false);
    static constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, D, false, true);
};

struct AttendBars {
    uint64_t q_full, q_empty;
    uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
    uint64_t s_full[2], p_full[2], o_done[2];
    uint64_t o_empty, merge, drain;
    uint64_t pair[2][4];  // per group and TMEM lane quarter: the two halves' row-max exchange
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

// Items of this launch: all n_items, or the redo list's length. Item i is then i, or redo_items[i].
__device__ __forceinline__ int launch_items(const AttendArgs& a) {
    return a.redo_count != nullptr ? *a.redo_count : a.n_items;
}
__device__ __forceinline__ int item_at(const AttendArgs& a, int i) {
    return a.redo_items != nullptr ? a.redo_items[i] : i;
}

// Item order: the dense global query tiles first (they are the longest), then head-major video tiles,
// so that neighbouring slots work on neighbouring query tiles of one head (shared K/V in L2).
__device__ __forceinline__ void decode_item(const AttendArgs& a, int item, int* hh, int* qt) {
    const int n_glob_items = a.n_heads * a.n_global;
    if (item < n_glob_items) {
        *hh = item / a.n_global;
        *qt = a.n_video + item % a.n_global;
    } else {
        const int v = item - n_glob_items;
        *hh = v / a.n_video;
        *qt = v % a.n_video;
    }
}


// A softmax group index carried as a type, so that code written once for both groups sees it as a constant.
template <int W>
struct GroupId {
    static constexpr int value = W;
};

// Tiles of an item that softmax group w handles: the item-local tiles j = w, w + 2, ...
__device__ __forceinline__ int group_tiles(int n, int w) { return (n - w + 1) >> 1; }

template <int D, int kQK, bool kDirect>
__global__ void __launch_bounds__(640, 1)
    attend_kernel(const __grid_constant__ AttendMaps maps, const AttendArgs a) {
    using C = AttendCfg<D, kQK>;
    constexpr bool kFp8 = C::kFp8;  // 8-bit Q/K codes (either format)
    constexpr int KS = C::kKStages, VS = C::kVStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw;
    const int n_items = launch_items(a);
    if (int(blockIdx.x) >= n_items) return;  // uniform: a redo pass with fewer items than CTAs
    if ((ptx::smem_addr(smem) & 1023) != 0) {  // the swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0) atomicOr(a.err, kErrLayout);
        return;
    }
    AttendBars& B = *reinterpret_cast<AttendBars*>(smem + C::kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&B + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float2* stats = reinterpret_cast<float2*>(smem + C::kOffStats);  // [2 groups][2 halves][128 rows] (max, sum)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&B.q_full, 1);
        ptx::mbar_init(&B.q_empty, 1);
        for (int i = 0; i < KS; ++i) {
            ptx::mbar_init(&B.k_full[i], 1);
            ptx::mbar_init(&B.k_empty[i], 1);
        }
        for (int i = 0; i < VS; ++i) {
            ptx::mbar_init(&B.v_full[i], 1);
            ptx::mbar_init(&B.v_empty[i], 1);
        }
        for (int w = 0; w < 2; ++w) {
            ptx::mbar_init(&B.s_full[w], 1);
            ptx::mbar_init(&B.p_full[w], 256);
            ptx::mbar_init(&B.o_done[w], 1);
            for (int q = 0; q < 4; ++q) ptx::mbar_init(&B.pair[w][q], 64);
        }
        ptx::mbar_init(&B.o_empty, 512);
        ptx::mbar_init(&B.merge, 512);
        ptx::mbar_init(&B.drain, 1);
        *abort_flag = 0;
        ptx::fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        const int sets = kDirect ? a.n_map_spans : 1;
        for (int i = 0; i < kMapSets; ++i) {
            if (i < sets || (kDirect && i == kGlobalMapSet && a.n_global > 0)) {
                ptx::tma_prefetch_desc(&maps.q[i]);
                ptx::tma_prefetch_desc(&maps.k[i]);
                ptx::tma_prefetch_desc(&maps.v[i]);
            }
        }
    }
    if (warp == 1) ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint64_t tmo = a.timeout_ns;

    // registers: the copy/MMA warpgroup (warps 0-3) hands most of its share to the four softmax warpgroups,
    // whose 64-column halves of S then fit. Each role sets its budget at the top of its own branch (the
    // compiler allocates each branch within it); the budgets add up to no more than the 640 x 96 registers
    // the block is launched with, so the increases can always be granted.
    constexpr uint32_t kRegsLow = 56, kRegsHigh = 104;
    static_assert(128 * kRegsLow + 512 * kRegsHigh <= 640 * 96, "register split");
    if (warp == 3) {
        ptx::regs_dec<kRegsLow>();  // idle, but part of the copy/MMA warpgroup
    } else if (warp == 0 || warp == 2) {
        ptx::regs_dec<kRegsLow>();
        // ------------------------------------------------------------- producers: warp 0 Q and K, warp 2 V
        const bool kq = warp == 0;
        const int S = kq ? KS : VS;
        const uint64_t keep = ptx::policy_evict_last();
        int issued_q = 0, issued = 0;  // copies issued so far (warp-uniform): Q tiles; K or V tiles
        for (int i = blockIdx.x; i < n_items; i += gridDim.x) {
            int hh, qt;
            decode_item(a, item_at(a, i), &hh, &qt);
            const int32_t* list;
            bool bad;
            const int n = item_tiles(a, hh, qt, &list, &bad);
            if (kq && bad && lane == 0) atomicOr(a.err, kErrBadList);
            if (n == 0) continue;
            const int32_t row0 = int32_t(int64_t(hh) * a.n_slots);
            const int head = kDirect ? __ldg(a.heads + hh) : 0;  // head index in the packed tensors
            if (kq && !a.hold_q &&
                __all_sync(0xffffffffu, ptx::mbar_wait(&B.q_empty, (issued_q & 1) ^ 1, abort_flag, tmo))) {
                if (ptx::elect_one()) {
                    ptx::mbar_arrive_expect_tx(&B.q_full, C::kQKBytes);
                    if constexpr (kDirect) {
                        const int4 tc = __ldg(a.tile_coord + qt);
                        for (int x = 0; x < C::kBoxes; ++x) {
                            if (tc.x >= 0)
                                ptx::tma_load_5d_hint(smem + C::kOffQ + x * 16384, &maps.q[tc.x], x * 64, head, tc.y,
                                                      tc.z, tc.w, &B.q_full, keep);
                            else
                                ptx::tma_load_3d_hint(smem + C::kOffQ + x * 16384, &maps.q[kGlobalMapSet], x * 64, head,
                                                      tc.y, &B.q_full, keep);
                        }
                    } else {
                        for (int x = 0; x < C::kBoxesQK; ++x)
                            ptx::tma_load_2d(smem + C::kOffQ + x * 16384, &maps.q[0], x * (kFp8 ? 128 : 64),
                                             row0 + qt * 128, &B.q_full);
                    }
                }
                __syncwarp();
                ++issued_q;
            }
            if (__any_sync(0xffffffffu, *abort_flag)) break;
            int mine = 0;
            int4 cmine = make_int4(0, 0, 0, 0);  // gather-free variant: box origin of this lane's tile
            for (int j = 0; j < n; ++j) {
                if ((j & 31) == 0) {
                    mine = (j + lane < n) ? __ldg(list + j + lane) : 0;
                    if constexpr (kDirect) cmine = __ldg(a.tile_coord + mine);
                }
                const int y = row0 + __shfl_sync(0xffffffffu, mine, j & 31) * 128;
                int4 tc = make_int4(0, 0, 0, 0);
                if constexpr (kDirect) {
                    tc.x = __shfl_sync(0xffffffffu, cmine.x, j & 31);
                    tc.y = __shfl_sync(0xffffffffu, cmine.y, j & 31);
                    tc.z = __shfl_sync(0xffffffffu, cmine.z, j & 31);
                    tc.w = __shfl_sync(0xffffffffu, cmine.w, j & 31);
                }
                const int st = issued % S, u = issued / S;
                uint64_t* empty = kq ? &B.k_empty[st] : &B.v_empty[st];
                uint64_t* full = kq ? &B.k_full[st] : &B.v_full[st];
                const int bytes = kq ? C::kQKBytes : C::kTileBytes;
                uint8_t* dst = smem + (kq ? C::kOffK : C::kOffV) + st * bytes;
                if (__all_sync(0xffffffffu, ptx::mbar_wait(empty, (u & 1) ^ 1, abort_flag, tmo))) {
                    if (ptx::elect_one()) {
                        ptx::mbar_arrive_expect_tx(full, bytes);
                        const int boxes = kq ? C::kBoxesQK : C::kBoxes, xstep = (kq && kFp8) ? 128 : 64;
                        for (int x = 0; x < boxes; ++x) {
                            if constexpr (kDirect) {
                                const AttendMaps& m = maps;
                                if (tc.x >= 0)
                                    ptx::tma_load_5d_hint(dst + x * 16384, kq ? &m.k[tc.x] : &m.v[tc.x], x * 64, head,
                                                          tc.y, tc.z, tc.w, full, keep);
                                else
                                    ptx::tma_load_3d_hint(dst + x * 16384, kq ? &m.k[kGlobalMapSet] : &m.v[kGlobalMapSet],
                                                          x * 64, head, tc.y, full, keep);
                            } else {
                                ptx::tma_load_2d_hint(dst + x * 16384, kq ? &maps.k[0] : &maps.v[0], x * xstep, y, full,
                                                      keep);
                            }
                        }
                    }
                    __syncwarp();
                    ++issued;
                }
                if (__any_sync(0xffffffffu, *abort_flag)) break;
            }
            if (__any_sync(0xffffffffu, *abort_flag)) break;
        }
        if (*abort_flag && lane == 0) {
            // every copy already issued must land before the CTA releases its shared memory
            volatile int never = 0;
            for (int k = (issued > S ? issued - S : 0); k < issued; ++k)
                ptx::mbar_wait(kq ? &B.k_full[k % KS] : &B.v_full[k % VS], (k / S) & 1, &never, kDrainNs);
            if (kq && issued_q > 0) ptx::mbar_wait(&B.q_full, (issued_q - 1) & 1, &never, kDrainNs);
        }
    } else if (warp == 1) {
        ptx::regs_dec<kRegsLow>();
        // ------------------------------------------------------------- MMA issuer (whole warp, one lane issues)
        // Per item: S_0 and S_1, then for each tile j: O_(j%2) += P_j V_j, then S_(j+2). S_j lands in S
        // buffer j%2, which softmax group j%2 turns into P_j in place.
        int it = 0;              // items with tiles so far
        int ks = 0, kph = 0;     // K ring slot of the next S and its phase
        int vs = 0, vph = 0;     // V ring slot of the next PV and its phase
        int pu0 = 0, pu1 = 0;    // tiles each group has had so far (barrier phases); scalars, not an
                                 // array indexed by the group, which would live in local memory
        // shared-memory descriptors of the first Q, K and V boxes; a k-step or a ring slot only moves the
        // start address, which is the descriptor's low field (address / 16, below 2^14 for any CTA address)
        const uint64_t dq = ptx::smem_desc_sw128(ptx::smem_addr(smem + C::kOffQ), 16, 1024);
        const uint64_t dk = ptx::smem_desc_sw128(ptx::smem_addr(smem + C::kOffK), 16, 1024);
        const uint64_t dv = ptx::smem_desc_sw128(ptx::smem_addr(smem + C::kOffV), 16384, 1024);
        for (int i = blockIdx.x; i < n_items; i += gridDim.x) {
            int hh, qt;
            decode_item(a, item_at(a, i), &hh, &qt);
            const int32_t* list;
            bool bad;
            const int n = item_tiles(a, hh, qt, &list, &bad);
            if (n == 0) continue;
            {
                // one issue step: PV of tile j - 2 and S of tile j, both of group W = j % 2 (a compile-time
                // constant, so barrier addresses and TMEM columns are immediates)
                auto step = [&](const int j, auto wc) -> bool {
                    constexpr int w = decltype(wc)::value;
                    if (j >= 2) {
                        const int jj = j - 2, idx = (w ? pu1 : pu0) + (jj >> 1);
                        bool ok = ptx::mbar_wait(&B.p_full[w], idx & 1, abort_flag, tmo) &&
                                  ptx::mbar_wait(&B.v_full[vs], vph, abort_flag, tmo) &&
                                  (jj > 0 || ptx::mbar_wait(&B.o_empty, (it & 1) ^ 1, abort_flag, tmo));
                        if (!__all_sync(0xffffffffu, ok)) return false;
                        ptx::tc_fence_after();
                        const uint64_t dvs = dv + uint64_t(vs * (C::kTileBytes >> 4));
                        const uint32_t o = tmem + 256 + 128 * w, p = tmem + 128 * w;
#pragma unroll
                        // P of keys 0-63 sits in the group's columns 0-31, of keys 64-127 in 64-95
                        for (int kk = 0; kk < 8; ++kk)
                            ptx::mma_bf16_ts_w(o, p + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8),
                                               dvs + uint64_t(kk * (2048 >> 4)), C::kIdescPV, (jj >= 2 || kk > 0) ? 1u : 0u);
                        ptx::mma_commit_w(&B.v_empty[vs]);
                        if (jj >= n - 2) ptx::mma_commit_w(&B.o_done[w]);  // the group's last tile of the item
                        if (++vs == VS) vs = 0, vph ^= 1;
                    }
                    if (j < n) {
                        if (!__all_sync(0xffffffffu, ptx::mbar_wait(&B.k_full[ks], kph, abort_flag, tmo))) return false;
                        ptx::tc_fence_after();
                        const uint64_t dks = dk + uint64_t(ks * (C::kQKBytes >> 4));
                        if constexpr (kFp8) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                if constexpr (kQK == kQKI8)
                                    ptx::mma_i8_ss_w(tmem + 128 * w, dq + uint64_t(kk * 2), dks + uint64_t(kk * 2), C::kIdescS,
                                                     kk > 0);
                                else
                                    ptx::mma_f8_ss_w(tmem + 128 * w, dq + uint64_t(kk * 2), dks + uint64_t(kk * 2), C::kIdescS,
                                                     kk > 0);
                            }
                        } else {
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint64_t off = uint64_t((kk >> 2) * (16384 >> 4) + (kk & 3) * 2);
                                ptx::mma_bf16_ss_w(tmem + 128 * w, dq + off, dks + off, C::kIdescS, kk > 0);
                            }
                        }
                        ptx::mma_commit_w(&B.s_full[w]);
                        if (j == n - 1) ptx::mma_commit_w(&B.q_empty);
                        if (++ks == KS) ks = 0, kph ^= 1;
                    }
                    return true;
                };
                bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(&B.q_full, it & 1, abort_flag, tmo));
                for (int j = 0; ok && j < n + 2; j += 2) {
                    ok = step(j, GroupId<0>{});
                    if (ok && j + 1 < n + 2) ok = step(j + 1, GroupId<1>{});
                }
            }
            pu0 += group_tiles(n, 0);
            pu1 += group_tiles(n, 1);
            ++it;
            __syncwarp();
            if (__any_sync(0xffffffffu, *abort_flag)) break;
        }
        {
            // every MMA issued so far must finish before the TMEM is released
            volatile int never = 0;
            ptx::mma_commit_w(&B.drain);
            ptx::mbar_wait(&B.drain, 0, &never, kDrainNs);
        }
    } else if (warp >= 4) {
        ptx::regs_inc<kRegsHigh>();
        // ------------------------------------------------------------- softmax groups (warps 4-11, 12-19)
        // Group w takes the item-local tiles j with j % 2 == w. Each query row (its TMEM lane) is shared by
        // two threads of the group, in warps four apart (the same lane quarter): half 0 takes key columns
        // 0-63 of every S tile, half 1 columns 64-127, and each writes its P (bf16 pairs) over the first 32
        // of its own S columns, so neither overwrites S the other has yet to read. The two halves keep one
        // reference m per row: they exchange partial row maxima (through shared memory and a bounded
        // per-pair barrier) on tiles that take the row max - with the logit bound only an item's first.
        const int sw = warp - 4;
        const int w = sw >> 3;           // group
        const int half = (sw >> 2) & 1;  // key columns [64 half, 64 half + 64) of each S tile
        const int q4 = warp & 3;         // TMEM lane quarter this warp may access
        const int row = q4 * 32 + lane;
        const uint32_t lane_base = uint32_t(q4 * 32) << 16;
        const uint32_t t_s = tmem + lane_base + 128 * w + 64 * half;  // this half's S columns (its P: the first 32)
        const uint32_t t_o = tmem + lane_base + 256 + 128 * w;        // O of this group
        const uint32_t t_o0 = tmem + lane_base + 256;
        float* xch = reinterpret_cast<float*>(smem + C::kOffXch);      // [parity][group][half][row]
        uint64_t* pair_bar = &B.pair[w][q4];
        int xc = 0;  // row-max exchanges so far: the pair barrier's phase and the exchange buffer's parity
        // this thread's partial row max -> the row max of both halves (false: a wait gave up)
        auto pair_max = [&](float pm, float* mx) -> bool {
            float* x = xch + ((xc & 1) * 4 + w * 2) * 128;
            x[half * 128 + row] = pm;
            ptx::mbar_arrive(pair_bar);  // release: the store above is visible once the phase completes
            const bool done = ptx::mbar_wait(pair_bar, xc & 1, abort_flag, tmo);
            ++xc;
            *mx = fmaxf(pm, x[(half ^ 1) * 128 + row]);
            return done;
        };
        int cu = 0;          // tiles this group has had so far (barrier phases)
        int it = 0, t = 0;   // items with tiles so far; tiles so far (K ring positions)
        int od_mine = 0, od_other = 0;  // o_done phases of this group and the other: one per item with a tile
        const bool releaser = (sw & 7) == 0 && lane == 0;  // one thread per group frees K slots
        constexpr int kCols = D / 4;  // output columns each thread writes (four threads per row)
        for (int i = blockIdx.x; i < n_items; i += gridDim.x) {
            int hh, qt;
            decode_item(a, item_at(a, i), &hh, &qt);
            const int32_t* list;
            bool bad;
            const int n = item_tiles(a, hh, qt, &list, &bad);
            const int head = __ldg(a.heads + hh);
            const bool head_ok = head >= 0 && head < a.h_total;
            if (!head_ok && threadIdx.x == 128) atomicOr(a.err, 4);
            const int prow = head_ok ? __ldg(a.perm + int64_t(qt) * 128 + row) : -1;
            // this thread writes output columns [(2 w + half) D / 4, (2 w + half + 1) D / 4) of its row
            const int ocol = (2 * w + half) * kCols;
            __nv_bfloat16* dst = a.out + int64_t(prow < 0 ? 0 : prow) * a.out_s0 +
                                 int64_t(head_ok ? head : 0) * a.out_s1 + ocol;
            if (n == 0) {
                if (prow >= 0) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int c = 0; c < kCols / 8; ++c) reinterpret_cast<uint4*>(dst)[c] = z;
                }
                continue;
            }
            const int nw = group_tiles(n, w);
            // log2-domain bound on every logit of this row (padding slots need none); both halves of a row
            // compute the same value
            float bound = INFINITY;
            if (!kFp8 && a.q_row_sq != nullptr && prow >= 0)
                bound = sqrtf(__ldg(a.q_row_sq + int64_t(hh) * a.seq_len + prow) * __ldg(a.k_max_sq + hh)) *
                        a.scale_log2;
            bool skip = false;  // later tiles of the item keep the first tile's reference (no row max)
            float m_ref = -INFINITY;
            uint64_t lsum = ptx::f2_pack(0.f, 0.f);
            bool ok = true;
            int my_vc = 128;
            int my_tile = 0;  // gather-free variant: the tile id, for its position mask
            float my_sk = 1.f;
            const float sq = kFp8 ? __ldg(a.scales_q + int64_t(hh) * a.n_tiles + qt) : 1.f;
            for (int k = 0; k < nw; ++k) {
                if ((k & 31) == 0) {
                    const int jj = 2 * (k + lane) + w;
                    const int tile = jj < n ? __ldg(list + jj) : -1;
                    my_vc = tile >= 0 ? __ldg(a.valid_count + tile) : 128;
                    if (kDirect) my_tile = tile;
                    if (kFp8) my_sk = tile >= 0 ? __ldg(a.scales_k + int64_t(hh) * a.n_tiles + tile) : 1.f;
                }
                const int vc = __shfl_sync(0xffffffffu, my_vc, k & 31);
                // log2-domain scale of this tile's logits (the FP8 path also undoes both tiles' scales)
                const float sl2 = kFp8 ? a.scale_log2 * (sq * __shfl_sync(0xffffffffu, my_sk, k & 31)) : a.scale_log2;
                const uint64_t sl2x2 = ptx::f2_pack(sl2, sl2);
                const int idx = cu + k;
                ok = ptx::mbar_wait(&B.s_full[w], idx & 1, abort_flag, tmo);
                if (!ok) break;
                ptx::tc_fence_after();
                // S of this tile is complete, so its K slot may be refilled. S of this group's tile was also
                // issued after the PV of the group's previous tile, so that PV is complete as well: O may be
                // rescaled and the P columns rewritten without another wait.
                if (releaser) ptx::mbar_arrive(&B.k_empty[(t + 2 * k + w) % KS]);
                uint32_t s[64];
                ptx::tmem_ld32(t_s, *reinterpret_cast<uint32_t(*)[32]>(s));
                ptx::tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(s + 32));
                ptx::tmem_wait_ld();
                if constexpr (kQK == kQKI8) {
                    // int32 -> fp32, exactly: adding the bit pattern of 1.5 * 2^23 puts |S| < 2^22 in the
                    // low mantissa bits of a float in [2^23, 2^24); subtracting 1.5 * 2^23 is then exact
                    const uint64_t magic = ptx::f2_pack(-12582912.f, -12582912.f);
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        float f0, f1;
                        ptx::f2_unpack(ptx::f2_add(ptx::f2_pack(__uint_as_float(s[c] + 0x4B400000u),
                                                                __uint_as_float(s[c + 1] + 0x4B400000u)), magic), f0, f1);
                        s[c] = __float_as_uint(f0);
                        s[c + 1] = __float_as_uint(f1);
                    }
                }
                if (vc < 128) {
                    if constexpr (kDirect) {
                        // box order: the tile's rows sit where its mask says (padding in place)
                        const uint4 m = __ldg(a.tile_mask + __shfl_sync(0xffffffffu, my_tile, k & 31));
                        const uint32_t mw0 = half ? m.z : m.x, mw1 = half ? m.w : m.y;
#pragma unroll
                        for (int c = 0; c < 64; ++c)
                            if ((((c < 32 ? mw0 : mw1) >> (c & 31)) & 1u) == 0) s[c] = __float_as_uint(-INFINITY);
                    } else {
#pragma unroll
                        for (int c = 0; c < 64; ++c)
                            if (64 * half + c >= vc) s[c] = __float_as_uint(-INFINITY);
                    }
                }
                bool resc = false;
                float alpha = 1.f;
                if (!skip) {
                    // row max: 8 independent chains of 3-input maxima over this half, then both halves
                    float mx8[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) mx8[q] = fmaxf(__uint_as_float(s[q]), __uint_as_float(s[8 + q]));
#pragma unroll
                    for (int c = 16; c < 64; c += 16) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            mx8[q] = ptx::max3(mx8[q], __uint_as_float(s[c + q]), __uint_as_float(s[c + 8 + q]));
                    }
                    const float pmx = ptx::max3(ptx::max3(mx8[0], mx8[1], mx8[2]), ptx::max3(mx8[3], mx8[4], mx8[5]),
                                                fmaxf(mx8[6], mx8[7]));
                    float mx;
                    ok = pair_max(pmx, &mx);
                    if (!ok) break;
                    const float m_new = mx * sl2;
                    resc = m_new > m_ref + 8.0f;
                    if (resc) {
                        alpha = ptx::ex2(m_ref - m_new);
                        lsum = ptx::f2_mul(lsum, ptx::f2_pack(alpha, alpha));
                        m_ref = m_new;
                    }
                    // the same decision in both warps of the pair: bound and m_ref are equal for a row
                    if (k == 0 && a.q_row_sq != nullptr)
                        skip = __all_sync(0xffffffffu, prow < 0 || bound - m_ref <= kSkipLimit);
                }
                const float negm = m_ref == -INFINITY ? 0.f : -m_ref;
                const uint64_t negm2 = ptx::f2_pack(negm, negm);
                // row sums over the bf16 P the PV product reads (eight independent chains)
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const uint64_t x = ptx::f2_fma(ptx::f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sl2x2, negm2);
                    float p0, p1;
                    if (((c >> 1) & 7) < kPolyPairs) {  // this pair on the FMA pipe
                        ptx::f2_unpack(ptx::f2_exp2_poly(x), p0, p1);
                    } else {  // this pair on the MUFU
                        float x0, x1;
                        ptx::f2_unpack(x, x0, x1);
                        p0 = ptx::ex2(x0);
                        p1 = ptx::ex2(x1);
                    }
                    s[c >> 1] = ptx::pack_bf16(p0, p1);
                }
                // the row sum over the bf16 P the PV product reads (eight independent chains); lsum was scaled
                // with O above when the reference moved
                auto add_row_sum = [&]() {
                    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int c = 0; c < 32; ++c) ptx::add_bf16x2(s[c], acc[c & 3], acc[4 + (c & 3)]);
                    lsum = ptx::f2_add(lsum, ptx::f2_add(ptx::f2_add(ptx::f2_pack(acc[0], acc[4]), ptx::f2_pack(acc[1], acc[5])),
                                                         ptx::f2_add(ptx::f2_pack(acc[2], acc[6]), ptx::f2_pack(acc[3], acc[7]))));
                };
                // P (bf16 pairs of this half's 64 keys) over the first 32 of its S columns: the A operand
                // of O += P V reads keys 0-63 from the group's columns 0-31 and keys 64-127 from 64-95
                ptx::tmem_st32(t_s, *reinterpret_cast<uint32_t(*)[32]>(s));
                ptx::tmem_wait_st();
                const bool rescale = k > 0 && __any_sync(0xffffffffu, resc);
                if (rescale) {
                    // a new reference: rescale this half's share of the accumulator's columns before P is
                    // handed over (the row sum is taken first, so P's registers are free here)
                    add_row_sum();
#pragma unroll 1
                    for (int i = 0; i < D / 64; ++i) {
                        uint32_t o[32];
                        const uint32_t ta = t_o + (D / 2) * half + 32 * i;
                        ptx::tmem_ld32(ta, o);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                        ptx::tmem_st32(ta, o);
                    }
                    ptx::tmem_wait_st();
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(&B.p_full[w]);
                if (!rescale) add_row_sum();  // off the path to the PV
            }
            if (!ok) break;
            // both groups' last PVs of this item must be complete before either accumulator is read. This
            // group's own barrier first: it has followed it phase by phase, and once its last PV is done every
            // earlier MMA is too, so the other group's barrier is at most one phase short of its last PV
            // (a parity wait is only meaningful within one phase).
            const int n0 = group_tiles(n, 0), n1 = group_tiles(n, 1);
            const int nmine = w ? n1 : n0, nother = w ? n0 : n1;
            ok = (nmine == 0 || ptx::mbar_wait(&B.o_done[w], od_mine & 1, abort_flag, tmo)) &&
                 (nother == 0 || ptx::mbar_wait(&B.o_done[w ^ 1], od_other & 1, abort_flag, tmo));
            od_mine += nmine > 0;
            od_other += nother > 0;
            cu += nmine;
            t += n;
            if (!ok) break;
            // merge the two groups: each half publishes its group's reference and its part of the row sum
            float l0, l1;
            ptx::f2_unpack(lsum, l0, l1);
            stats[(w * 2 + half) * 128 + row] = make_float2(m_ref, l0 + l1);
            ptx::mbar_arrive(&B.merge);
            ok = ptx::mbar_wait(&B.merge, it & 1, abort_flag, tmo);
            ++it;
            if (!ok) break;
            const float2 g00 = stats[row], g01 = stats[128 + row], g10 = stats[256 + row], g11 = stats[384 + row];
            const float m0 = g00.x, sum0 = g00.y + g01.y, m1 = g10.x, sum1 = g10.y + g11.y;
            const float m = fmaxf(m0, m1);
            const float a0 = sum0 > 0.f ? ptx::ex2(m0 - m) : 0.f;
            const float a1 = sum1 > 0.f ? ptx::ex2(m1 - m) : 0.f;
            const float den = a0 * sum0 + a1 * sum1;
            const float inv = den > 0.f ? 1.f / den : 0.f;
            const float s0 = a0 * inv, s1 = a1 * inv;
            ptx::tc_fence_after();
            // both accumulators' columns of this thread's share are read (and merged into bf16 pairs) before
            // O is released to the next item's first PV; the global stores come after the release
            uint32_t res[kCols / 2];
#pragma unroll
            for (int h16 = 0; h16 < kCols / 16; ++h16) {  // 16 columns at a time (keeps registers for P's loop)
                uint32_t o0[16], o1[16];
                ptx::tmem_ld16(t_o0 + ocol + 16 * h16, o0);
                ptx::tmem_ld16(t_o0 + 128 + ocol + 16 * h16, o1);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    float v[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const float x0 = s0 != 0.f ? __uint_as_float(o0[2 * c + u]) * s0 : 0.f;
                        const float x1 = s1 != 0.f ? __uint_as_float(o1[2 * c + u]) * s1 : 0.f;
                        v[u] = x0 + x1;
                    }
                    res[8 * h16 + c] = ptx::pack_bf16(v[0], v[1]);
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&B.o_empty);
            if (prow >= 0) {
                uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                for (int c = 0; c < kCols / 8; ++c) d4[c] = make_uint4(res[4 * c], res[4 * c + 1], res[4 * c + 2], res[4 * c + 3]);
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
