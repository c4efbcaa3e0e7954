// Block-sparse flash attention over kept 128x128 tiles for two neighbouring query tiles at once, sm_100a
// (tcgen05 + TMA), with the logit bound; Q/K in bf16 or as 8-bit codes with per-tile scales (e4m3 or int8,
// as attend.cuh's 8-bit variants: S = Q K^T on the kind::f8f6f4 / kind::i8 path, times both tiles' scales),
// V in bf16. Same operation as attend.cuh (veda_core.py
// (ComfyUI-FunPack), "selection", reference_attend, then "tiles", scatter_): for query tile i of head h,
// softmax(q k^T * D^-0.5) v over the real key slots of its kept tiles, 0 for a row that sees no key.
//
// Why pairs: the kept lists of query tiles 2i and 2i+1 share most of their tiles (neighbouring tiles of
// the video grid rank the same key tiles highly), so one CTA takes both and loads every K/V tile of the
// union once. Work units are the (key tile, query tile) pairs of the union in key-tile order, a tile in
// both lists giving two consecutive units; each K/V tile then crosses L2 once for up to two S and PV
// products, which cuts the L2-to-SM traffic that bounds the single-tile kernel.
//
// Fixed reference: with ||q||^2 per row and the head's largest ||k||^2 (veda_pool), every logit of a row
// is at most bound = sqrt(||q||^2 max ||k||^2) D^-0.5 log2(e) (Cauchy-Schwarz), so each row takes
// m = bound - kBoundOffset for the whole item: P = 2^(s - m) stays at most 2^kBoundOffset, no row max is
// taken and O is never rescaled. That lets both softmax groups add into one O per query tile (the
// single-tile kernel keeps one O per group and merges them). The result is the same softmax; only when
// the bound is loose by more than kBoundOffset + 60 (log2 units) would the row's largest P drop below
// 2^-60 - the row sum tells - and the query tile is then listed for a redo by the single-tile kernel's
// exact path (attend_kernel over AttendArgs::redo_items), which rewrites all of its rows.
//
// Roles (640 threads, one persistent CTA per SM, one pair item at a time):
//   warp 0       TMA producer of the two Q tiles (one buffer pair) and the union's K tiles (ring);
//   warp 2       TMA producer of the union's V tiles (ring);
//   warp 1       TMEM owner and MMA issuer (whole warp, elect.sync issues): unit u's S = Q_x K_t^T into the
//                S columns of group u % 2, then O_x += P_u V_t; issue order S_0, S_1, then per unit PV_u
//                followed by S_(u+2). A K slot is released by a commit after the last S of its tile, a V
//                slot after the last PV.
//   warps 4-19   two softmax groups of eight warps (units 0, 2, 4, ... and 1, 3, 5, ...), two threads per
//                TMEM lane (key columns 0-63 and 64-127 of S), as in attend.cuh; each thread keeps the
//                row sums of both query tiles. At the end of the item the four threads of a row add up
//                the sums (before the item's last PVs complete), group 0 writes query tile A and group 1
//                query tile B, each thread half of the row's columns.
// TMEM columns: S/P of group 0 [0,128), group 1 [128,256); O of query tile A [256, 256 + D), B [384, 384 + D).
// Every wait is bounded (as in attend.cuh): on expiry the CTA drains, frees its TMEM and returns.
#pragma once

#include "attend.cuh"

namespace veda {

// m = bound - kBoundOffset: P <= 2^64 and a row sum of at most 2^20 keys <= 2^84, far from fp32's 2^128
constexpr float kBoundOffset = 64.f;
// a row sum outside [2^-60, 2^100] (or NaN) flags its query tile for the exact redo
constexpr float kRedoBelow = 8.673617379884035e-19f;
constexpr float kRedoAbove = 1.2676506002282294e30f;

// ------------------------------------------------------------------------------------------------ units
// A unit is one int32: key tile << 3 | last << 2 | first << 1 | x, where x is the query tile (0: A, 1: B),
// first marks the first unit of its key tile (its K/V are loaded for it) and last the last one (its K/V
// slots are released after it).
struct PairUnitsArgs {
    const int32_t* kept_idx;  // [n_heads, n_video, max_kept]
    const int32_t* kept_cnt;  // [n_heads, n_video]
    int32_t n_video, max_kept, n_tiles, n_heads, n_pairs;
    int32_t* units;  // [n_heads, n_pairs, 2 * max_kept]
    int2* counts;    // [n_heads, n_pairs]: (units, units of query tile A)
    int* err;
};

// Length of the valid prefix of a kept list: count within [0, max_kept], ids in [0, n_tiles), strictly
// ascending; *bad when anything was cut. The valid entries are copied to dst. Warp-collective.
__device__ __forceinline__ int load_checked_list(const int32_t* l, int cnt, int max_kept, int n_tiles, bool* bad,
                                                 int32_t* dst) {
    const int lane = threadIdx.x & 31;
    bool b = false;
    if (cnt < 0 || cnt > max_kept) {
        b = true;
        cnt = cnt < 0 ? 0 : max_kept;
    }
    int n = cnt, prev_last = -1;
    for (int base = 0; base < cnt; base += 32) {
        const int j = base + lane;
        const int v = j < cnt ? __ldg(l + j) : 0x7fffffff;
        int prev = __shfl_up_sync(0xffffffffu, v, 1);
        if (lane == 0) prev = prev_last;
        const bool ok = j >= cnt || (v >= 0 && v < n_tiles && v > prev);
        const unsigned badmask = __ballot_sync(0xffffffffu, !ok);
        if (badmask) {
            n = base + __ffs(badmask) - 1;
            if (j < n) dst[j] = v;
            b = true;
            break;
        }
        if (j < cnt) dst[j] = v;
        prev_last = __shfl_sync(0xffffffffu, v, 31);
    }
    *bad = b;
    return n;
}

// Entries of the ascending list l[0, n) that are below v.
__device__ __forceinline__ int count_below(const int32_t* l, int n, int v) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (l[mid] < v)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

// One warp per (head, pair of video query tiles 2p, 2p + 1): the checked lists of both rows, staged in
// the warp's slice of shared memory (2 max_kept entries), merged into units. Unit (t, A) lands at
// (entries of A below t) + (entries of B below t), unit (t, B) at (entries of A up to t) + (entries of B
// below t), so a tile in both lists gives (t, A), (t, B) next to each other.
__global__ void __launch_bounds__(256) pair_units_kernel(const PairUnitsArgs a) {
    extern __shared__ int32_t staged[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t gw = int64_t(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (gw >= int64_t(a.n_heads) * a.n_pairs) return;  // whole warps
    const int hh = int(gw / a.n_pairs), p = int(gw % a.n_pairs);
    const int64_t row_a = int64_t(hh) * a.n_video + 2 * p;
    const bool has_b = 2 * p + 1 < a.n_video;
    int32_t* sa = staged + int64_t(warp) * 2 * a.max_kept;
    int32_t* sb = sa + a.max_kept;
    const int32_t* la = a.kept_idx + row_a * a.max_kept;
    bool bad_a = false, bad_b = false;
    const int na = load_checked_list(la, __ldg(a.kept_cnt + row_a), a.max_kept, a.n_tiles, &bad_a, sa);
    const int nb = has_b ? load_checked_list(la + a.max_kept, __ldg(a.kept_cnt + row_a + 1), a.max_kept, a.n_tiles,
                                             &bad_b, sb)
                         : 0;
    if ((bad_a || bad_b) && lane == 0) atomicOr(a.err, kErrBadList);
    __syncwarp();
    int32_t* out = a.units + gw * (2 * int64_t(a.max_kept));
    for (int i = lane; i < na; i += 32) {
        const int t = sa[i];
        const int below = count_below(sb, nb, t);
        const bool both = below < nb && sb[below] == t;
        out[i + below] = (t << 3) | (both ? 0 : 4) | 2;
    }
    for (int j = lane; j < nb; j += 32) {
        const int t = sb[j];
        const int upto = count_below(sa, na, t + 1);
        const bool both = upto > 0 && sa[upto - 1] == t;
        out[upto + j] = (t << 3) | 4 | (both ? 0 : 2) | 1;
    }
    if (lane == 0) a.counts[gw] = make_int2(na + nb, na);
}

// ------------------------------------------------------------------------------------------------ kernel
struct PairArgs {
    const int32_t* units;        // from pair_units_kernel
    const int2* counts;
    const int32_t* ok_list;      // [n_ok] non-empty tiles (the list of every global query tile)
    const int32_t* valid_count;  // [n_tiles]
    const int32_t* perm;         // [n_slots] packed row per slot (box order in the gather-free variant)
    const int32_t* heads;        // [n_heads]
    __nv_bfloat16* out;          // [S, H_total, D] strided
    int64_t out_s0, out_s1;
    int64_t n_slots;
    int32_t max_kept, n_ok, n_tiles, n_video, n_global, n_heads, h_total;
    int32_t n_pairs, n_gpairs;  // pairs of video / global query tiles per head
    int32_t n_items;            // n_heads * (n_gpairs + n_pairs): global pairs first, then video pairs
    float scale_log2;           // D^-0.5 * log2(e)
    uint64_t timeout_ns;
    int* err;
    int hold_q;  // test hook: the producer withholds every Q load, so every wait on Q expires
    const int4* tile_coord;  // gather-free variant, as in AttendArgs
    const uint4* tile_mask;
    int32_t n_map_spans;
    const float* scales_q;  // 8-bit variants: [n_heads, n_tiles] per-tile scales of the Q and K codes
    const float* scales_k;
    const float* q_row_sq;  // [n_heads, seq_len]
    const float* k_max_sq;  // [n_heads]
    int64_t seq_len;
    // query tiles that need the exact redo: a flag per (head index, tile) (zero on entry) and the list of
    // their single-tile item numbers (attend.cuh's order) with its length (zero on entry)
    int32_t* redo_flags;  // [n_heads, n_tiles]
    int32_t* redo_items;  // [n_heads * n_tiles]
    int32_t* redo_count;
};

struct PairItem {
    int hh, qa, qb;  // head index, query tiles A and B (qb = -1: A alone)
    int64_t pair;    // video pair index into units/counts (-1: a global pair)
};

__device__ __forceinline__ PairItem decode_pair(const PairArgs& a, int item) {
    PairItem it;
    const int n_glob = a.n_heads * a.n_gpairs;
    if (item < n_glob) {
        it.hh = item / a.n_gpairs;
        const int p = item % a.n_gpairs;
        it.qa = a.n_video + 2 * p;
        it.qb = 2 * p + 1 < a.n_global ? it.qa + 1 : -1;
        it.pair = -1;
    } else {
        const int v = item - n_glob;
        it.hh = v / a.n_pairs;
        const int p = v % a.n_pairs;
        it.qa = 2 * p;
        it.qb = 2 * p + 1 < a.n_video ? 2 * p + 1 : -1;
        it.pair = int64_t(it.hh) * a.n_pairs + p;
    }
    return it;
}

// Units of an item; *n_a of them belong to query tile A.
__device__ __forceinline__ int item_units(const PairArgs& a, const PairItem& it, int* n_a) {
    if (it.pair < 0) {
        *n_a = a.n_ok;
        return it.qb >= 0 ? 2 * a.n_ok : a.n_ok;
    }
    const int2 c = a.counts[it.pair];
    *n_a = c.y;
    return c.x;
}

// Unit j (< the item's unit count). Global query tiles all see the dense list.
__device__ __forceinline__ int32_t item_unit(const PairArgs& a, const PairItem& it, int j) {
    if (it.pair < 0) {
        if (it.qb < 0) return (__ldg(a.ok_list + j) << 3) | 6;
        return (__ldg(a.ok_list + (j >> 1)) << 3) | ((j & 1) ? 5 : 2);
    }
    return a.units[it.pair * (2 * int64_t(a.max_kept)) + j];
}

template <int D, int kQK = kQKBf16>
struct PairCfg {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr bool kFp8 = kQK != kQKBf16;  // Q and K are 8-bit codes with per-tile scales
    static_assert(!kFp8 || D == 128, "the 8-bit Q/K variants are built for head_dim 128");
    static constexpr int kWarps = 20;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kQKBytes = 128 * D * (kFp8 ? 1 : 2);  // one Q or K tile
    static constexpr int kTileBytes = 128 * D * 2;             // one V tile (bf16)
    static constexpr int kBoxesQK = kFp8 ? 1 : D / 64;         // 128-byte-wide TMA boxes per Q or K tile
    static constexpr int kBoxes = D / 64;                      // 128-byte-wide TMA boxes per V tile
    static constexpr int kKStages = kFp8 ? 4 : (D == 128 ? 2 : 4);
    static constexpr int kVStages = kFp8 ? 3 : (D == 128 ? 2 : 4);
    // header: barriers, then the end-of-item (sum A, sum B) of each [item parity][group][half][row]; then
    // the 1024-aligned tiles (201 KB of the 227 KB a CTA may use at head_dim 128, either format)
    static constexpr int kOffBar = 0;
    static constexpr int kOffStats = 512;
    static constexpr int kHeader = 9216;
    static_assert(kOffStats + 2 * 2 * 2 * 128 * 8 <= kHeader, "header layout");
    static constexpr int kOffQ = kHeader;  // Q of tile A, then of tile B
    static constexpr int kOffK = kOffQ + 2 * kQKBytes;
    static constexpr int kOffV = kOffK + kKStages * kQKBytes;
    static constexpr int kSmem = kOffV + kVStages * kTileBytes;
    static_assert(kSmem <= 227 * 1024, "shared memory");
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kIdescS = kQK == kQKI8    ? ptx::idesc_s8_s32(128, 128)
                                        : kQK == kQKE4M3 ? ptx::idesc_e4m3_f32(128, 128)
                                                         : ptx::idesc_bf16_f32(128, 128, false, false);
    static constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(128, D, false, true);
};

struct PairBars {
    uint64_t q_full, q_empty;
    uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
    uint64_t s_full[2], p_full[2];
    uint64_t o_done, o_empty, merge, drain;
};

template <int D, int kQK, bool kDirect>
__global__ void __launch_bounds__(640, 1)
    attend_pair_kernel(const __grid_constant__ AttendMaps maps, const PairArgs a) {
    using C = PairCfg<D, kQK>;
    constexpr bool kFp8 = C::kFp8;
    static_assert(!(kFp8 && kDirect), "the 8-bit Q/K codes are tile-ordered copies");
    constexpr int KS = C::kKStages, VS = C::kVStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw;
    if ((ptx::smem_addr(smem) & 1023) != 0) {
        if (threadIdx.x == 0) atomicOr(a.err, kErrLayout);
        return;
    }
    PairBars& B = *reinterpret_cast<PairBars*>(smem + C::kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&B + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float2* stats = reinterpret_cast<float2*>(smem + C::kOffStats);  // [item parity][2 groups][2 halves][128 rows]

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
        }
        ptx::mbar_init(&B.o_done, 1);
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

    // register split as in attend.cuh: the copy/MMA warpgroup gives most of its share to the softmax warps
    constexpr uint32_t kRegsLow = 56, kRegsHigh = 104;
    static_assert(128 * kRegsLow + 512 * kRegsHigh <= 640 * 96, "register split");
    if (warp == 3) {
        ptx::regs_dec<kRegsLow>();
    } else if (warp == 0 || warp == 2) {
        ptx::regs_dec<kRegsLow>();
        // ------------------------------------------------------------- producers: warp 0 Q and K, warp 2 V
        const bool kq = warp == 0;
        const int S = kq ? KS : VS;
        const uint64_t keep = ptx::policy_evict_last();
        int issued_q = 0, issued = 0;  // copies issued so far (warp-uniform): Q pairs; K or V tiles
        for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
            const PairItem pi = decode_pair(a, item);
            int n_a;
            const int n = item_units(a, pi, &n_a);
            if (n == 0) continue;
            const int32_t row0 = int32_t(int64_t(pi.hh) * a.n_slots);
            const int head = kDirect ? __ldg(a.heads + pi.hh) : 0;
            if (kq && !a.hold_q &&
                __all_sync(0xffffffffu, ptx::mbar_wait(&B.q_empty, (issued_q & 1) ^ 1, abort_flag, tmo))) {
                if (ptx::elect_one()) {
                    const int nq = pi.qb >= 0 ? 2 : 1;
                    ptx::mbar_arrive_expect_tx(&B.q_full, nq * C::kQKBytes);
                    for (int x = 0; x < nq; ++x) {
                        const int qt = x ? pi.qb : pi.qa;
                        uint8_t* dst = smem + C::kOffQ + x * C::kQKBytes;
                        if constexpr (kDirect) {
                            const int4 tc = __ldg(a.tile_coord + qt);
                            for (int b = 0; b < C::kBoxes; ++b) {
                                if (tc.x >= 0)
                                    ptx::tma_load_5d_hint(dst + b * 16384, &maps.q[tc.x], b * 64, head, tc.y, tc.z, tc.w,
                                                          &B.q_full, keep);
                                else
                                    ptx::tma_load_3d_hint(dst + b * 16384, &maps.q[kGlobalMapSet], b * 64, head, tc.y,
                                                          &B.q_full, keep);
                            }
                        } else {
                            for (int b = 0; b < C::kBoxesQK; ++b)
                                ptx::tma_load_2d(dst + b * 16384, &maps.q[0], b * (kFp8 ? 128 : 64), row0 + qt * 128,
                                                 &B.q_full);
                        }
                    }
                }
                __syncwarp();
                ++issued_q;
            }
            if (__any_sync(0xffffffffu, *abort_flag)) break;
            int mine = 0;
            int4 cmine = make_int4(0, 0, 0, 0);  // gather-free variant: box origin of this lane's unit's tile
            for (int j = 0; j < n; ++j) {
                if ((j & 31) == 0) {
                    mine = (j + lane < n) ? item_unit(a, pi, j + lane) : 0;
                    if constexpr (kDirect) cmine = __ldg(a.tile_coord + (mine >> 3));
                }
                const int u = __shfl_sync(0xffffffffu, mine, j & 31);
                int4 tc = make_int4(0, 0, 0, 0);
                if constexpr (kDirect) {
                    tc.x = __shfl_sync(0xffffffffu, cmine.x, j & 31);
                    tc.y = __shfl_sync(0xffffffffu, cmine.y, j & 31);
                    tc.z = __shfl_sync(0xffffffffu, cmine.z, j & 31);
                    tc.w = __shfl_sync(0xffffffffu, cmine.w, j & 31);
                }
                if ((u & 2) == 0) continue;  // the tile came with the unit before
                const int y = row0 + (u >> 3) * 128;
                const int st = issued % S, ph = issued / S;
                uint64_t* empty = kq ? &B.k_empty[st] : &B.v_empty[st];
                uint64_t* full = kq ? &B.k_full[st] : &B.v_full[st];
                const int bytes = kq ? C::kQKBytes : C::kTileBytes;
                uint8_t* dst = smem + (kq ? C::kOffK : C::kOffV) + st * bytes;
                if (__all_sync(0xffffffffu, ptx::mbar_wait(empty, (ph & 1) ^ 1, abort_flag, tmo))) {
                    if (ptx::elect_one()) {
                        ptx::mbar_arrive_expect_tx(full, bytes);
                        const int boxes = kq ? C::kBoxesQK : C::kBoxes, xstep = (kq && kFp8) ? 128 : 64;
                        for (int b = 0; b < boxes; ++b) {
                            if constexpr (kDirect) {
                                if (tc.x >= 0)
                                    ptx::tma_load_5d_hint(dst + b * 16384, kq ? &maps.k[tc.x] : &maps.v[tc.x], b * 64, head,
                                                          tc.y, tc.z, tc.w, full, keep);
                                else
                                    ptx::tma_load_3d_hint(dst + b * 16384,
                                                          kq ? &maps.k[kGlobalMapSet] : &maps.v[kGlobalMapSet], b * 64,
                                                          head, tc.y, full, keep);
                            } else {
                                ptx::tma_load_2d_hint(dst + b * 16384, kq ? &maps.k[0] : &maps.v[0], b * xstep, y, full,
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
        int it = 0;            // items with units so far
        int ks = 0, kph = 0;   // K ring slot of the current key tile and its phase
        int vs = 0, vph = 0;   // V ring slot of the current key tile's PVs and its phase
        int pu0 = 0, pu1 = 0;  // units each group has had so far (barrier phases)
        const uint64_t dq = ptx::smem_desc_sw128(ptx::smem_addr(smem + C::kOffQ), 16, 1024);
        const uint64_t dk = ptx::smem_desc_sw128(ptx::smem_addr(smem + C::kOffK), 16, 1024);
        const uint64_t dv = ptx::smem_desc_sw128(ptx::smem_addr(smem + C::kOffV), 16384, 1024);
        for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
            const PairItem pi = decode_pair(a, item);
            int n_a;
            const int n = item_units(a, pi, &n_a);
            if (n == 0) continue;
            {
                int mine = 0;
                int u1 = 0, u2 = 0;                        // units of the two steps before this one
                bool wrote_a = false, wrote_b = false;     // O of query tile A / B written in this item
                // one issue step: PV of unit j - 2 and S of unit j, both of group W = j % 2
                auto step = [&](const int j, auto wc) -> bool {
                    constexpr int w = decltype(wc)::value;
                    int us = 0;
                    if (j < n) {
                        if ((j & 31) == 0) mine = (j + lane < n) ? item_unit(a, pi, j + lane) : 0;
                        us = __shfl_sync(0xffffffffu, mine, j & 31);
                    }
                    if (j >= 2) {
                        const int jj = j - 2, up = u2, idx = (w ? pu1 : pu0) + (jj >> 1);
                        bool ok = ptx::mbar_wait(&B.p_full[w], idx & 1, abort_flag, tmo) &&
                                  ((up & 2) == 0 || ptx::mbar_wait(&B.v_full[vs], vph, abort_flag, tmo)) &&
                                  (jj > 0 || ptx::mbar_wait(&B.o_empty, (it & 1) ^ 1, abort_flag, tmo));
                        if (!__all_sync(0xffffffffu, ok)) return false;
                        ptx::tc_fence_after();
                        const int x = up & 1;
                        const bool acc = x ? wrote_b : wrote_a;
                        const uint64_t dvs = dv + uint64_t(vs * (C::kTileBytes >> 4));
                        const uint32_t o = tmem + 256 + 128 * x, p = tmem + 128 * w;
#pragma unroll
                        // P of keys 0-63 sits in the group's columns 0-31, of keys 64-127 in 64-95
                        for (int kk = 0; kk < 8; ++kk)
                            ptx::mma_bf16_ts_w(o, p + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8),
                                               dvs + uint64_t(kk * (2048 >> 4)), C::kIdescPV, (acc || kk > 0) ? 1u : 0u);
                        if (x)
                            wrote_b = true;
                        else
                            wrote_a = true;
                        if (up & 4) {  // the key tile's last PV: its V slot may be refilled once it completes
                            ptx::mma_commit_w(&B.v_empty[vs]);
                            if (++vs == VS) vs = 0, vph ^= 1;
                        }
                        if (jj == n - 1) ptx::mma_commit_w(&B.o_done);
                    }
                    if (j < n) {
                        if ((us & 2) && !__all_sync(0xffffffffu, ptx::mbar_wait(&B.k_full[ks], kph, abort_flag, tmo)))
                            return false;
                        ptx::tc_fence_after();
                        const uint64_t dks = dk + uint64_t(ks * (C::kQKBytes >> 4));
                        const uint64_t dqx = dq + uint64_t((us & 1) * (C::kQKBytes >> 4));
                        if constexpr (kFp8) {
                            // 8-bit codes: one 128-byte box holds the tile's 128 columns, 32 per k-step
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                if constexpr (kQK == kQKI8)
                                    ptx::mma_i8_ss_w(tmem + 128 * w, dqx + uint64_t(kk * 2), dks + uint64_t(kk * 2),
                                                     C::kIdescS, kk > 0);
                                else
                                    ptx::mma_f8_ss_w(tmem + 128 * w, dqx + uint64_t(kk * 2), dks + uint64_t(kk * 2),
                                                     C::kIdescS, kk > 0);
                            }
                        } else {
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                const uint64_t off = uint64_t((kk >> 2) * (16384 >> 4) + (kk & 3) * 2);
                                ptx::mma_bf16_ss_w(tmem + 128 * w, dqx + off, dks + off, C::kIdescS, kk > 0);
                            }
                        }
                        ptx::mma_commit_w(&B.s_full[w]);
                        if (us & 4) {  // the key tile's last S: its K slot may be refilled once it completes
                            ptx::mma_commit_w(&B.k_empty[ks]);
                            if (++ks == KS) ks = 0, kph ^= 1;
                        }
                        if (j == n - 1) ptx::mma_commit_w(&B.q_empty);
                    }
                    u2 = u1;
                    u1 = us;
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
        const int sw = warp - 4;
        const int w = sw >> 3;           // group: units j with j % 2 == w; writes out query tile w (A or B)
        const int half = (sw >> 2) & 1;  // key columns [64 half, 64 half + 64) of each S tile
        const int q4 = warp & 3;         // TMEM lane quarter this warp may access
        const int row = q4 * 32 + lane;
        const uint32_t lane_base = uint32_t(q4 * 32) << 16;
        const uint32_t t_s = tmem + lane_base + 128 * w + 64 * half;  // this half's S columns (its P: the first 32)
        constexpr int kCols = D / 2;                                  // output columns each thread writes
        const uint32_t t_o = tmem + lane_base + 256 + 128 * w + half * kCols;
        int cu = 0;  // units this group has had so far (barrier phases)
        int it = 0;  // items with units so far
        for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
            const PairItem pi = decode_pair(a, item);
            int n_a;
            const int n = item_units(a, pi, &n_a);
            const int head = __ldg(a.heads + pi.hh);
            const bool head_ok = head >= 0 && head < a.h_total;
            if (!head_ok && threadIdx.x == 128) atomicOr(a.err, 4);
            const int prow_a = head_ok ? __ldg(a.perm + int64_t(pi.qa) * 128 + row) : -1;
            const int prow_b = head_ok && pi.qb >= 0 ? __ldg(a.perm + int64_t(pi.qb) * 128 + row) : -1;
            const int prow = w ? prow_b : prow_a;  // the row this thread writes out
            const int qt_out = w ? pi.qb : pi.qa;
            const int n_out = w ? n - n_a : n_a;   // units of that query tile
            __nv_bfloat16* dst = a.out + int64_t(prow < 0 ? 0 : prow) * a.out_s0 +
                                 int64_t(head_ok ? head : 0) * a.out_s1 + half * kCols;
            if (n == 0) {
                if (prow >= 0) {
                    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int c = 0; c < kCols / 8; ++c) reinterpret_cast<uint4*>(dst)[c] = z;
                }
                continue;
            }
            // -m of each row of A and B: m = bound - kBoundOffset; padding rows take m = +inf (P = 0)
            auto neg_ref = [&](int pr) -> float {
                if (pr < 0) return -INFINITY;
                const float bound =
                    sqrtf(__ldg(a.q_row_sq + int64_t(pi.hh) * a.seq_len + pr) * __ldg(a.k_max_sq + pi.hh)) * a.scale_log2;
                return kBoundOffset - bound;
            };
            const float negm_a = neg_ref(prow_a), negm_b = neg_ref(prow_b);
            // 8-bit codes: the query tiles' scales (the key tiles' come with their units)
            const float sq_a = kFp8 ? __ldg(a.scales_q + int64_t(pi.hh) * a.n_tiles + pi.qa) : 1.f;
            const float sq_b = kFp8 && pi.qb >= 0 ? __ldg(a.scales_q + int64_t(pi.hh) * a.n_tiles + pi.qb) : 1.f;
            uint64_t sum_a = ptx::f2_pack(0.f, 0.f), sum_b = ptx::f2_pack(0.f, 0.f);
            bool ok = true;
            int my_unit = 0, my_vc = 128;
            float my_sk = 1.f;
            const int nw = group_tiles(n, w);
            for (int k = 0; k < nw; ++k) {
                if ((k & 31) == 0) {
                    const int jj = 2 * (k + lane) + w;
                    my_unit = jj < n ? item_unit(a, pi, jj) : 0;
                    my_vc = jj < n ? __ldg(a.valid_count + (my_unit >> 3)) : 128;
                    if (kFp8) my_sk = jj < n ? __ldg(a.scales_k + int64_t(pi.hh) * a.n_tiles + (my_unit >> 3)) : 1.f;
                }
                const int u = __shfl_sync(0xffffffffu, my_unit, k & 31);
                const int vc = __shfl_sync(0xffffffffu, my_vc, k & 31);
                // log2-domain scale of this unit's logits (the 8-bit codes also undo both tiles' scales)
                const float sl2 =
                    kFp8 ? a.scale_log2 * (((u & 1) ? sq_b : sq_a) * __shfl_sync(0xffffffffu, my_sk, k & 31))
                         : a.scale_log2;
                const uint64_t sl2x2 = ptx::f2_pack(sl2, sl2);
                ok = ptx::mbar_wait(&B.s_full[w], (cu + k) & 1, abort_flag, tmo);
                if (!ok) break;
                ptx::tc_fence_after();
                // S of this unit is complete; it was issued after the PV of this group's previous unit, so
                // that PV is complete too and the P columns may be rewritten
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
                        const uint4 m = __ldg(a.tile_mask + (u >> 3));
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
                const float negm = (u & 1) ? negm_b : negm_a;
                const uint64_t negm2 = ptx::f2_pack(negm, negm);
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    const uint64_t x =
                        ptx::f2_fma(ptx::f2_pack(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sl2x2, negm2);
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
                ptx::tmem_st32(t_s, *reinterpret_cast<uint32_t(*)[32]>(s));
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(&B.p_full[w]);
                // the row sums come after the hand-off, off the path to the PV: over the bf16 P the PV
                // product reads (eight independent chains)
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 32; ++c) ptx::add_bf16x2(s[c], acc[c & 3], acc[4 + (c & 3)]);
                const uint64_t tot = ptx::f2_add(ptx::f2_add(ptx::f2_pack(acc[0], acc[4]), ptx::f2_pack(acc[1], acc[5])),
                                                 ptx::f2_add(ptx::f2_pack(acc[2], acc[6]), ptx::f2_pack(acc[3], acc[7])));
                if (u & 1)
                    sum_b = ptx::f2_add(sum_b, tot);
                else
                    sum_a = ptx::f2_add(sum_a, tot);
            }
            if (!ok) break;
            cu += nw;
            // the row sums of A and B are final with the thread's last unit: each thread publishes its part
            // and reads the row's four parts while the item's last PVs still run, so that after them only
            // the read of O stands before its release. The sums of consecutive items use the two halves of
            // the buffer: a thread can publish the next item's before every thread has read this one's
            float2* st = stats + (it & 1) * 512;
            {
                float a0, a1, b0, b1;
                ptx::f2_unpack(sum_a, a0, a1);
                ptx::f2_unpack(sum_b, b0, b1);
                st[(w * 2 + half) * 128 + row] = make_float2(a0 + a1, b0 + b1);
            }
            ptx::mbar_arrive(&B.merge);
            ok = ptx::mbar_wait(&B.merge, it & 1, abort_flag, tmo);
            if (!ok) break;
            const float2 g00 = st[row], g01 = st[128 + row], g10 = st[256 + row], g11 = st[384 + row];
            const float l = w ? (g00.y + g01.y) + (g10.y + g11.y) : (g00.x + g01.x) + (g10.x + g11.x);
            const bool have = n_out > 0;
            // a real row whose sum left [2^-60, 2^100] (or is NaN): the exact redo rewrites its query tile
            const bool redo = prow >= 0 && have && !(l >= kRedoBelow && l <= kRedoAbove);
            if (__any_sync(0xffffffffu, redo) && lane == 0 &&
                atomicOr(a.redo_flags + int64_t(pi.hh) * a.n_tiles + qt_out, 1) == 0) {
                // the first warp to flag the tile lists it
                const int single = qt_out >= a.n_video ? pi.hh * a.n_global + (qt_out - a.n_video)
                                                       : a.n_heads * a.n_global + pi.hh * a.n_video + qt_out;
                a.redo_items[atomicAdd(a.redo_count, 1)] = single;
            }
            const float inv = l > 0.f ? 1.f / l : 0.f;
            ok = ptx::mbar_wait(&B.o_done, it & 1, abort_flag, tmo);  // every PV of the item is complete
            ++it;
            if (!ok) break;
            ptx::tc_fence_after();
            // this thread's half of the row is read (and scaled into bf16 pairs) before O is released to the
            // next item's first PV; the global stores come after the release
            uint32_t res[kCols / 2];
            if (have) {
#pragma unroll
                for (int h16 = 0; h16 < kCols / 16; ++h16) {
                    uint32_t o[16];
                    ptx::tmem_ld16(t_o + 16 * h16, o);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        res[8 * h16 + c] =
                            ptx::pack_bf16(__uint_as_float(o[2 * c]) * inv, __uint_as_float(o[2 * c + 1]) * inv);
                }
            } else {
#pragma unroll
                for (int c = 0; c < kCols / 2; ++c) res[c] = 0u;
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&B.o_empty);
            if (prow >= 0) {
                uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
                for (int c = 0; c < kCols / 8; ++c)
                    d4[c] = make_uint4(res[4 * c], res[4 * c + 1], res[4 * c + 2], res[4 * c + 3]);
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
