// Head-aware top-k selection of key tiles, emitted directly as ascending index lists.
// veda_core.py (ComfyUI-FunPack), "selection": select (per column block: empty key tiles never kept,
// the own tile first, then the best scores; the first k_lo + bresenham(row) are kept; a keeps-all block
// keeps every non-empty tile), block_mask (every non-empty global tile is added to every video row) and
// tile_index_list (the row's kept tiles, ascending).
//
// Order: (score descending, column ascending). Scores are mapped to order-preserving unsigned keys;
// the own tile takes the +inf key; NaN, -inf and empty tiles take the -inf key and are never kept.
// One CTA per (video query row, head). Per block the row's keys sit in shared memory; a 4-pass 8-bit
// radix select finds the threshold key T and how many keys equal to T are taken (the lowest columns);
// two block-wide prefix sums then place the kept columns in ascending order.
#pragma once

#include <cstdint>

namespace veda {

constexpr int kSelectThreads = 256;
constexpr int kSelectMaxCols = 16384;

struct SelectArgs {
    const float* scores;         // [n_heads, n_video, n_video]
    const int32_t* valid_count;  // [n_tiles]
    const int32_t* allowed;      // [n_blocks, n_video]
    const int32_t* ok_list;      // [n_kv_ok]; its last n_global_ok entries are the global tiles
    int32_t* kept_idx;           // [n_heads, n_video, max_kept]
    int32_t* kept_cnt;           // [n_heads, n_video]
    int32_t n_video, n_blocks, max_kept, n_kv_ok, n_global_ok;
    int32_t blk_start[2], blk_stop[2], blk_all[2];
    int32_t n_heads;
    int32_t all_ok;  // every video tile holds a real row (no column is excluded as empty)
};

constexpr uint32_t kKeyNeg = 0x007FFFFFu;  // key of -inf
constexpr uint32_t kKeyPos = 0xFF800000u;  // key of +inf

__device__ __forceinline__ uint32_t order_key(float s) {
    if (s != s) return kKeyNeg;  // NaN ranks as -inf
    uint32_t u = __float_as_uint(s);
    // -0.0 and +0.0 compare equal, so they are one score and tie (the lower column first): both take the
    // key of +0.0
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the CTA (kSelectThreads threads); returns this thread's offset, *total the sum.
__device__ __forceinline__ int block_exclusive_scan(int v, int* total, int* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kSelectThreads / 32 ? scratch[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        if (lane < kSelectThreads / 32) scratch[lane] = w;  // inclusive warp totals
    }
    __syncthreads();
    const int before = (warp ? scratch[warp - 1] : 0) + x - v;
    *total = scratch[kSelectThreads / 32 - 1];
    __syncthreads();
    return before;
}

__global__ void __launch_bounds__(kSelectThreads) select_kernel(const SelectArgs a) {
    extern __shared__ uint32_t keys[];  // [widest block]
    __shared__ int hist[256];
    __shared__ int scratch[32];
    __shared__ uint32_t s_digit;
    __shared__ int s_need;

    const int row = blockIdx.x, hh = blockIdx.y, tid = threadIdx.x;
    const int64_t rowid = int64_t(hh) * a.n_video + row;
    const float* srow = a.scores + rowid * a.n_video;
    int32_t* out = a.kept_idx + rowid * a.max_kept;
    int pos = 0;

    for (int b = 0; b < a.n_blocks; ++b) {
        const int start = a.blk_start[b], n = a.blk_stop[b] - start;
        const int per = (n + kSelectThreads - 1) / kSelectThreads;  // contiguous columns per thread
        const int c0 = tid * per, c1 = min(c0 + per, n);
        if (a.blk_all[b]) {
            int cnt = 0;
            for (int c = c0; c < c1; ++c) cnt += __ldg(a.valid_count + start + c) > 0;
            int total;
            int at = block_exclusive_scan(cnt, &total, scratch) + pos;
            for (int c = c0; c < c1; ++c)
                if (__ldg(a.valid_count + start + c) > 0) out[at++] = start + c;
            pos += total;
            continue;
        }
        const int allowed = __ldg(a.allowed + int64_t(b) * a.n_video + row);
        for (int c = tid; c < n; c += kSelectThreads) {
            const int col = start + c;
            uint32_t k = order_key(__ldg(srow + col));
            if (__ldg(a.valid_count + col) <= 0) k = kKeyNeg;
            if (col == row) k = kKeyPos;
            keys[c] = k;
        }
        __syncthreads();
        uint32_t thr = 0;  // keep keys > thr, plus the first `need` keys == thr
        int need = 0;
        if (allowed <= 0) {
            thr = 0xFFFFFFFFu;  // above every key: nothing is kept
        } else if (allowed < n) {
            uint32_t prefix = 0, pmask = 0;
            int want = allowed;
            for (int shift = 24; shift >= 0; shift -= 8) {
                hist[tid] = 0;  // kSelectThreads == 256 bins
                __syncthreads();
                for (int c = tid; c < n; c += kSelectThreads) {
                    const uint32_t k = keys[c];
                    if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255], 1);
                }
                __syncthreads();
                if (tid < 32) {
                    // lane l owns digits 255-8l .. 248-8l (descending); find where the running count
                    // from the top reaches `want`
                    int local[8], sum = 0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        local[e] = hist[255 - 8 * tid - e];
                        sum += local[e];
                    }
                    int incl = sum;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const int y = __shfl_up_sync(0xffffffffu, incl, off);
                        if (tid >= off) incl += y;
                    }
                    const int excl = incl - sum;
                    const unsigned hit = __ballot_sync(0xffffffffu, incl >= want && excl < want);
                    const int owner = __ffs(hit) - 1;
                    if (tid == owner) {
                        int run = excl;
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            if (run + local[e] >= want) {
                                s_digit = uint32_t(255 - 8 * tid - e);
                                s_need = want - run;
                                break;
                            }
                            run += local[e];
                        }
                    }
                }
                __syncthreads();
                prefix |= s_digit << shift;
                pmask |= 0xFFu << shift;
                want = s_need;
                __syncthreads();
            }
            thr = prefix;
            need = want;
        }
        // ties at the threshold: the lowest columns first
        int eq = 0;
        if (allowed < n)
            for (int c = c0; c < c1; ++c) eq += keys[c] == thr;
        int eq_total;
        int eq_rank = block_exclusive_scan(eq, &eq_total, scratch);
        int sel = 0;
        for (int c = c0; c < c1; ++c) {
            const uint32_t k = keys[c];
            bool take;
            if (allowed >= n && allowed > 0) {
                take = true;
            } else if (k > thr) {
                take = true;
            } else if (k == thr) {
                take = eq_rank < need;
                ++eq_rank;
            } else {
                take = false;
            }
            sel += take && k != kKeyNeg;
        }
        int sel_total;
        int at = block_exclusive_scan(sel, &sel_total, scratch) + pos;
        eq_rank -= eq;
        for (int c = c0; c < c1; ++c) {
            const uint32_t k = keys[c];
            bool take;
            if (allowed >= n && allowed > 0) {
                take = true;
            } else if (k > thr) {
                take = true;
            } else if (k == thr) {
                take = eq_rank < need;
                ++eq_rank;
            } else {
                take = false;
            }
            if (take && k != kKeyNeg) out[at++] = start + c;
        }
        pos += sel_total;
        __syncthreads();  // keys[] is reused by the next block
    }
    const int* glob = a.ok_list + (a.n_kv_ok - a.n_global_ok);
    for (int i = tid; i < a.n_global_ok; i += kSelectThreads) out[pos + i] = __ldg(glob + i);
    if (tid == 0) a.kept_cnt[rowid] = pos + a.n_global_ok;
}

// The same selection with one warp per (video query row, head), for column blocks of at most 32 kPer
// tiles. Column c of a block sits in lane c % 32, slot c / 32, so ballots over a slot list columns in
// ascending order. The threshold key T (the allowed-th largest key of the block) is built bit by bit from
// the top: a candidate bit stays set when at least `allowed` keys are >= the candidate (when exactly
// `allowed` are, T is the smallest of them and the search stops). Keys above T are
// kept, and of the keys equal to T the lowest columns, as many as are still needed. No shared memory and
// no block barriers: a warp owns its row.
template <int kPer>
__global__ void __launch_bounds__(256) select_warp_kernel(const SelectArgs a) {
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5), hh = blockIdx.y;
    if (row >= a.n_video) return;  // whole warps only
    const unsigned lower = (1u << lane) - 1u;
    const int64_t rowid = int64_t(hh) * a.n_video + row;
    const float* srow = a.scores + rowid * a.n_video;
    int32_t* out = a.kept_idx + rowid * a.max_kept;
    int pos = 0;
    for (int b = 0; b < a.n_blocks; ++b) {
        const int start = a.blk_start[b], n = a.blk_stop[b] - start;
        if (a.blk_all[b]) {
            for (int i = 0; i * 32 < n; ++i) {
                const int c = i * 32 + lane;
                const bool ok = c < n && __ldg(a.valid_count + start + c) > 0;
                const unsigned bal = __ballot_sync(0xffffffffu, ok);
                if (ok) out[pos + __popc(bal & lower)] = start + c;
                pos += __popc(bal);
            }
            continue;
        }
        const int allowed = __ldg(a.allowed + int64_t(b) * a.n_video + row);
        uint32_t key[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int c = i * 32 + lane, col = start + c;
            uint32_t k = 0;  // below every real key (the -inf key is 0x007FFFFF); never counted or kept
            if (c < n) {
                k = order_key(__ldg(srow + col));
                if (__ldg(a.valid_count + col) <= 0) k = kKeyNeg;
                if (col == row) k = kKeyPos;
            }
            key[i] = k;
        }
        uint32_t thr;  // keep keys > thr, plus the first `need` keys == thr (lowest columns)
        int need = 0;
        if (allowed <= 0) {
            thr = 0xFFFFFFFFu;  // nothing is kept
        } else if (allowed >= n) {
            thr = 0u;  // every real key is > 0
        } else {
            // thr keeps at least `allowed` keys >= thr. A candidate with exactly `allowed` keys >= it ends the
            // search: the allowed-th largest key is then the smallest of those keys.
            thr = 0u;
            bool exact = false;
            for (int bit = 31; bit >= 0; --bit) {
                const uint32_t cand = thr | (1u << bit);
                unsigned cnt = 0;
#pragma unroll
                for (int i = 0; i < kPer; ++i) cnt += key[i] >= cand;
                const int total = int(__reduce_add_sync(0xffffffffu, cnt));
                if (total >= allowed) {
                    thr = cand;
                    if (total == allowed) {
                        exact = true;
                        break;
                    }
                }
            }
            if (exact) {
                uint32_t lo = 0xFFFFFFFFu;
#pragma unroll
                for (int i = 0; i < kPer; ++i)
                    if (key[i] >= thr) lo = min(lo, key[i]);
                thr = __reduce_min_sync(0xffffffffu, lo);
            }
            unsigned above = 0;
#pragma unroll
            for (int i = 0; i < kPer; ++i) above += key[i] > thr;
            need = allowed - int(__reduce_add_sync(0xffffffffu, above));
        }
        int ties = 0;  // keys == thr taken so far, in column order
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const uint32_t k = key[i];
            const unsigned tie = __ballot_sync(0xffffffffu, k == thr && thr != 0u);
            const bool take = k != 0u && k != kKeyNeg &&
                              (k > thr || (k == thr && ties + __popc(tie & lower) < need));
            ties += __popc(tie);
            const unsigned bal = __ballot_sync(0xffffffffu, take);
            if (take) out[pos + __popc(bal & lower)] = start + i * 32 + lane;
            pos += __popc(bal);
        }
    }
    const int* glob = a.ok_list + (a.n_kv_ok - a.n_global_ok);
    for (int i = lane; i < a.n_global_ok; i += 32) out[pos + i] = __ldg(glob + i);
    if (lane == 0) a.kept_cnt[rowid] = pos + a.n_global_ok;
}

// ---------------------------------------------------------------------------------------------------
// select_rows_kernel: the same selection with one warp per (head, video row), for rows of at most 32 kPer
// video tiles.
//
// Column c of the row sits in lane c % 32, slot c / 32 (ballots over a slot list columns in ascending
// order). Per column block the warp first works on a 16-bit image of the scores: every score rounded to
// fp16, a monotone map (a > b gives h(a) >= h(b)), packed two columns per register so that one fp16x2
// compare and one fp16x2 add count two columns. Columns that are never kept (NaN, -inf, empty tiles) and
// columns outside the block get an fp16 NaN image, which no comparison counts; the own tile gets +inf.
//   Phase A bisects the 16-bit order key of the images for the allowed-th largest image T. A column whose
//   image is above T scores above every column whose image is T or less, so it is kept; a column below T
//   is not. When a candidate value v has exactly `allowed` images >= v, those columns are the kept set.
//   Phase B ranks the columns whose image equals T by their exact scores (32-bit order keys, the own tile
//   as +inf, ties to the lower column) and keeps as many as are still needed: with at most 32 such
//   columns lane j ranks the j-th against the others; beyond that a bisection of the exact key runs over
//   them, reading their scores again.
// The outcome of each stage is a per-lane bit mask over the slots, and the loops over slots run on those
// masks (not unrolled), which keeps the kernel's code and register footprint small. No block barriers
// after the start: a warp owns its row. The CTA shares a bitmap of the non-empty video tiles (built once,
// when some tile is empty) and per warp a 32-entry candidate list and a kept-candidate mask per lane.
constexpr int kRowsWarps = 8;  // warps per CTA

__device__ __forceinline__ uint32_t h2_pack(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}
__device__ __forceinline__ uint32_t h2_set_ge(uint32_t a, uint32_t b) {  // 1.0 / 0.0 per half
    uint32_t d;
    asm("set.ge.f16x2.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t h2_set_gt(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("set.gt.f16x2.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t h2_set_eq(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("set.eq.f16x2.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t h2_add(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// fp16 bits of a 16-bit order key (the inverse of: non-negative h -> h | 0x8000, negative h -> ~h)
__device__ __forceinline__ uint32_t key16_half(uint32_t k) { return (k & 0x8000u) ? (k & 0x7FFFu) : (~k & 0xFFFFu); }

constexpr uint32_t kHalfNaN = 0x7E00u;       // OR-ing it into an fp16 value makes a NaN
constexpr uint32_t kKey16NegInf = 0x03FFu;  // order key of fp16 -inf

// The two slot bits (low half, high half) of one fp16x2 comparison result (1.0 where true).
__device__ __forceinline__ uint64_t pair_bits(uint32_t r) {
    return uint64_t((r & 0xFFFFu) != 0u) | (uint64_t((r >> 16) != 0u) << 1);
}

// Phase B with more than 32 candidates (slots in `cand`): bisection of their exact keys for the need-th
// largest, ties to the lower column, reading the scores again. Returns this lane's kept candidates.
__device__ __noinline__ uint64_t select_wide_candidates(const float* srow, int row, uint64_t cand, int n_slots,
                                                        int need) {
    const int lane = threadIdx.x & 31;
    const unsigned lower = (1u << lane) - 1u;
    auto key_of = [&](int i) -> uint32_t {
        const int c = i * 32 + lane;
        return c == row ? kKeyPos : order_key(__ldg(srow + c));
    };
    uint32_t thr = 0;
    bool exact = false;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cv = thr | (1u << bit);
        unsigned cnt = 0;
        for (int i = 0; i < n_slots; ++i)
            if ((cand >> i) & 1u) cnt += key_of(i) >= cv;
        const int total = int(__reduce_add_sync(0xffffffffu, cnt));
        if (total >= need) {
            thr = cv;
            if (total == need) {
                exact = true;
                break;
            }
        }
    }
    if (exact) {
        uint32_t lo = 0xFFFFFFFFu;
        for (int i = 0; i < n_slots; ++i)
            if ((cand >> i) & 1u) {
                const uint32_t k = key_of(i);
                if (k >= thr) lo = min(lo, k);
            }
        thr = __reduce_min_sync(0xffffffffu, lo);
    }
    unsigned above = 0;
    for (int i = 0; i < n_slots; ++i)
        if ((cand >> i) & 1u) above += key_of(i) > thr;
    const int need2 = need - int(__reduce_add_sync(0xffffffffu, above));
    int ties = 0;  // candidates == thr taken so far, in column order
    uint64_t kept = 0;
    for (int i = 0; i < n_slots; ++i) {
        const bool is_c = (cand >> i) & 1u;
        const uint32_t k = is_c ? key_of(i) : 0u;
        const bool is_tie = is_c && k == thr;
        const unsigned tie = __ballot_sync(0xffffffffu, is_tie);
        const bool take = is_c && (k > thr || (is_tie && ties + __popc(tie & lower) < need2));
        ties += __popc(tie);
        kept |= uint64_t(take) << i;
    }
    return kept;
}

// kTwo: the layout has two column blocks (references and target), so each block works on a masked copy of
// the row's images; with one block (every video tile) the images are used as packed.
template <int kPer, bool kTwo>
__global__ void __launch_bounds__(32 * kRowsWarps) select_rows_kernel(const SelectArgs a) {
    static_assert(kPer % 2 == 0 && kPer <= 64, "slots per lane");
    constexpr int kPairs = kPer / 2;
    __shared__ uint32_t okbits[kPer];             // bit c % 32 of word c / 32: video tile c holds a real row
    __shared__ int32_t cand_col[kRowsWarps][32];  // phase B: the first 32 candidate columns, ascending
    __shared__ uint64_t keep_mask[kRowsWarps][32];  // phase B: per lane, the slots of its kept candidates
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const unsigned lower = (1u << lane) - 1u;
    const int nv = a.n_video;
    if (!a.all_ok) {
        for (int w = threadIdx.x; w < kPer; w += blockDim.x) okbits[w] = 0u;
        __syncthreads();
        for (int c = threadIdx.x; c < nv; c += blockDim.x)
            if (__ldg(a.valid_count + c) > 0) atomicOr(&okbits[c >> 5], 1u << (c & 31));
        __syncthreads();
    }
    const int64_t rowid = int64_t(blockIdx.x) * kRowsWarps + wib;
    if (rowid >= int64_t(a.n_heads) * nv) return;  // whole warps only
    const int row = int(rowid % nv);
    const float* srow = a.scores + rowid * nv;
    int32_t* out = a.kept_idx + rowid * a.max_kept;

    // fp16 images of the row: NaN where a column can never be kept, +inf for the own tile
    uint32_t hrow[kPairs];
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        float v[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = 2 * j + u, c = i * 32 + lane;
            const float x = c < nv ? __ldg(srow + c) : 0.f;
            const bool ok = c < nv && (a.all_ok || ((okbits[i] >> lane) & 1u)) && x == x && x != -INFINITY;
            v[u] = c == row ? INFINITY : ok ? x : __int_as_float(0x7fc00000);
        }
        hrow[j] = h2_pack(v[0], v[1]);
    }
    int pos = 0;
    for (int b = 0; b < (kTwo ? 2 : 1); ++b) {
        // (selects, not a.blk_*[b]: a runtime index into the kernel arguments would copy them to the stack)
        const int start = b ? a.blk_start[1] : a.blk_start[0], stop = b ? a.blk_stop[1] : a.blk_stop[0];
        uint64_t take = 0;  // this lane's kept slots in the block
        if (b ? a.blk_all[1] : a.blk_all[0]) {
            for (int i = 0; i < kPer; ++i) {
                const int c = i * 32 + lane;
                take |= uint64_t(c >= start && c < stop && (a.all_ok || ((okbits[i] >> lane) & 1u))) << i;
            }
        } else {
            const int allowed = __ldg(a.allowed + int64_t(b) * nv + row);
            // the block's images: NaN outside [start, stop) (a single block holds every video tile)
            uint32_t h[kPairs];
            int fin = 0;
#pragma unroll
            for (int j = 0; j < kPairs; ++j) {
                const int c0 = 2 * j * 32 + lane, c1 = c0 + 32;
                h[j] = kTwo ? hrow[j] | ((c0 >= start && c0 < stop) ? 0u : kHalfNaN) |
                                  ((c1 >= start && c1 < stop) ? 0u : (kHalfNaN << 16))
                            : hrow[j];
                fin += __popcll(pair_bits(h2_set_eq(h[j], h[j])));  // not NaN
            }
            const int n_fin = int(__reduce_add_sync(0xffffffffu, uint32_t(fin)));
            if (allowed >= n_fin) {
#pragma unroll
                for (int j = 0; j < kPairs; ++j) take |= pair_bits(h2_set_eq(h[j], h[j])) << (2 * j);
            } else if (allowed > 0) {
                // phase A: the largest 16-bit key whose image has at least `allowed` images >= it
                uint32_t thr = 0;
                bool exact = false;
                for (int bit = 15; bit >= 0; --bit) {
                    const uint32_t cand = thr | (1u << bit);
                    const uint32_t hv = key16_half(cand);
                    const uint32_t c2 = hv | (hv << 16);
                    uint32_t acc[4] = {0x64006400u, 0x64006400u, 0x64006400u, 0x64006400u};  // 1024.0 + count
#pragma unroll
                    for (int j = 0; j < kPairs; ++j) acc[j & 3] = h2_add(acc[j & 3], h2_set_ge(h[j], c2));
                    uint32_t cnt = 0;
#pragma unroll
                    for (int q = 0; q < 4; ++q) cnt += (acc[q] & 0x3FFu) + ((acc[q] >> 16) & 0x3FFu);
                    const int total = int(__reduce_add_sync(0xffffffffu, cnt));
                    if (total >= allowed) {
                        thr = cand;
                        if (total == allowed) {
                            exact = true;
                            break;
                        }
                    }
                }
                // keys below that of fp16 -inf hold NaN images and count nothing: when every key above it
                // fails, the allowed-th largest image is -inf itself
                if (thr < kKey16NegInf) thr = kKey16NegInf;
                const uint32_t hv = key16_half(thr);
                const uint32_t t2 = hv | (hv << 16);
                uint64_t cand = 0;  // images equal to T (phase B candidates)
#pragma unroll
                for (int j = 0; j < kPairs; ++j) {
                    take |= pair_bits(exact ? h2_set_ge(h[j], t2) : h2_set_gt(h[j], t2)) << (2 * j);
                    cand |= pair_bits(h2_set_eq(h[j], t2)) << (2 * j);
                }
                if (!exact) {
                    const int need = allowed - int(__reduce_add_sync(0xffffffffu, uint32_t(__popcll(take))));
                    const int n_cand = int(__reduce_add_sync(0xffffffffu, uint32_t(__popcll(cand))));
                    if (n_cand <= 32) {
                        // list the candidates in ascending column order, lane j ranks the j-th
                        keep_mask[wib][lane] = 0;
                        int at = 0;
                        const unsigned any_lo = __reduce_or_sync(0xffffffffu, uint32_t(cand));
                        const unsigned any_hi = __reduce_or_sync(0xffffffffu, uint32_t(cand >> 32));
                        uint64_t slots = (uint64_t(any_hi) << 32) | any_lo;  // slots where some lane has one
                        while (slots) {
                            const int i = __ffsll(static_cast<long long>(slots)) - 1;
                            slots &= slots - 1;
                            const bool is_c = (cand >> i) & 1u;
                            const unsigned bal = __ballot_sync(0xffffffffu, is_c);
                            if (is_c) cand_col[wib][at + __popc(bal & lower)] = i * 32 + lane;
                            at += __popc(bal);
                        }
                        __syncwarp();
                        uint32_t key = 0;
                        int c = 0;
                        if (lane < n_cand) {
                            c = cand_col[wib][lane];
                            key = c == row ? kKeyPos : order_key(__ldg(srow + c));
                        }
                        int rank = 0;
                        for (int i = 0; i < n_cand; ++i) {
                            const uint32_t ki = __shfl_sync(0xffffffffu, key, i);
                            rank += (ki > key) || (ki == key && i < lane);
                        }
                        if (lane < n_cand && rank < need)
                            atomicOr(reinterpret_cast<unsigned long long*>(&keep_mask[wib][c & 31]), 1ull << (c >> 5));
                        __syncwarp();
                        take |= keep_mask[wib][lane];
                        __syncwarp();  // cand_col and keep_mask are rewritten by the next block
                    } else {
                        take |= select_wide_candidates(srow, row, cand, kPer, need);
                    }
                }
            }
        }
        // output: ascending columns, over the slots where some lane keeps a column
        const unsigned any_lo = __reduce_or_sync(0xffffffffu, uint32_t(take));
        const unsigned any_hi = __reduce_or_sync(0xffffffffu, uint32_t(take >> 32));
        uint64_t slots = (uint64_t(any_hi) << 32) | any_lo;
        while (slots) {
            const int i = __ffsll(static_cast<long long>(slots)) - 1;
            slots &= slots - 1;
            const bool t = (take >> i) & 1u;
            const unsigned bal = __ballot_sync(0xffffffffu, t);
            if (t) out[pos + __popc(bal & lower)] = i * 32 + lane;
            pos += __popc(bal);
        }
    }
    const int* glob = a.ok_list + (a.n_kv_ok - a.n_global_ok);
    for (int i = lane; i < a.n_global_ok; i += 32) out[pos + i] = __ldg(glob + i);
    if (lane == 0) a.kept_cnt[rowid] = pos + a.n_global_ok;
}

}  // namespace veda
