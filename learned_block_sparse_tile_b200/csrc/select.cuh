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

}  // namespace veda
