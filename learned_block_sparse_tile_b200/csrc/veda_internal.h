// Internal declarations of libveda (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <string>
#include <vector>

#include "veda.h"

namespace veda {

constexpr int kTile = VEDA_TILE;
constexpr int kMaxDevices = 64;
constexpr int kMaxDirectSpans = 4;  // tiled spans the gather-free attend takes (one TMA map set each)

// A tiled span as the gather-free attend sees it: rows start + (t * h + y) * w + x of a (t, h, w) grid,
// cut into (st, sh, sw) boxes.
struct DirectSpan {
    int64_t start;
    int32_t t, h, w, st, sh, sw;
};

// Device copy of a layout's index data, made once per device on first use.
struct DeviceCopy {
    bool ready = false;
    int32_t* perm = nullptr;         // [n_slots] packed row per slot, -1 on padding
    int32_t* valid_count = nullptr;  // [n_tiles]
    int32_t* ok_list = nullptr;      // [n_kv_ok] ascending ids of non-empty tiles
    int32_t* allowed = nullptr;      // [n_blocks * n_video]
    int32_t* box_perm = nullptr;     // [n_slots] (gather-free attend)
    int32_t* tile_coord = nullptr;   // [n_tiles * 4]
    int32_t* tile_mask = nullptr;    // [n_tiles * 4] (bit patterns)
};

// Records `msg` as the calling thread's last error and returns `code`.
int fail(int code, const std::string& msg);
void clear_error();

// Floats of scratch the predictor's products need per head: the projected q and k features (2 n_video D)
// and the two projections transposed (2 x 3D x D).
inline int64_t score_scratch_per_head(int64_t n_video, int64_t dim) { return 2 * n_video * dim + 6 * dim * dim; }

// Enqueues the predictor's products for n_heads heads on `s` (veda_score's arithmetic): P^T into pt_q /
// pt_k ([n_heads][D][3D]), q_hat / k_hat into qh / kh ([n_heads][n_video][D]), then the scores
// ([n_heads][n_video][n_video]). All pointers 16-byte aligned device memory. Returns a VEDA_* status.
int launch_score_gemms(const float* feats_q, const float* feats_k, const float* proj_q, const float* proj_k, float* qh,
                       float* kh, float* pt_q, float* pt_k, float* scores, int nv, int dim, int n_heads,
                       cudaStream_t s);

}  // namespace veda

struct veda_layout {
    veda_layout_desc desc{};
    std::vector<int32_t> perm;         // [n_slots]
    std::vector<int32_t> valid_count;  // [n_tiles]
    std::vector<int32_t> ok_list;      // [n_kv_ok]
    std::vector<int32_t> allowed;      // [n_blocks * n_video]
    // The tiles as TMA boxes of the packed tensors, for the gather-free attend. A span tile is the 3D box
    // of its span's grid at its origin, positions in box order (t, h, w row-major), padding left in
    // place (positions outside the grid). A global tile is the run of 128 rows from its first row, which
    // needs the tile's rows to be consecutive.
    std::vector<int32_t> box_perm;    // [n_slots] packed row of each box position; -1 where the tile has no row
    std::vector<int32_t> tile_coord;  // [n_tiles * 4] span tile {span, w0, h0, t0}; global tile {-1, row0, 0, 0}
    std::vector<int32_t> tile_mask;   // [n_tiles * 4] bit c (word c / 32) set: box position c holds a row
    std::vector<veda::DirectSpan> spans;  // tiled spans, in tile order
    bool direct_ok = false;           // every global tile's rows are consecutive; spans <= kMaxDirectSpans
    std::string direct_why;           // why not, when direct_ok is false
    mutable std::mutex mu;
    mutable veda::DeviceCopy dev[veda::kMaxDevices];
};
