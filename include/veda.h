/*
 * veda.h - C ABI of the Veda tile-skip sparse-attention path for NVIDIA B200 (sm_100a).
 *
 * What the calls compute is defined by the page "veda_core.py" (ComfyUI-FunPack node pack, "Veda
 * sparse attention, the torch half"); each declaration below names the section and function it
 * follows. One attention layer is, per group of heads that share a target tile box:
 *
 *     veda_plan      -> tile layout of the packed sequence + per-row budgets   (host, once per geometry)
 *     veda_gather    -> Q, K (and V) in tile order; Q/K pooled to [mean|max|min] per tile
 *     veda_score     -> per-head projected tile-pair scores
 *     veda_select    -> kept key tiles of every video query tile (ascending index lists)
 *     veda_attend    -> flash attention over the kept K/V tiles, written back to packed row order
 *
 * Conventions shared by every call
 *  - Every pointer named "device" is CUDA device memory owned by the caller; the library never frees
 *    it and keeps no reference to it after the call returns. Host pointers are read during the call only.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Device calls are
 *    asynchronous: they enqueue kernels and return; errors detected inside a kernel (a bounded wait
 *    that expired, a malformed kept list) are latched in a per-device error word that
 *    veda_sync_status() reads.
 *  - bf16 tensors are IEEE bfloat16 (2 bytes). Strided [S, H, D] tensors need a unit stride on D,
 *    strides on S and H that are multiples of 8 elements, and a 16-byte aligned base.
 *  - Tile-ordered tensors are head-major: [n_heads, N, D] with N = 128 * n_tiles rows per head, row
 *    r of head h at ((h * N) + r) * D. Padding slots hold zeros.
 *  - Return value: VEDA_OK or an error code; the text of the last error of the calling thread is
 *    returned by veda_last_error(). There is no fallback path: a call that cannot run fails.
 */
#ifndef VEDA_H
#define VEDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VEDA_TILE 128

/* status codes */
#define VEDA_OK 0
#define VEDA_ERR_INVALID 1     /* a layout, budget, shape, stride or pointer the method cannot use */
#define VEDA_ERR_CUDA 2        /* a CUDA runtime/driver call failed */
#define VEDA_ERR_TIMEOUT 3     /* a bounded device-side wait expired (the kernel stopped cleanly) */
#define VEDA_ERR_UNSUPPORTED 4 /* not an sm_100 device, or a size beyond a kernel's limit */
#define VEDA_ERR_BAD_LIST 5    /* a kept list was out of range or not ascending (device check) */

/* budget kinds: exactly one must be set (veda_core.py, "budgets": a budget is (ratio, tiles)) */
#define VEDA_BUDGET_RATIO 1
#define VEDA_BUDGET_TILES 2

typedef struct veda_layout veda_layout; /* opaque; created by veda_plan, freed by veda_layout_destroy */

/* A span of packed rows forming a row-major 3D grid (t, h, w), w fastest. A zero box (st = sh = sw = 0)
 * asks for the least-padding box of the grid (veda_core.py, "tiles", least_padding_shape). */
typedef struct {
    int64_t start;
    int32_t t, h, w;
    int32_t st, sh, sw;
} veda_span;

/* kind = VEDA_BUDGET_RATIO: keep `ratio` of the key tiles (at equal kernel cost);
 * kind = VEDA_BUDGET_TILES: keep exactly `tiles` key tiles per query tile. Any other kind is invalid
 * (neither or both set). veda_core.py, "budgets": sparsity_budget, keeps_all, _per_row. */
typedef struct {
    int32_t kind;
    double ratio;
    int64_t tiles;
} veda_budget;

/* One key-column block with its own top-k (veda_core.py, "selection", column_blocks and _split). */
typedef struct {
    int32_t start, stop;  /* video key tiles [start, stop) */
    int32_t keeps_all;    /* 1: every non-empty tile of the block is kept */
    int32_t k_lo, k_hi;   /* per-row kept count is k_lo or k_lo + 1 (Bresenham) */
    double frac;          /* fractional budget spread by the Bresenham pattern */
    double row_budget;    /* the fractional per-row budget before the split */
} veda_block_desc;

typedef struct {
    int64_t seq_len;      /* packed rows S */
    int64_t n_slots;      /* N = 128 * n_tiles */
    int32_t n_video;      /* span tiles (references first, then the target) */
    int32_t n_ref;        /* reference tiles (0 when references are untiled) */
    int32_t n_global;     /* tiles of the uncovered ("global") rows, after the span tiles */
    int32_t n_tiles;      /* n_video + n_global */
    int32_t n_kv_ok;      /* tiles holding at least one real row */
    int32_t n_global_ok;  /* non-empty global tiles */
    int32_t max_kept;     /* width of one kept-list row (an upper bound on any video row's count) */
    int32_t tile_refs;    /* 1 when reference spans are tiled, 0 when their rows are global */
    int64_t ref_tokens, target_tokens;
    int32_t target_box[3];
    int32_t n_blocks;     /* 1 (target) or 2 (references, target) */
    veda_block_desc blocks[2];
} veda_layout_desc;

/* Row ranges of a model's packed sequence and their kinds (veda_core.py, "what the packed layout holds",
 * describe_layout: one generated video segment, reference segments of kind cond or ref_img, and others). */
enum { VEDA_SEG_OTHER = 0, VEDA_SEG_VIDEO = 1, VEDA_SEG_COND = 2, VEDA_SEG_REF_IMG = 3 };
typedef struct {
    int64_t start, stop;  /* packed rows [start, stop) */
    int32_t kind;         /* VEDA_SEG_* */
} veda_segment;

#define VEDA_MAX_PACKED_REFS 64

/* What a packed sequence holds, in the terms veda_plan takes. */
typedef struct {
    int64_t seq_len;
    int64_t target_start;                       /* the video segment's first row */
    int32_t target_grid[3];                     /* (lt, lh / 2, lw / 2) */
    int32_t n_refs;                             /* reference segments whose rows are a verified grid */
    int64_t ref_start[VEDA_MAX_PACKED_REFS];
    int32_t ref_grid[VEDA_MAX_PACKED_REFS][3];
    int32_t n_skipped;                          /* cond / ref_img segments left as global rows */
    int32_t skipped[VEDA_MAX_PACKED_REFS];      /* their indices in the segment array */
} veda_packed_desc;

/* ------------------------------------------------------------------------------------------ host */

/* Builds the tile layout of one head group (veda_core.py, "tiles", build_layout and span_tiles;
 * "one layer", attention: references are tiled at their least-padding box unless the reference
 * budget keeps all, in which case their rows become global rows).
 *  spans   host [n_spans]: references in packed order, then the target span (last). The target's box is
 *          the head group's box; a reference box of zero means least-padding (any other is honoured).
 *  seq_len packed rows S; every row no (tiled) span covers is a global row.
 *  generated / reference: budgets of the target block and of the reference block.
 *  out     receives the new layout. Device copies of its index data are made on first device use,
 *          once per device.
 * Errors: VEDA_ERR_INVALID for no spans, spans out of packed order or overlapping or running past
 * seq_len, a box that is not a power-of-two (t,h,w) with t*h*w = 128, and a budget with neither or
 * both kinds set, a negative ratio or a tile count below 0. */
int veda_plan(const veda_span* spans, int32_t n_spans, int64_t seq_len, veda_budget generated,
              veda_budget reference, veda_layout** out);

/* The layout's tiles as TMA boxes of the packed tensors, the form veda_attend_direct reads (host). A span
 * tile is the (st, sh, sw) box of its span's grid at its origin, positions in box order (t, h, w
 * row-major) with padding left in place; a global tile is the run of 128 rows from its first row.
 *  box_perm    [n_slots] int32: packed row of each box position, -1 where the tile has no row
 *  tile_coord  [n_tiles * 4] int32: span tile {span, w0, h0, t0} (span = index among the tiled spans in
 *              tile order); global tile {-1, first row, 0, 0}
 *  tile_mask   [n_tiles * 4] int32 bit patterns: bit c % 32 of word c / 32 set iff box position c holds
 *              a row of the tile
 * Any pointer may be NULL. Returns VEDA_ERR_UNSUPPORTED (and copies nothing) when the gathered path is
 * the only one for this layout: a global tile whose rows are not consecutive, or more than 4 tiled spans. */
int veda_layout_export_direct(const veda_layout* layout, int32_t* box_perm, int32_t* tile_coord, int32_t* tile_mask);

/* Sizes and budget split of a layout (host). */
int veda_layout_info(const veda_layout* layout, veda_layout_desc* out);

/* Copies the layout's index data to host arrays; any pointer may be NULL.
 *  perm         [n_slots] int32: packed row of each tile slot, -1 on padding (veda_core.py, build_layout)
 *  valid_count  [n_tiles] int32: real rows per tile (a prefix of the tile)
 *  allowed      [n_blocks * n_video] int32: per block, the kept count k_lo + extra(row) of every video
 *               query row (veda_core.py, "selection", select with _bresenham); n_block_cols for a
 *               keeps-all block. */
int veda_layout_export(const veda_layout* layout, int32_t* perm, int32_t* valid_count, int32_t* allowed);

/* Frees a layout and its device copies (on every device that used it). NULL is ignored. */
void veda_layout_destroy(veda_layout* layout);

/* The least-padding box of a grid (veda_core.py, "tiles", least_padding_shape): among the power-of-two
 * boxes that fit the grid (all 36 if none fits), fewest tiles, then most cubic, then lexicographic. */
int veda_least_padding_box(int32_t t, int32_t h, int32_t w, int32_t box_out[3]);

/* Whether packed rows [a, b) hold a row-major T x H x W grid of positions (veda_core.py, "what the packed
 * layout holds", _grid_of): the distinct values of each position column are the axes; their sizes must
 * multiply to b - a and the rows must list the axes' Cartesian product in row-major order (t slowest,
 * w fastest, each axis ascending).
 *  position_ids  host double [>= b, 3]: (t, h, w) position of every packed row, row-major.
 *  grid_out      receives (T, H, W) when *is_grid is set to 1; *is_grid is 0 otherwise.
 * Errors: VEDA_ERR_INVALID for NULL pointers or a < 0, b < a. */
int veda_grid_of(const double* position_ids, int64_t a, int64_t b, int32_t grid_out[3], int32_t* is_grid);

/* The spans a model's packed sequence holds (veda_core.py, "what the packed layout holds",
 * describe_layout), ready for veda_plan: the one video segment is the target, with grid
 * (lt, lh / 2, lw / 2) (two-by-two spatial patches of the latent grid); a cond or ref_img segment is a
 * reference span when its rows are a verified row-major grid (veda_grid_of on the position ids) and stays
 * global otherwise (always correct); segments of other kinds stay global.
 *  segments      host [n_segments]; position_ids host double [seq_len, 3], or NULL (no reference can be
 *                verified: every cond / ref_img segment stays global).
 *  latent        (lt, lh, lw).
 * Errors: VEDA_ERR_INVALID for NULL segments or out, a segment outside [0, seq_len), no video segment or
 * more than one, or a video segment whose row count is not lt * (lh / 2) * (lw / 2);
 * VEDA_ERR_UNSUPPORTED for more than VEDA_MAX_PACKED_REFS reference segments. */
int veda_describe_packed_layout(const veda_segment* segments, int32_t n_segments, int64_t seq_len,
                                const int32_t latent[3], const double* position_ids, veda_packed_desc* out);

/* ---------------------------------------------------------------------------------------- device */

/* Tile-order gather with the pooled features fused in (veda_core.py, "tiles", gather; "predictor", pool).
 *  x          device bf16 [S, H_total, D] with element strides x_strides[3] (S, H, D).
 *  heads      device int32 [n_heads]: which of the H_total heads form this group (any order).
 *  x_t        device bf16 [n_heads, N, D] out: x_t[h, i] = x[perm[i], heads[h]], zero on padding.
 *  feats      device fp32 [n_heads, n_video, 3D] out, or NULL to skip pooling: per video tile and head
 *             [mean | max | min] over the tile's real rows (0 for an empty tile); mean = fp32 sum / count.
 *  row_sq     device fp32 [n_heads, S] out, or NULL: ||x||^2 of every real row, at its packed row (the
 *             attend's logit bound takes it for Q; rows no tile holds are left as they were).
 *  max_sq     device fp32 [n_heads] out, or NULL: the largest ||x||^2 over the head's real rows (the
 *             attend's logit bound takes it for K); zeroed by the call before the kernel raises it.
 * D must be 64 or 128. */
int veda_gather(const veda_layout* layout, const void* x, const int64_t x_strides[3], int32_t h_total,
                int32_t dim, const int32_t* heads, int32_t n_heads, void* x_t, float* feats, float* row_sq,
                float* max_sq, void* stream);

/* The pooled features of veda_gather without the tile-order copy (veda_core.py, "predictor", pool): per
 * video tile and head [mean | max | min] over the tile's real rows, mean = fp32 sum / count, 0 for an
 * empty tile; the same values veda_gather writes to its feats.
 *  x      device bf16 [S, H_total, D] with element strides x_strides[3] (S, H, D).
 *  heads  device int32 [n_heads].
 *  feats  device fp32 [n_heads, n_video, 3D] out.
 *  row_sq, max_sq  optional norm outputs, as for veda_gather (when either is given, the call reads the
 *         global tiles' rows too).
 * D must be 64 or 128. With veda_attend_direct this is all the scoring path needs of Q and K. */
int veda_pool(const veda_layout* layout, const void* x, const int64_t x_strides[3], int32_t h_total,
              int32_t dim, const int32_t* heads, int32_t n_heads, float* feats, float* row_sq, float* max_sq,
              void* stream);

/* Workspace bytes veda_score needs (projected features of Q and K, and both projections transposed):
 * n_heads * (2 * n_video * D + 6 * D * D) * 4. */
size_t veda_score_workspace_bytes(const veda_layout* layout, int32_t n_heads, int32_t dim);

/* Tile-pair logits (veda_core.py, "predictor", logits): per head, q_hat = fq @ Pq + fq[:, :D],
 * k_hat = fk @ Pk + fk[:, :D], scores = q_hat @ k_hat^T / sqrt(D), all fp32 (on the tensor cores as split tf32:
 * each operand as a tf32 high part and its fp32 remainder, three tf32 products per product, which keeps the
 * error at the level of fp32 rounding).
 *  feats_q/k  device fp32 [n_heads, n_video, 3D] (from veda_gather).
 *  proj_q/k   device fp32 [n_heads, 3D, D]: the group's heads' projections, in the group's head order.
 *  workspace  device, at least veda_score_workspace_bytes(), 16-byte aligned; caller-owned scratch (the
 *             projected features and the transposed projections), overwritten by every call.
 *  scores     device fp32 [n_heads, n_video, n_video] out.
 * Errors: VEDA_ERR_INVALID for NULL or unaligned buffers, a workspace below the size, D other than 64 or
 * 128 or n_heads <= 0; VEDA_ERR_CUDA when a launch or a tensor-map encoding fails. The kernels' waits are
 * bounded: one that expires stops the kernel early and veda_sync_status reports VEDA_ERR_TIMEOUT. */
int veda_score(const veda_layout* layout, const float* feats_q, const float* feats_k, int32_t n_heads,
               int32_t dim, const float* proj_q, const float* proj_k, void* workspace,
               size_t workspace_bytes, float* scores, void* stream);

/* veda_score without a workspace argument, for callers that cannot allocate device memory when they
 * need the scores: plugins whose device memory belongs to a pool the host application owns and budgets,
 * and real-time loops where an allocation, which can block on or synchronise with the device, is not
 * allowed. The pages have no counterpart: this is a service of this library.
 * Same inputs, outputs and arithmetic as veda_score; the projected features (and the transposed
 * projections) live in one 4 MiB array of
 * this library's device memory (1,048,576 floats, held by every GPU that loads the library until exit)
 * and heads are processed in chunks that fit it. Nothing is allocated and nothing needs to start at zero.
 * The first call on a device looks up the array's device address and keeps it for the process's life
 * (make that call before any stream capture; after cudaDeviceReset the kept address is stale, so do not
 * call this entry point again in that process).
 * All calls on a device share the array: calls whose kernels overlap on the GPU race and must be
 * serialised. Errors: VEDA_ERR_UNSUPPORTED when one head needs more than the array holds
 * (2 * n_video * D + 6 * D * D > 1,048,576, i.e. n_video > 3712 at D = 128); otherwise as veda_score. */
int veda_score_noalloc(const veda_layout* layout, const float* feats_q, const float* feats_k, int32_t n_heads,
                       int32_t dim, const float* proj_q, const float* proj_k, float* scores, void* stream);

/* Head-aware top-k (veda_core.py, "selection", select, block_mask and tile_index_list).
 * Per head and video query row, per column block: empty key tiles are never kept; the row's own tile
 * is kept first when it lies in the block; the other columns are ranked by (score descending, column
 * ascending) and the first k_lo + extra(row) are kept (all non-empty columns for a keeps-all block).
 * A NaN or -inf score is never kept. Every non-empty global tile is appended.
 *  scores     device fp32 [n_heads, n_video, n_video] (any source).
 *  kept_idx   device int32 [n_heads, n_video, max_kept] out: ascending tile ids; entries past the count
 *             are left untouched.
 *  kept_cnt   device int32 [n_heads, n_video] out.
 * Global query rows are dense over every non-empty tile and need no list.
 * Limit: a column block of at most 16384 tiles (VEDA_ERR_UNSUPPORTED beyond). */
int veda_select(const veda_layout* layout, const float* scores, int32_t n_heads, int32_t* kept_idx,
                int32_t* kept_cnt, void* stream);

/* Block-sparse flash attention over the kept tiles, scattered back to packed rows (veda_core.py,
 * "selection", reference_attend: scale D^-0.5, key slots restricted to real rows, a row that sees no
 * key gives 0; "tiles", scatter_).
 *  q_t, k_t, v_t  device bf16 [n_heads, N, D] tile order (from veda_gather).
 *  kept_idx/cnt   as written by veda_select (or any lists in that format: ids ascending in
 *                 [0, n_tiles), count <= max_kept; a malformed row is cut at its first bad entry and
 *                 latched as VEDA_ERR_BAD_LIST).
 *  out            device bf16 [S, H_total, D] with element strides out_strides[3]: rows of this group's
 *                 heads (heads[h]) are overwritten; padding slots are dropped.
 *  q_row_sq   device fp32 [n_heads, S] (row_sq of veda_gather/veda_pool on Q) and
 *  k_max_sq   device fp32 [n_heads] (max_sq of veda_gather/veda_pool on K), or both NULL: a bound on every
 *             logit of a row, sqrt(||q||^2 max ||k||^2) (Cauchy-Schwarz). Where a softmax group's first
 *             tile leaves every row of a warp within 2^48 of that bound, its later tiles skip the row max
 *             and the rescale of the accumulator; the result is the same softmax (the common scale of
 *             P, O and the row sum differs, and fp32 holds it: V entries up to 2^60 in magnitude).
 *             With NULL every tile takes its exact row max.
 * D must be 64 or 128. Runs bf16 tensor-core MMAs (tcgen05) with fp32 accumulation and an fp32 online
 * softmax; needs an sm_100 device. */
int veda_attend(const veda_layout* layout, const void* q_t, const void* k_t, const void* v_t,
                int32_t n_heads, int32_t dim, const int32_t* kept_idx, const int32_t* kept_cnt,
                void* out, const int64_t out_strides[3], int32_t h_total, const int32_t* heads,
                const float* q_row_sq, const float* k_max_sq, void* stream);

/* veda_attend reading the packed tensors directly, with no tile-order copies (gather-free): every tile
 * is loaded as a TMA box of q, k and v (veda_layout_export_direct gives the boxes). Same operation as
 * veda_attend on the same lists; the keys of a partial span tile come in box order, so its sums run in
 * another order (within rounding of veda_attend's).
 *  q, k, v    device bf16 [S, H_total, D] with element strides q/k/v_strides[3] (S, H, D); bases 16-byte
 *             aligned, S and H strides multiples of 8 elements.
 *  heads      device int32 [n_heads]: the group's heads among the H_total.
 *  kept_idx/cnt, out, out_strides, q_row_sq, k_max_sq: as for veda_attend (the norms from veda_pool).
 * D must be 64 or 128. VEDA_ERR_UNSUPPORTED when the layout has no box form (see
 * veda_layout_export_direct); veda_gather + veda_attend take every layout. */
int veda_attend_direct(const veda_layout* layout, const void* q, const int64_t q_strides[3], const void* k,
                       const int64_t k_strides[3], const void* v, const int64_t v_strides[3], int32_t h_total,
                       int32_t dim, const int32_t* heads, int32_t n_heads, const int32_t* kept_idx,
                       const int32_t* kept_cnt, void* out, const int64_t out_strides[3], const float* q_row_sq,
                       const float* k_max_sq, void* stream);

/* Paired attend: the same operation as veda_attend / veda_attend_direct on the same lists (veda_core.py,
 * "selection", reference_attend, then "tiles", scatter_), computed two neighbouring query tiles at a time.
 * Video query tiles 2p and 2p + 1 of a head (and global query tiles likewise) share one CTA, which loads
 * each key tile of the union of their two kept lists once for both, so neighbouring tiles that keep the
 * same key tiles read them from L2 once instead of twice. Each query row takes its softmax reference
 * from the logit bound, m = sqrt(q_row_sq * k_max_sq) D^-0.5 log2(e) - 64 (log2 units, so every 2^(s - m)
 * is at most 2^64); no row max is taken and both softmax halves add into one accumulator per query tile.
 * A real row whose sum of 2^(s - m) ends outside [2^-60, 2^100] (the bound loose by more than 124 log2
 * units, or not finite) flags its query tile, and a second launch of veda_attend's kernel recomputes
 * every row of the flagged tiles with the exact per-tile maxima. Results agree with veda_attend within
 * rounding (sums run in another order).
 *  q_row_sq, k_max_sq  required (device fp32, from veda_pool or veda_gather of the same Q and K).
 *  workspace, workspace_bytes  device buffer of at least veda_attend_paired_workspace_bytes(layout,
 *             n_heads) bytes, 256-byte aligned, owned by the caller; overwritten by the call (the merged
 *             lists and the redo flags) and free for other use once the call's kernels have finished on
 *             `stream`.
 * Other arguments, limits and errors as veda_attend / veda_attend_direct (a malformed kept list is cut at
 * its first bad entry and veda_sync_status reports VEDA_ERR_BAD_LIST); VEDA_ERR_INVALID also for NULL
 * norms or a NULL, unaligned or too small workspace. */
size_t veda_attend_paired_workspace_bytes(const veda_layout* layout, int32_t n_heads);
int veda_attend_paired(const veda_layout* layout, const void* q_t, const void* k_t, const void* v_t,
                       int32_t n_heads, int32_t dim, const int32_t* kept_idx, const int32_t* kept_cnt, void* out,
                       const int64_t out_strides[3], int32_t h_total, const int32_t* heads, const float* q_row_sq,
                       const float* k_max_sq, void* workspace, size_t workspace_bytes, void* stream);
int veda_attend_direct_paired(const veda_layout* layout, const void* q, const int64_t q_strides[3], const void* k,
                              const int64_t k_strides[3], const void* v, const int64_t v_strides[3], int32_t h_total,
                              int32_t dim, const int32_t* heads, int32_t n_heads, const int32_t* kept_idx,
                              const int32_t* kept_cnt, void* out, const int64_t out_strides[3],
                              const float* q_row_sq, const float* k_max_sq, void* workspace, size_t workspace_bytes,
                              void* stream);

/* FP8 Q/K variant, step 1 (not on the pages: their kernel quantises to INT8 by a recipe they do not
 * print; this follows the FP8 e4m3 variant of the 104k budget sweep). Per (head, 128-row tile) of a
 * tile-ordered bf16 tensor: scale = amax(|x|) over the tile's real rows / 448 (1 when 0), and each code is
 * x / scale rounded to nearest-even e4m3 with saturation at +-448 (padding rows stay 0).
 *  x_t     device bf16 [n_heads, N, D] (from veda_gather).
 *  codes   device e4m3 bytes [n_heads, N, D] out.
 *  scales  device fp32 [n_heads, n_tiles] out.
 * D must be 64 or 128. */
int veda_quantize_fp8(const veda_layout* layout, const void* x_t, int32_t n_heads, int32_t dim, void* codes,
                      float* scales, void* stream);

/* FP8 Q/K variant, steps 0 and 1 in one pass: veda_gather with the tile written as e4m3 codes and its
 * per-tile scale (the quantisation of veda_quantize_fp8, bit for bit) instead of bf16, so the bf16 tile
 * copy is never written or read back.
 *  x, x_strides, h_total, heads, feats, row_sq, max_sq  as veda_gather (feats, row_sq and max_sq may be
 *          NULL; the norms are those of the bf16 input, for the paired attend's logit bound).
 *  codes   device e4m3 bytes [n_heads, N, D] out (padding slots 0).
 *  scales  device fp32 [n_heads, n_tiles] out.
 * D must be 64 or 128. Errors as veda_gather. */
int veda_gather_fp8(const veda_layout* layout, const void* x, const int64_t x_strides[3], int32_t h_total,
                    int32_t dim, const int32_t* heads, int32_t n_heads, void* codes, float* scales, float* feats,
                    float* row_sq, float* max_sq, void* stream);

/* FP8 Q/K variant, step 2: veda_attend with Q and K given as e4m3 codes and per-tile scales (from
 * veda_quantize_fp8); S = Q K^T runs as an e4m3 x e4m3 tensor-core product with fp32 accumulation and is
 * multiplied by scale_q(query tile) * scale_k(key tile) * D^-0.5; P and V stay bf16. Selection is not
 * affected (it pools the bf16 Q and K). D must be 128. Other arguments and errors as veda_attend. */
int veda_attend_fp8(const veda_layout* layout, const void* q_codes, const void* k_codes, const float* scales_q,
                    const float* scales_k, const void* v_t, int32_t n_heads, int32_t dim, const int32_t* kept_idx,
                    const int32_t* kept_cnt, void* out, const int64_t out_strides[3], int32_t h_total,
                    const int32_t* heads, void* stream);

/* INT8 Q/K variant. The pages' own kernel computes Q K^T in INT8 (a SageAttention-derived kernel;
 * veda_core.py and the Vflash guide) but does not print its quantisation recipe; this library's reading
 * is the symmetric per-tile one: per (head, 128-row tile) scale = amax(|x|) over the tile's real rows / 127
 * (1 when 0), stored as fp32; each code is x / scale rounded to the nearest integer, ties to even, within
 * +-127 (padding rows stay 0). S = Q K^T runs as an s8 x s8 tensor-core product with exact int32
 * accumulation and is multiplied by scale_q(query tile) * scale_k(key tile) * D^-0.5; P and V stay bf16.
 * Selection is not affected (it pools the bf16 Q and K).
 *
 * veda_gather_int8: veda_gather with the tile written as int8 codes and its scale (arguments as
 *   veda_gather_fp8; codes are int8 bytes [n_heads, N, D]). D must be 64 or 128.
 * veda_quantize_int8: the same codes from tile-ordered bf16 (arguments as veda_quantize_fp8).
 * veda_attend_int8: veda_attend on int8 codes and scales (arguments as veda_attend_fp8). D must be 128. */
int veda_gather_int8(const veda_layout* layout, const void* x, const int64_t x_strides[3], int32_t h_total,
                     int32_t dim, const int32_t* heads, int32_t n_heads, void* codes, float* scales, float* feats,
                     float* row_sq, float* max_sq, void* stream);
int veda_quantize_int8(const veda_layout* layout, const void* x_t, int32_t n_heads, int32_t dim, void* codes,
                       float* scales, void* stream);
int veda_attend_int8(const veda_layout* layout, const void* q_codes, const void* k_codes, const float* scales_q,
                     const float* scales_k, const void* v_t, int32_t n_heads, int32_t dim, const int32_t* kept_idx,
                     const int32_t* kept_cnt, void* out, const int64_t out_strides[3], int32_t h_total,
                     const int32_t* heads, void* stream);

/* The paired attend (see veda_attend_paired) on 8-bit Q/K codes: veda_attend_fp8 / veda_attend_int8's
 * operation, two neighbouring query tiles per work item sharing each kept K/V tile load. Each row's softmax
 * reference comes from the logit bound of the bf16 inputs (q_row_sq and k_max_sq from veda_gather_fp8 /
 * veda_gather_int8 or veda_pool): the codes' logits differ from the bf16 ones only by the quantisation
 * error, far inside the reference's 2^64 headroom, and a query tile the bound cannot serve is recomputed by
 * veda_attend_fp8 / veda_attend_int8's kernel. Arguments as veda_attend_fp8 plus q_row_sq, k_max_sq,
 * workspace and workspace_bytes as veda_attend_paired. D must be 128. */
int veda_attend_fp8_paired(const veda_layout* layout, const void* q_codes, const void* k_codes,
                           const float* scales_q, const float* scales_k, const void* v_t, int32_t n_heads,
                           int32_t dim, const int32_t* kept_idx, const int32_t* kept_cnt, void* out,
                           const int64_t out_strides[3], int32_t h_total, const int32_t* heads, const float* q_row_sq,
                           const float* k_max_sq, void* workspace, size_t workspace_bytes, void* stream);
int veda_attend_int8_paired(const veda_layout* layout, const void* q_codes, const void* k_codes,
                            const float* scales_q, const float* scales_k, const void* v_t, int32_t n_heads,
                            int32_t dim, const int32_t* kept_idx, const int32_t* kept_cnt, void* out,
                            const int64_t out_strides[3], int32_t h_total, const int32_t* heads, const float* q_row_sq,
                            const float* k_max_sq, void* workspace, size_t workspace_bytes, void* stream);

/* Synchronizes `stream`, then reads and clears this device's latched kernel error word.
 * Returns VEDA_OK, VEDA_ERR_TIMEOUT, VEDA_ERR_BAD_LIST or VEDA_ERR_CUDA. */
int veda_sync_status(void* stream);

/* Text of the calling thread's last error ("" if none). Valid until the thread's next veda_* call. */
const char* veda_last_error(void);

/* VEDA_OK when the current device is sm_100 (B200 class), else VEDA_ERR_UNSUPPORTED / VEDA_ERR_CUDA. */
int veda_device_check(void);

/* Upper bound, in nanoseconds, of every bounded device-side wait (default 1e9). Process-wide. */
void veda_set_wait_timeout_ns(uint64_t ns);

/* Test hook for the failure path (the pages have no counterpart): the calling thread's next veda_attend
 * (any variant; the paired ones' first kernel) withholds its Q tile loads, so the kernel's waits on them expire; the kernel then lets its in-flight
 * copies and MMAs finish, frees its tensor memory and returns, and veda_sync_status reports
 * VEDA_ERR_TIMEOUT. The output of that call is unspecified; the device stays usable. */
void veda_debug_hold_next_attend(void);

/* Test hook (the pages have no counterpart): caps the number of CTAs of the calling thread's attend
 * launches (every variant, and both kernels of the paired ones) at n, so that each CTA of a small case
 * walks many work items in a row, as on a full-size layer; n <= 0 removes the cap. Results do not
 * depend on it. */
void veda_debug_attend_ctas(int32_t n);

/* Test hook for the attend kernel's exponentials (the pages have no counterpart): evaluates, for each of
 * n fp32 inputs x, the three forms of 2^x the library has on the device: the FMA-pipe polynomial the
 * attend softmax uses for part of its columns (Cody-Waite reduction plus a cubic; inputs below -126 are
 * taken as -126), the MUFU approximation (ex2.approx.ftz) it uses for the rest, and CUDA's exp2f.
 *  x        device fp32 [n] in.
 *  poly, mufu, exp2f_out  device fp32 [n] out (any may be NULL to skip it).
 * Errors: VEDA_ERR_INVALID for a NULL x or negative n. */
int veda_debug_exp2(const float* x, float* poly, float* mufu, float* exp2f_out, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* VEDA_H */
