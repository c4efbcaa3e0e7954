// Host planner of the Veda tile-skip path: tile boxes, span tiling, the layout permutation and the
// per-row budgets. Follows the page "veda_core.py" (ComfyUI-FunPack), sections "budgets" and "tiles",
// and the reference handling of its "one layer" section. Build with -ffp-contract=off: the budget
// arithmetic must round exactly like the page's IEEE double expressions.
#include <algorithm>
#include <array>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <string>
#include <tuple>
#include <vector>

#include "veda_internal.h"

namespace {

using Box = std::array<int32_t, 3>;

// All power-of-two (t, h, w) with t*h*w = 128, ascending lexicographically (36 boxes).
std::vector<Box> all_boxes() {
    std::vector<Box> out;
    for (int a = 0; a < 8; ++a)
        for (int b = 0; a + b < 8; ++b) out.push_back({1 << a, 1 << b, 128 >> (a + b)});
    std::sort(out.begin(), out.end());
    return out;
}

bool is_box(const Box& s) {
    for (int v : s)
        if (v <= 0 || (v & (v - 1)) != 0) return false;
    return int64_t(s[0]) * s[1] * s[2] == veda::kTile;
}

int64_t round_up(int64_t g, int64_t s) { return (g + s - 1) / s * s; }

int64_t boxes_in(const Box& grid, const Box& s) {
    return round_up(grid[0], s[0]) * round_up(grid[1], s[1]) * round_up(grid[2], s[2]) / veda::kTile;
}

// veda_core.py, "tiles", least_padding_shape: fewest tiles, then smallest max/min edge ratio (a
// double), then the lexicographically first box; only boxes that fit the grid compete unless none does.
Box least_padding(const Box& grid) {
    std::vector<Box> every = all_boxes(), fit;
    for (const Box& s : every)
        if (s[0] <= grid[0] && s[1] <= grid[1] && s[2] <= grid[2]) fit.push_back(s);
    const std::vector<Box>& cand = fit.empty() ? every : fit;
    Box best = cand[0];
    auto key = [&](const Box& s) {
        double lo = std::min({s[0], s[1], s[2]}), hi = std::max({s[0], s[1], s[2]});
        return std::make_tuple(boxes_in(grid, s), hi / lo, s);
    };
    for (const Box& s : cand)
        if (key(s) < key(best)) best = s;
    return best;
}

// veda_core.py, "tiles", span_tiles: boxes visited h-box outermost, then w-box, then t-box; inside a
// box cells run t, h, w row-major; real rows first (stable), padding (-1) after.
void tile_span(int64_t start, const Box& grid, const Box& box, std::vector<int32_t>& perm) {
    const int64_t T = grid[0], H = grid[1], W = grid[2];
    const int64_t nt = round_up(T, box[0]) / box[0];
    const int64_t nh = round_up(H, box[1]) / box[1];
    const int64_t nw = round_up(W, box[2]) / box[2];
    int32_t slot[veda::kTile];
    for (int64_t bh = 0; bh < nh; ++bh)
        for (int64_t bw = 0; bw < nw; ++bw)
            for (int64_t bt = 0; bt < nt; ++bt) {
                int n = 0;
                for (int dt = 0; dt < box[0]; ++dt)
                    for (int dh = 0; dh < box[1]; ++dh)
                        for (int dw = 0; dw < box[2]; ++dw) {
                            int64_t t = bt * box[0] + dt, h = bh * box[1] + dh, w = bw * box[2] + dw;
                            if (t < T && h < H && w < W) slot[n++] = int32_t(start + (t * H + h) * W + w);
                        }
                for (int i = 0; i < n; ++i) perm.push_back(slot[i]);
                for (int i = n; i < veda::kTile; ++i) perm.push_back(-1);
            }
}

// The same boxes in the same order as tile_span, as TMA boxes of the packed tensor: box_perm holds the
// packed row of every box position (t, h, w row-major inside the box) and -1 outside the grid, and
// tile_coord the box origin {span, w0, h0, t0}.
void span_boxes(int64_t start, const Box& grid, const Box& box, int32_t span, std::vector<int32_t>& box_perm,
                std::vector<int32_t>& tile_coord) {
    const int64_t T = grid[0], H = grid[1], W = grid[2];
    const int64_t nt = round_up(T, box[0]) / box[0];
    const int64_t nh = round_up(H, box[1]) / box[1];
    const int64_t nw = round_up(W, box[2]) / box[2];
    for (int64_t bh = 0; bh < nh; ++bh)
        for (int64_t bw = 0; bw < nw; ++bw)
            for (int64_t bt = 0; bt < nt; ++bt) {
                tile_coord.insert(tile_coord.end(),
                                  {span, int32_t(bw * box[2]), int32_t(bh * box[1]), int32_t(bt * box[0])});
                for (int dt = 0; dt < box[0]; ++dt)
                    for (int dh = 0; dh < box[1]; ++dh)
                        for (int dw = 0; dw < box[2]; ++dw) {
                            int64_t t = bt * box[0] + dt, h = bh * box[1] + dh, w = bw * box[2] + dw;
                            box_perm.push_back(t < T && h < H && w < W ? int32_t(start + (t * H + h) * W + w) : -1);
                        }
            }
}

bool budget_ok(const veda_budget& b) {
    if (b.kind == VEDA_BUDGET_RATIO) return std::isfinite(b.ratio) && b.ratio >= 0.0;
    if (b.kind == VEDA_BUDGET_TILES) return b.tiles >= 0;
    return false;
}

// veda_core.py, "budgets", keeps_all: a ratio of at least one and no tile count.
bool keeps_everything(const veda_budget& b) { return b.kind == VEDA_BUDGET_RATIO && b.ratio >= 1.0; }

// veda_core.py, "budgets", _per_row: tiles as a double, or ((ratio * ideal) * ideal) / n_cols with
// ideal = ceil(real / 128); each product rounded to double in that order.
double per_row_budget(const veda_budget& b, int64_t real_tokens, int64_t n_cols) {
    if (b.kind == VEDA_BUDGET_TILES) return double(b.tiles);
    volatile double ideal = double((real_tokens + veda::kTile - 1) / veda::kTile);
    volatile double v = b.ratio * ideal;
    v = v * ideal;
    v = v / double(n_cols);
    return v;
}

// Python's round(x, 12) for x in [0, 1]: the correctly rounded 12-decimal string, parsed back.
double round12(double x) {
    char buf[64];
    std::snprintf(buf, sizeof buf, "%.12f", x);
    return std::strtod(buf, nullptr);
}

// veda_core.py, "budgets", _split.
void split(double b, int64_t n, veda_block_desc& out) {
    out.row_budget = b;
    if (b >= double(n)) {
        out.k_lo = out.k_hi = int32_t(n);
        out.frac = 0.0;
        return;
    }
    int64_t lo = int64_t(std::floor(b));
    lo = std::min<int64_t>(std::max<int64_t>(1, lo), n);
    out.k_lo = int32_t(lo);
    out.k_hi = int32_t(std::min<int64_t>(lo + 1, n));
    double f = b - double(lo);
    f = std::min(std::max(f, 0.0), 1.0);
    out.frac = round12(f);
}

}  // namespace

extern "C" int veda_least_padding_box(int32_t t, int32_t h, int32_t w, int32_t box_out[3]) {
    veda::clear_error();
    if (t <= 0 || h <= 0 || w <= 0 || !box_out) return veda::fail(VEDA_ERR_INVALID, "grid axes must be positive");
    Box b = least_padding({t, h, w});
    for (int i = 0; i < 3; ++i) box_out[i] = b[i];
    return VEDA_OK;
}

extern "C" int veda_plan(const veda_span* spans, int32_t n_spans, int64_t seq_len, veda_budget generated,
                         veda_budget reference, veda_layout** out) {
    veda::clear_error();
    if (!out) return veda::fail(VEDA_ERR_INVALID, "veda_plan: out is NULL");
    *out = nullptr;
    if (!spans || n_spans <= 0) return veda::fail(VEDA_ERR_INVALID, "the target span must be tiled");
    if (seq_len <= 0 || seq_len > INT32_MAX) return veda::fail(VEDA_ERR_INVALID, "seq_len must be in [1, 2^31)");
    if (!budget_ok(generated) || !budget_ok(reference))
        return veda::fail(VEDA_ERR_INVALID,
                          "a budget sets exactly one of ratio (>= 0) and tiles (>= 0)");

    // references are tiled unless their budget keeps everything ("one layer": tile_refs)
    const bool tile_refs = !keeps_everything(reference);
    struct S { int64_t start; Box grid, box; };
    std::vector<S> use;
    int64_t end = 0;
    for (int32_t i = 0; i < n_spans; ++i) {
        const veda_span& sp = spans[i];
        Box grid{sp.t, sp.h, sp.w}, box{sp.st, sp.sh, sp.sw};
        if (grid[0] <= 0 || grid[1] <= 0 || grid[2] <= 0)
            return veda::fail(VEDA_ERR_INVALID, "span " + std::to_string(i) + ": grid axes must be positive");
        const bool target = i == n_spans - 1;
        if (box[0] == 0 && box[1] == 0 && box[2] == 0) box = least_padding(grid);
        if (!is_box(box))
            return veda::fail(VEDA_ERR_INVALID, "span " + std::to_string(i) +
                                                    ": box must be power-of-two (t,h,w) with t*h*w = 128");
        const int64_t rows = int64_t(grid[0]) * grid[1] * grid[2];
        if (sp.start < end || sp.start + rows > seq_len)
            return veda::fail(VEDA_ERR_INVALID, "span at " + std::to_string(sp.start) +
                                                    " overlaps another or runs past " + std::to_string(seq_len));
        end = sp.start + rows;
        if (target || tile_refs) use.push_back({sp.start, grid, box});
    }

    auto lay = new veda_layout();
    veda_layout_desc& d = lay->desc;
    std::vector<int32_t>& perm = lay->perm;
    std::vector<char> covered(size_t(seq_len), 0);
    int64_t ref_tiles = 0, ref_tokens = 0;
    for (size_t i = 0; i < use.size(); ++i) {
        const S& s = use[i];
        const int64_t rows = int64_t(s.grid[0]) * s.grid[1] * s.grid[2];
        std::fill(covered.begin() + s.start, covered.begin() + s.start + rows, 1);
        const size_t before = perm.size();
        tile_span(s.start, s.grid, s.box, perm);
        span_boxes(s.start, s.grid, s.box, int32_t(i), lay->box_perm, lay->tile_coord);
        lay->spans.push_back({s.start, s.grid[0], s.grid[1], s.grid[2], s.box[0], s.box[1], s.box[2]});
        if (i + 1 < use.size()) {
            ref_tiles += int64_t(perm.size() - before) / veda::kTile;
            ref_tokens += rows;
        }
    }
    const int64_t n_video = int64_t(perm.size()) / veda::kTile;
    int64_t n_rest = 0;
    for (int64_t r = 0; r < seq_len; ++r)
        if (!covered[size_t(r)]) {
            perm.push_back(int32_t(r));
            ++n_rest;
        }
    const int64_t n_global = (n_rest + veda::kTile - 1) / veda::kTile;
    perm.resize(size_t((n_video + n_global) * veda::kTile), -1);
    const int64_t n_tiles = n_video + n_global;

    lay->valid_count.assign(size_t(n_tiles), 0);
    for (int64_t i = 0; i < n_tiles; ++i) {
        int32_t c = 0;
        for (int j = 0; j < veda::kTile; ++j) c += perm[size_t(i * veda::kTile + j)] >= 0;
        lay->valid_count[size_t(i)] = c;
        if (c > 0) lay->ok_list.push_back(int32_t(i));
    }

    // box form of the global tiles: a run of 128 rows from the tile's first row, its own rows a prefix
    lay->direct_ok = lay->spans.size() <= size_t(veda::kMaxDirectSpans);
    if (!lay->direct_ok)
        lay->direct_why = std::to_string(lay->spans.size()) + " tiled spans (the gather-free attend takes at most " +
                          std::to_string(veda::kMaxDirectSpans) + ")";
    for (int64_t i = n_video; i < n_tiles; ++i) {
        const int32_t* rows = perm.data() + i * veda::kTile;
        const int32_t c = lay->valid_count[size_t(i)];
        const bool run = c > 0 && rows[c - 1] - rows[0] == c - 1;
        if (!run && lay->direct_ok) {
            lay->direct_ok = false;
            lay->direct_why = "global tile " + std::to_string(i) + " is not a run of consecutive rows";
        }
        const int32_t row0 = c > 0 ? rows[0] : 0;
        lay->tile_coord.insert(lay->tile_coord.end(), {-1, row0, 0, 0});
        for (int j = 0; j < veda::kTile; ++j) lay->box_perm.push_back(run && j < c ? row0 + j : -1);
    }
    lay->tile_mask.assign(size_t(n_tiles) * 4, 0);
    for (int64_t i = 0; i < n_tiles; ++i)
        for (int j = 0; j < veda::kTile; ++j)
            if (lay->box_perm[size_t(i * veda::kTile + j)] >= 0)
                lay->tile_mask[size_t(i * 4 + j / 32)] |= int32_t(1u << (j % 32));

    d.seq_len = seq_len;
    d.n_slots = n_tiles * veda::kTile;
    d.n_video = int32_t(n_video);
    d.n_ref = int32_t(ref_tiles);
    d.n_global = int32_t(n_global);
    d.n_tiles = int32_t(n_tiles);
    d.n_kv_ok = int32_t(lay->ok_list.size());
    d.n_global_ok = 0;
    for (int64_t i = n_video; i < n_tiles; ++i) d.n_global_ok += lay->valid_count[size_t(i)] > 0;
    d.tile_refs = tile_refs ? 1 : 0;
    d.ref_tokens = ref_tokens;
    const S& tgt = use.back();
    d.target_tokens = int64_t(tgt.grid[0]) * tgt.grid[1] * tgt.grid[2];
    for (int i = 0; i < 3; ++i) d.target_box[i] = tgt.box[i];

    // column blocks ("selection", column_blocks): references then target, each with its own budget
    struct B { int64_t start, stop; veda_budget budget; int64_t real; };
    std::vector<B> blocks;
    if (d.n_ref > 0) blocks.push_back({0, d.n_ref, reference, d.ref_tokens});
    blocks.push_back({d.n_ref, d.n_video, generated, d.target_tokens});
    d.n_blocks = int32_t(blocks.size());
    lay->allowed.assign(size_t(d.n_blocks) * size_t(n_video), 0);
    int64_t max_kept = d.n_global_ok;
    for (size_t b = 0; b < blocks.size(); ++b) {
        veda_block_desc& bd = d.blocks[b];
        const B& blk = blocks[b];
        const int64_t n = blk.stop - blk.start;
        bd.start = int32_t(blk.start);
        bd.stop = int32_t(blk.stop);
        int32_t* allowed = lay->allowed.data() + b * size_t(n_video);
        if (keeps_everything(blk.budget)) {
            bd.keeps_all = 1;
            bd.k_lo = bd.k_hi = int32_t(n);
            bd.frac = 0.0;
            bd.row_budget = double(n);
            std::fill(allowed, allowed + n_video, int32_t(n));
            int64_t ok = 0;
            for (int64_t c = blk.start; c < blk.stop; ++c) ok += lay->valid_count[size_t(c)] > 0;
            max_kept += ok;
            continue;
        }
        bd.keeps_all = 0;
        split(per_row_budget(blk.budget, blk.real, n), n, bd);
        // "budgets", _bresenham over all n_video rows: row r gets one more tile when
        // floor((r + 1) * frac) > floor(r * frac), products in double
        int32_t widest = 0;
        for (int64_t r = 0; r < n_video; ++r) {
            volatile double a = double(r) * bd.frac, c = double(r + 1) * bd.frac;
            allowed[r] = bd.k_lo + (std::floor(c) > std::floor(a) ? 1 : 0);
            widest = std::max(widest, allowed[r]);
        }
        max_kept += widest;
    }
    d.max_kept = int32_t(std::max<int64_t>(max_kept, 1));
    *out = lay;
    return VEDA_OK;
}

extern "C" int veda_layout_info(const veda_layout* layout, veda_layout_desc* out) {
    veda::clear_error();
    if (!layout || !out) return veda::fail(VEDA_ERR_INVALID, "veda_layout_info: NULL argument");
    *out = layout->desc;
    return VEDA_OK;
}

extern "C" int veda_layout_export_direct(const veda_layout* layout, int32_t* box_perm, int32_t* tile_coord,
                                         int32_t* tile_mask) {
    veda::clear_error();
    if (!layout) return veda::fail(VEDA_ERR_INVALID, "veda_layout_export_direct: NULL layout");
    if (!layout->direct_ok)
        return veda::fail(VEDA_ERR_UNSUPPORTED, "the gather-free attend cannot take this layout: " + layout->direct_why);
    if (box_perm) std::copy(layout->box_perm.begin(), layout->box_perm.end(), box_perm);
    if (tile_coord) std::copy(layout->tile_coord.begin(), layout->tile_coord.end(), tile_coord);
    if (tile_mask) std::copy(layout->tile_mask.begin(), layout->tile_mask.end(), tile_mask);
    return VEDA_OK;
}

extern "C" int veda_layout_export(const veda_layout* layout, int32_t* perm, int32_t* valid_count,
                                  int32_t* allowed) {
    veda::clear_error();
    if (!layout) return veda::fail(VEDA_ERR_INVALID, "veda_layout_export: NULL layout");
    if (perm) std::copy(layout->perm.begin(), layout->perm.end(), perm);
    if (valid_count) std::copy(layout->valid_count.begin(), layout->valid_count.end(), valid_count);
    if (allowed) std::copy(layout->allowed.begin(), layout->allowed.end(), allowed);
    return VEDA_OK;
}

// veda_core.py, "what the packed layout holds", _grid_of: rows [a, b) are a row-major grid of the
// distinct values of their three position columns.
static bool grid_of(const double* pos, int64_t a, int64_t b, int32_t grid[3]) {
    std::vector<double> axis[3];
    for (int c = 0; c < 3; ++c) {
        axis[c].reserve(size_t(b - a));
        for (int64_t r = a; r < b; ++r) axis[c].push_back(pos[r * 3 + c]);
        std::sort(axis[c].begin(), axis[c].end());
        axis[c].erase(std::unique(axis[c].begin(), axis[c].end()), axis[c].end());
    }
    const int64_t t = int64_t(axis[0].size()), h = int64_t(axis[1].size()), w = int64_t(axis[2].size());
    if (t * h * w != b - a) return false;
    for (int64_t i = 0; i < b - a; ++i) {
        const double* p = pos + (a + i) * 3;
        if (p[0] != axis[0][size_t(i / (h * w))] || p[1] != axis[1][size_t((i / w) % h)] ||
            p[2] != axis[2][size_t(i % w)])
            return false;
    }
    grid[0] = int32_t(t);
    grid[1] = int32_t(h);
    grid[2] = int32_t(w);
    return true;
}

extern "C" int veda_grid_of(const double* position_ids, int64_t a, int64_t b, int32_t grid_out[3], int32_t* is_grid) {
    veda::clear_error();
    if (!position_ids || !grid_out || !is_grid) return veda::fail(VEDA_ERR_INVALID, "veda_grid_of: NULL argument");
    if (a < 0 || b < a) return veda::fail(VEDA_ERR_INVALID, "veda_grid_of: rows must satisfy 0 <= a <= b");
    *is_grid = grid_of(position_ids, a, b, grid_out) ? 1 : 0;
    return VEDA_OK;
}

extern "C" int veda_describe_packed_layout(const veda_segment* segments, int32_t n_segments, int64_t seq_len,
                                           const int32_t latent[3], const double* position_ids,
                                           veda_packed_desc* out) {
    veda::clear_error();
    if (!segments || !latent || !out || n_segments < 0)
        return veda::fail(VEDA_ERR_INVALID, "veda_describe_packed_layout: NULL argument");
    int video = -1, n_video = 0;
    for (int32_t i = 0; i < n_segments; ++i) {
        const veda_segment& g = segments[i];
        if (g.start < 0 || g.stop < g.start || g.stop > seq_len)
            return veda::fail(VEDA_ERR_INVALID, "veda_describe_packed_layout: segment " + std::to_string(i) +
                                                    " is outside the packed rows");
        if (g.kind == VEDA_SEG_VIDEO) {
            video = i;
            ++n_video;
        }
    }
    if (n_video != 1)
        return veda::fail(VEDA_ERR_INVALID, "expected one target video segment, found " + std::to_string(n_video));
    const int32_t grid[3] = {latent[0], latent[1] / 2, latent[2] / 2};
    if (int64_t(grid[0]) * grid[1] * grid[2] != segments[video].stop - segments[video].start)
        return veda::fail(VEDA_ERR_INVALID, "the video segment does not match the latent grid (" +
                                                std::to_string(grid[0]) + ", " + std::to_string(grid[1]) + ", " +
                                                std::to_string(grid[2]) + ")");
    veda_packed_desc d{};
    d.seq_len = seq_len;
    d.target_start = segments[video].start;
    for (int c = 0; c < 3; ++c) d.target_grid[c] = grid[c];
    for (int32_t i = 0; i < n_segments; ++i) {
        const veda_segment& g = segments[i];
        if (g.kind != VEDA_SEG_COND && g.kind != VEDA_SEG_REF_IMG) continue;
        if (d.n_refs + d.n_skipped >= VEDA_MAX_PACKED_REFS)
            return veda::fail(VEDA_ERR_UNSUPPORTED, "veda_describe_packed_layout: more than " +
                                                        std::to_string(VEDA_MAX_PACKED_REFS) + " reference segments");
        int32_t rg[3];
        if (position_ids && grid_of(position_ids, g.start, g.stop, rg)) {
            d.ref_start[d.n_refs] = g.start;
            for (int c = 0; c < 3; ++c) d.ref_grid[d.n_refs][c] = rg[c];
            ++d.n_refs;
        } else {
            d.skipped[d.n_skipped++] = i;
        }
    }
    *out = d;
    return VEDA_OK;
}
