// C ABI entry points of libveda: argument checks, device copies of layouts, tensor maps and launches.
// The kernels themselves live in gather.cuh, score.cuh, select.cuh and attend.cuh (one translation
// unit, so they share the latched device error word).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>

#include "veda_internal.h"
#include "gather.cuh"
#include "score.cuh"
#include "select.cuh"
#include "attend.cuh"
#include "attend_pair.cuh"
#include "quant.cuh"

namespace veda {

constexpr int kErrBadHead = 4;

__device__ int g_err;  // latched kernel error bits (kErrTimeout | kErrBadList | kErrBadHead)

namespace {

thread_local std::string t_error;
thread_local bool t_hold_next_attend = false;
thread_local int t_attend_ctas = 0;  // test hook: cap on the CTAs of this thread's attend launches (0: none)
std::atomic<uint64_t> g_timeout_ns{1000000000ull};

struct DeviceState {
    bool init = false;
    int sms = 0;
    int* err = nullptr;  // device address of g_err
    bool attend_attr[8] = {};  // (head_dim 128) + 2 * Q/K format; 6 + (head_dim 128) for the gather-free variant
    bool pair_attr[12] = {};   // paired kernel: (head_dim 128) + 2 * gather-free + 4 * Q/K format
    bool score_attr = false;   // the score GEMM's shared-memory size is set
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

int cuda_fail(cudaError_t e, const char* what) {
    return fail(VEDA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

int device_state(DeviceState** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(VEDA_ERR_UNSUPPORTED, "device ordinal beyond the library's table");
    std::lock_guard<std::mutex> g(g_dev_mu);
    DeviceState& s = g_dev[dev];
    if (!s.init) {
        cudaDeviceProp p;
        e = cudaGetDeviceProperties(&p, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
        if (p.major != 10 || p.minor != 0)
            return fail(VEDA_ERR_UNSUPPORTED, "libveda needs an sm_100 (B200-class) device; found sm_" +
                                                  std::to_string(p.major) + std::to_string(p.minor));
        s.sms = p.multiProcessorCount;
        e = cudaGetSymbolAddress(reinterpret_cast<void**>(&s.err), g_err);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
        s.init = true;
    }
    *out = &s;
    return VEDA_OK;
}

// Device copy of a layout's index data on the current device (made on first use).
int device_copy(const veda_layout* lay, const DeviceCopy** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(VEDA_ERR_UNSUPPORTED, "device ordinal beyond the library's table");
    std::lock_guard<std::mutex> g(lay->mu);
    DeviceCopy& dc = lay->dev[dev];
    if (!dc.ready) {
        auto up = [&](int32_t** dst, const std::vector<int32_t>& src) -> cudaError_t {
            const size_t bytes = std::max<size_t>(src.size(), 1) * sizeof(int32_t);
            cudaError_t r = cudaMalloc(reinterpret_cast<void**>(dst), bytes);
            if (r != cudaSuccess) return r;
            if (!src.empty()) r = cudaMemcpy(*dst, src.data(), src.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
            return r;
        };
        if ((e = up(&dc.perm, lay->perm)) != cudaSuccess || (e = up(&dc.valid_count, lay->valid_count)) != cudaSuccess ||
            (e = up(&dc.ok_list, lay->ok_list)) != cudaSuccess || (e = up(&dc.allowed, lay->allowed)) != cudaSuccess ||
            (e = up(&dc.box_perm, lay->box_perm)) != cudaSuccess || (e = up(&dc.tile_coord, lay->tile_coord)) != cudaSuccess ||
            (e = up(&dc.tile_mask, lay->tile_mask)) != cudaSuccess)
            return cuda_fail(e, "uploading the layout");
        dc.ready = true;
    }
    *out = &dc;
    return VEDA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_strided(const int64_t* st, const void* base, const char* name) {
    if (!st) return fail(VEDA_ERR_INVALID, std::string(name) + ": strides are NULL");
    if (st[2] != 1 || st[0] % 8 != 0 || st[1] % 8 != 0 || st[0] <= 0 || st[1] <= 0 || !aligned16(base))
        return fail(VEDA_ERR_INVALID, std::string(name) +
                                          ": needs D stride 1, S and H strides positive multiples of 8, 16-byte base");
    return VEDA_OK;
}

int launch_check(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, what);
    return VEDA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2D map over a head-major tile-ordered tensor viewed as [rows, D]: boxes of 128 rows x 128 bytes (64 bf16
// or 128 e4m3 columns) with the 128-byte swizzle the MMA descriptors expect.
int make_tile_map(CUtensorMap* m, const void* base, int64_t rows, int dim, bool fp8 = false) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const int esize = fp8 ? 1 : 2;
    cuuint64_t gdim[2] = {cuuint64_t(dim), cuuint64_t(rows)};
    cuuint64_t gstride[1] = {cuuint64_t(dim) * esize};
    cuuint32_t box[2] = {cuuint32_t(128 / esize), 128};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void*>(base), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(int(r)) + ")");
    return VEDA_OK;
}

}  // namespace

int fail(int code, const std::string& msg) {
    t_error = msg;
    return code;
}

void clear_error() { t_error.clear(); }

}  // namespace veda

using namespace veda;

extern "C" const char* veda_last_error(void) { return t_error.c_str(); }

extern "C" void veda_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns = ns ? ns : 1; }

extern "C" void veda_debug_hold_next_attend(void) { t_hold_next_attend = true; }
extern "C" void veda_debug_attend_ctas(int32_t n) { t_attend_ctas = n > 0 ? n : 0; }

// CTAs of a persistent attend launch: one per item up to one per SM, or the test cap
static int attend_grid(int n_items, int sms) {
    int g = std::max(1, std::min(n_items, sms));
    return t_attend_ctas > 0 ? std::min(g, t_attend_ctas) : g;
}

namespace veda {
// The three device forms of 2^x, element by element (test hook for the attend kernel's exponentials).
__global__ void exp2_forms_kernel(const float* x, float* poly, float* mufu, float* accurate, int64_t n) {
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float v = x[i];
    if (poly) {
        float p0, p1;
        ptx::f2_unpack(ptx::f2_exp2_poly(ptx::f2_pack(v, v)), p0, p1);
        poly[i] = p0;
    }
    if (mufu) mufu[i] = ptx::ex2(v);
    if (accurate) accurate[i] = exp2f(v);
}
}  // namespace veda

extern "C" int veda_debug_exp2(const float* x, float* poly, float* mufu, float* exp2f_out, int64_t n, void* stream) {
    clear_error();
    if (!x || n < 0) return fail(VEDA_ERR_INVALID, "veda_debug_exp2: NULL input or negative count");
    if (n == 0) return VEDA_OK;
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const int threads = 256;
    const int64_t blocks = (n + threads - 1) / threads;
    if (blocks > 0x7fffffff) return fail(VEDA_ERR_INVALID, "veda_debug_exp2: too many elements");
    exp2_forms_kernel<<<unsigned(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(x, poly, mufu, exp2f_out, n);
    return launch_check("exp2_forms_kernel");
}

extern "C" int veda_device_check(void) {
    clear_error();
    DeviceState* s;
    return device_state(&s);
}

extern "C" void veda_layout_destroy(veda_layout* layout) {
    if (!layout) return;
    int cur = -1;
    const bool have = cudaGetDevice(&cur) == cudaSuccess;
    for (int d = 0; d < kMaxDevices; ++d) {
        DeviceCopy& dc = layout->dev[d];
        if (!dc.ready) continue;
        if (cudaSetDevice(d) == cudaSuccess) {
            cudaFree(dc.perm);
            cudaFree(dc.valid_count);
            cudaFree(dc.ok_list);
            cudaFree(dc.allowed);
            cudaFree(dc.box_perm);
            cudaFree(dc.tile_coord);
            cudaFree(dc.tile_mask);
        }
    }
    if (have) cudaSetDevice(cur);
    delete layout;
}

// Zeroes the per-head maxima that the pool/gather kernel raises with atomicMax.
static int clear_max_sq(float* max_sq, int32_t n_heads, cudaStream_t s) {
    if (!max_sq) return VEDA_OK;
    cudaError_t e = cudaMemsetAsync(max_sq, 0, size_t(n_heads) * sizeof(float), s);
    return e == cudaSuccess ? VEDA_OK : cuda_fail(e, "cudaMemsetAsync(max_sq)");
}

extern "C" int veda_gather(const veda_layout* layout, const void* x, const int64_t x_strides[3], int32_t h_total,
                           int32_t dim, const int32_t* heads, int32_t n_heads, void* x_t, float* feats, float* row_sq,
                           float* max_sq, void* stream) {
    clear_error();
    if (!layout || !x || !heads || !x_t) return fail(VEDA_ERR_INVALID, "veda_gather: NULL argument");
    if (dim != 64 && dim != 128) return fail(VEDA_ERR_INVALID, "veda_gather: head_dim must be 64 or 128");
    if (n_heads <= 0 || h_total <= 0) return fail(VEDA_ERR_INVALID, "veda_gather: head counts must be positive");
    if (int rc = check_strided(x_strides, x, "veda_gather x")) return rc;
    if (!aligned16(x_t) || (feats && !aligned16(feats))) return fail(VEDA_ERR_INVALID, "veda_gather: outputs need 16-byte alignment");
    if ((row_sq && !aligned16(row_sq)) || (max_sq && !aligned16(max_sq)))
        return fail(VEDA_ERR_INVALID, "veda_gather: norm outputs need 16-byte alignment");
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const DeviceCopy* dc;
    if (int rc = device_copy(layout, &dc)) return rc;
    const veda_layout_desc& d = layout->desc;
    GatherArgs a;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.s0 = x_strides[0];
    a.s1 = x_strides[1];
    a.heads = heads;
    a.perm = dc->perm;
    a.valid_count = dc->valid_count;
    a.x_t = static_cast<__nv_bfloat16*>(x_t);
    a.codes = nullptr;
    a.scales = nullptr;
    a.n_tiles = d.n_tiles;
    a.feats = feats;
    a.n_slots = d.n_slots;
    a.n_video = d.n_video;
    a.h_total = h_total;
    a.err = ds->err;
    a.row_sq = row_sq;
    a.max_sq = reinterpret_cast<unsigned*>(max_sq);
    a.seq_len = d.seq_len;
    dim3 grid(unsigned(d.n_tiles), unsigned(n_heads));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int rc = clear_max_sq(max_sq, n_heads, s)) return rc;
    if (dim == 128)
        gather_pool_kernel<128><<<grid, 256, 0, s>>>(a);
    else
        gather_pool_kernel<64><<<grid, 256, 0, s>>>(a);
    return launch_check("gather_pool_kernel");
}

extern "C" int veda_pool(const veda_layout* layout, const void* x, const int64_t x_strides[3], int32_t h_total,
                         int32_t dim, const int32_t* heads, int32_t n_heads, float* feats, float* row_sq,
                         float* max_sq, void* stream) {
    clear_error();
    if (!layout || !x || !heads || !feats) return fail(VEDA_ERR_INVALID, "veda_pool: NULL argument");
    if (dim != 64 && dim != 128) return fail(VEDA_ERR_INVALID, "veda_pool: head_dim must be 64 or 128");
    if (n_heads <= 0 || h_total <= 0) return fail(VEDA_ERR_INVALID, "veda_pool: head counts must be positive");
    if (int rc = check_strided(x_strides, x, "veda_pool x")) return rc;
    if (!aligned16(feats)) return fail(VEDA_ERR_INVALID, "veda_pool: feats needs 16-byte alignment");
    if ((row_sq && !aligned16(row_sq)) || (max_sq && !aligned16(max_sq)))
        return fail(VEDA_ERR_INVALID, "veda_pool: norm outputs need 16-byte alignment");
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const DeviceCopy* dc;
    if (int rc = device_copy(layout, &dc)) return rc;
    const veda_layout_desc& d = layout->desc;
    const bool norms = row_sq || max_sq;
    if (d.n_video == 0 && !norms) return VEDA_OK;
    GatherArgs a;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.s0 = x_strides[0];
    a.s1 = x_strides[1];
    a.heads = heads;
    a.perm = dc->perm;
    a.valid_count = dc->valid_count;
    a.x_t = nullptr;  // no tile copy: pooled features only
    a.codes = nullptr;
    a.scales = nullptr;
    a.n_tiles = d.n_tiles;
    a.feats = feats;
    a.n_slots = d.n_slots;
    a.n_video = d.n_video;
    a.h_total = h_total;
    a.err = ds->err;
    a.row_sq = row_sq;
    a.max_sq = reinterpret_cast<unsigned*>(max_sq);
    a.seq_len = d.seq_len;
    // video tiles only (global tiles are not pooled), unless row norms are asked for: those cover every tile
    dim3 grid(unsigned(norms ? d.n_tiles : d.n_video), unsigned(n_heads));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int rc = clear_max_sq(max_sq, n_heads, s)) return rc;
    if (dim == 128)
        gather_pool_kernel<128, 0, true><<<grid, 256, 0, s>>>(a);
    else
        gather_pool_kernel<64, 0, true><<<grid, 256, 0, s>>>(a);
    return launch_check("gather_pool_kernel");
}

// veda_gather_fp8 / veda_gather_int8: the gather writing 8-bit codes and per-tile scales.
static int gather_codes(const char* who, int code, const veda_layout* layout, const void* x,
                        const int64_t x_strides[3], int32_t h_total, int32_t dim, const int32_t* heads, int32_t n_heads,
                        void* codes, float* scales, float* feats, float* row_sq, float* max_sq, void* stream) {
    clear_error();
    if (!layout || !x || !heads || !codes || !scales) return fail(VEDA_ERR_INVALID, std::string(who) + ": NULL argument");
    if (dim != 64 && dim != 128) return fail(VEDA_ERR_INVALID, std::string(who) + ": head_dim must be 64 or 128");
    if (n_heads <= 0 || h_total <= 0) return fail(VEDA_ERR_INVALID, std::string(who) + ": head counts must be positive");
    if (int rc = check_strided(x_strides, x, who)) return rc;
    if (!aligned16(codes) || !aligned16(scales) || (feats && !aligned16(feats)) || (row_sq && !aligned16(row_sq)) ||
        (max_sq && !aligned16(max_sq)))
        return fail(VEDA_ERR_INVALID, std::string(who) + ": outputs need 16-byte alignment");
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const DeviceCopy* dc;
    if (int rc = device_copy(layout, &dc)) return rc;
    const veda_layout_desc& d = layout->desc;
    GatherArgs a;
    a.x = static_cast<const __nv_bfloat16*>(x);
    a.s0 = x_strides[0];
    a.s1 = x_strides[1];
    a.heads = heads;
    a.perm = dc->perm;
    a.valid_count = dc->valid_count;
    a.x_t = nullptr;
    a.codes = static_cast<uint8_t*>(codes);
    a.scales = scales;
    a.n_tiles = d.n_tiles;
    a.feats = feats;
    a.n_slots = d.n_slots;
    a.n_video = d.n_video;
    a.h_total = h_total;
    a.err = ds->err;
    a.row_sq = row_sq;
    a.max_sq = reinterpret_cast<unsigned*>(max_sq);
    a.seq_len = d.seq_len;
    dim3 grid(unsigned(d.n_tiles), unsigned(n_heads));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int rc = clear_max_sq(max_sq, n_heads, s)) return rc;
    if (code == kCodeI8) {
        if (dim == 128)
            gather_pool_kernel<128, kCodeI8><<<grid, 256, 0, s>>>(a);
        else
            gather_pool_kernel<64, kCodeI8><<<grid, 256, 0, s>>>(a);
    } else {
        if (dim == 128)
            gather_pool_kernel<128, kCodeE4M3><<<grid, 256, 0, s>>>(a);
        else
            gather_pool_kernel<64, kCodeE4M3><<<grid, 256, 0, s>>>(a);
    }
    return launch_check("gather_pool_kernel (8-bit codes)");
}

extern "C" int veda_gather_fp8(const veda_layout* layout, const void* x, const int64_t x_strides[3], int32_t h_total,
                               int32_t dim, const int32_t* heads, int32_t n_heads, void* codes, float* scales,
                               float* feats, float* row_sq, float* max_sq, void* stream) {
    return gather_codes("veda_gather_fp8", kCodeE4M3, layout, x, x_strides, h_total, dim, heads, n_heads, codes,
                        scales, feats, row_sq, max_sq, stream);
}

extern "C" int veda_gather_int8(const veda_layout* layout, const void* x, const int64_t x_strides[3], int32_t h_total,
                                int32_t dim, const int32_t* heads, int32_t n_heads, void* codes, float* scales,
                                float* feats, float* row_sq, float* max_sq, void* stream) {
    return gather_codes("veda_gather_int8", kCodeI8, layout, x, x_strides, h_total, dim, heads, n_heads, codes,
                        scales, feats, row_sq, max_sq, stream);
}

extern "C" size_t veda_score_workspace_bytes(const veda_layout* layout, int32_t n_heads, int32_t dim) {
    if (!layout || n_heads <= 0 || dim <= 0) return 0;
    return size_t(n_heads) * size_t(score_scratch_per_head(layout->desc.n_video, dim)) * sizeof(float);
}

namespace veda {

// 3D fp32 map over [batch][rows][K] (K innermost): boxes of 32 K-columns (128 bytes) x 128 rows with the
// 128-byte swizzle of the tf32 MMA operands; rows past `rows` read as zeros.
int make_f32_map(CUtensorMap* m, const float* base, int64_t K, int64_t rows, int64_t batch) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t gdim[3] = {cuuint64_t(K), cuuint64_t(rows), cuuint64_t(batch)};
    cuuint64_t gstride[2] = {cuuint64_t(K) * 4, cuuint64_t(rows) * cuuint64_t(K) * 4};
    cuuint32_t box[3] = {cuuint32_t(tf32x3::kBK), cuuint32_t(tf32x3::kBM), 1};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled (fp32 operand) failed (" + std::to_string(int(r)) + ")");
    return VEDA_OK;
}

int launch_score_gemms(const float* feats_q, const float* feats_k, const float* proj_q, const float* proj_k, float* qh,
                       float* kh, float* pt_q, float* pt_k, float* scores, int nv, int dim, int n_heads,
                       cudaStream_t s) {
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    if (!ds->score_attr) {
        cudaError_t e = cudaFuncSetAttribute(tf32x3::gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(tf32x3::kSmem));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(score gemm_kernel)");
        ds->score_attr = true;
    }
    if (nv <= 0) return VEDA_OK;
    // (P + E)^T: both operands of the projection K-major, the residual feats[:, :D] folded in
    tf32x3::transpose_kernel<<<dim3(unsigned(dim / 32), unsigned(3 * dim / 32), unsigned(2 * n_heads)), 256, 0, s>>>(
        proj_q, proj_k, pt_q, pt_k, n_heads, 3 * dim, dim);
    if (int rc = launch_check("score transpose_kernel")) return rc;

    // q_hat = fq (P_q + E) = fq P_q + fq[:, :D] and k_hat likewise, in one launch (two operand sets)
    tf32x3::Maps pm;
    if (int rc = make_f32_map(&pm.a[0], feats_q, 3 * dim, nv, n_heads)) return rc;
    if (int rc = make_f32_map(&pm.b[0], pt_q, 3 * dim, dim, n_heads)) return rc;
    if (int rc = make_f32_map(&pm.a[1], feats_k, 3 * dim, nv, n_heads)) return rc;
    if (int rc = make_f32_map(&pm.b[1], pt_k, 3 * dim, dim, n_heads)) return rc;
    tf32x3::Args pa{};
    pa.n_sets = 2;
    pa.nb = n_heads;
    pa.M = nv;
    pa.N = dim;
    pa.K = 3 * dim;
    pa.tiles_m = (nv + tf32x3::kBM - 1) / tf32x3::kBM;
    pa.tiles_n = 1;
    pa.n_tiles = 2 * n_heads * pa.tiles_m;
    pa.C[0] = qh;
    pa.C[1] = kh;
    pa.scale = 1.f;
    pa.timeout_ns = g_timeout_ns.load();
    pa.err = ds->err;
    tf32x3::gemm_kernel<<<unsigned(std::min(pa.n_tiles, ds->sms)), tf32x3::kThreads, tf32x3::kSmem, s>>>(pm, pa);
    if (int rc = launch_check("score gemm_kernel (projections)")) return rc;

    // scores = q_hat k_hat^T / sqrt(D), as a product with 1 / sqrt(D) rounded to fp32
    tf32x3::Maps lm;
    if (int rc = make_f32_map(&lm.a[0], qh, dim, nv, n_heads)) return rc;
    if (int rc = make_f32_map(&lm.b[0], kh, dim, nv, n_heads)) return rc;
    lm.a[1] = lm.a[0];
    lm.b[1] = lm.b[0];
    tf32x3::Args la{};
    la.n_sets = 1;
    la.nb = n_heads;
    la.M = nv;
    la.N = nv;
    la.K = dim;
    la.tiles_m = (nv + tf32x3::kBM - 1) / tf32x3::kBM;
    la.tiles_n = (nv + tf32x3::kBN - 1) / tf32x3::kBN;
    la.n_tiles = n_heads * la.tiles_m * la.tiles_n;
    la.C[0] = la.C[1] = scores;
    la.scale = float(1.0 / std::sqrt(double(dim)));
    la.timeout_ns = pa.timeout_ns;
    la.err = ds->err;
    tf32x3::gemm_kernel<<<unsigned(std::min(la.n_tiles, ds->sms)), tf32x3::kThreads, tf32x3::kSmem, s>>>(lm, la);
    return launch_check("score gemm_kernel (logits)");
}

}  // namespace veda

extern "C" int veda_score(const veda_layout* layout, const float* feats_q, const float* feats_k, int32_t n_heads,
                          int32_t dim, const float* proj_q, const float* proj_k, void* workspace,
                          size_t workspace_bytes, float* scores, void* stream) {
    clear_error();
    if (!layout || !feats_q || !feats_k || !proj_q || !proj_k || !workspace || !scores)
        return fail(VEDA_ERR_INVALID, "veda_score: NULL argument");
    if (dim != 64 && dim != 128) return fail(VEDA_ERR_INVALID, "veda_score: head_dim must be 64 or 128");
    if (n_heads <= 0) return fail(VEDA_ERR_INVALID, "veda_score: n_heads must be positive");
    if (workspace_bytes < veda_score_workspace_bytes(layout, n_heads, dim))
        return fail(VEDA_ERR_INVALID, "veda_score: workspace smaller than veda_score_workspace_bytes()");
    if (!aligned16(feats_q) || !aligned16(feats_k) || !aligned16(proj_q) || !aligned16(proj_k) ||
        !aligned16(workspace) || !aligned16(scores))
        return fail(VEDA_ERR_INVALID, "veda_score: buffers need 16-byte alignment");
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const int nv = layout->desc.n_video;
    float* qh = static_cast<float*>(workspace);
    float* kh = qh + int64_t(n_heads) * nv * dim;
    float* pt_q = kh + int64_t(n_heads) * nv * dim;
    float* pt_k = pt_q + int64_t(n_heads) * 3 * dim * dim;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return launch_score_gemms(feats_q, feats_k, proj_q, proj_k, qh, kh, pt_q, pt_k, scores, nv, dim, n_heads, s);
}

template <int kPer>
static int launch_rows(const SelectArgs& a, int64_t n_rows, cudaStream_t st) {
    const int64_t grid = (n_rows + kRowsWarps - 1) / kRowsWarps;
    if (grid > 0x7fffffff) return fail(VEDA_ERR_UNSUPPORTED, "veda_select: too many rows for one launch");
    if (a.n_blocks == 2)
        select_rows_kernel<kPer, true><<<unsigned(grid), 32 * kRowsWarps, 0, st>>>(a);
    else
        select_rows_kernel<kPer, false><<<unsigned(grid), 32 * kRowsWarps, 0, st>>>(a);
    return launch_check("select_rows_kernel");
}

// One warp per row; kPer = slots per lane, the row's width / 32 rounded up to a multiple of 4.
static int launch_select_rows(int per, const SelectArgs& a, int64_t n_rows, cudaStream_t st) {
    switch (per) {
        case 4: return launch_rows<4>(a, n_rows, st);
        case 8: return launch_rows<8>(a, n_rows, st);
        case 12: return launch_rows<12>(a, n_rows, st);
        case 16: return launch_rows<16>(a, n_rows, st);
        case 20: return launch_rows<20>(a, n_rows, st);
        case 24: return launch_rows<24>(a, n_rows, st);
        case 28: return launch_rows<28>(a, n_rows, st);
        case 32: return launch_rows<32>(a, n_rows, st);
        case 36: return launch_rows<36>(a, n_rows, st);
        case 40: return launch_rows<40>(a, n_rows, st);
        case 44: return launch_rows<44>(a, n_rows, st);
        case 48: return launch_rows<48>(a, n_rows, st);
        case 52: return launch_rows<52>(a, n_rows, st);
        case 56: return launch_rows<56>(a, n_rows, st);
        case 60: return launch_rows<60>(a, n_rows, st);
        default: return launch_rows<64>(a, n_rows, st);
    }
}

extern "C" int veda_select(const veda_layout* layout, const float* scores, int32_t n_heads, int32_t* kept_idx,
                           int32_t* kept_cnt, void* stream) {
    clear_error();
    if (!layout || !scores || !kept_idx || !kept_cnt) return fail(VEDA_ERR_INVALID, "veda_select: NULL argument");
    if (n_heads <= 0) return fail(VEDA_ERR_INVALID, "veda_select: n_heads must be positive");
    const veda_layout_desc& d = layout->desc;
    int widest = 1;
    for (int b = 0; b < d.n_blocks; ++b) widest = std::max(widest, d.blocks[b].stop - d.blocks[b].start);
    if (widest > kSelectMaxCols)
        return fail(VEDA_ERR_UNSUPPORTED, "veda_select: a column block wider than 16384 tiles");
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const DeviceCopy* dc;
    if (int rc = device_copy(layout, &dc)) return rc;
    SelectArgs a;
    a.scores = scores;
    a.valid_count = dc->valid_count;
    a.allowed = dc->allowed;
    a.ok_list = dc->ok_list;
    a.kept_idx = kept_idx;
    a.kept_cnt = kept_cnt;
    a.n_video = d.n_video;
    a.n_blocks = d.n_blocks;
    a.max_kept = d.max_kept;
    a.n_kv_ok = d.n_kv_ok;
    a.n_global_ok = d.n_global_ok;
    for (int b = 0; b < 2; ++b) {
        a.blk_start[b] = b < d.n_blocks ? d.blocks[b].start : 0;
        a.blk_stop[b] = b < d.n_blocks ? d.blocks[b].stop : 0;
        a.blk_all[b] = b < d.n_blocks ? d.blocks[b].keeps_all : 0;
    }
    a.n_heads = n_heads;
    a.all_ok = 1;
    for (int c = 0; c < d.n_video; ++c) a.all_ok &= layout->valid_count[c] > 0;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d.n_video <= 32 * 64) {
        // one warp per row (rows of up to 2048 video tiles)
        const int per = ((d.n_video + 31) / 32 + 3) / 4 * 4;  // slots per lane, a multiple of 4
        return launch_select_rows(per, a, int64_t(n_heads) * d.n_video, st);
    }
    if (widest <= 32 * 64) {
        // one warp per row, the block's keys in registers
        const dim3 grid(unsigned((d.n_video + 7) / 8), unsigned(n_heads));
        if (widest <= 32 * 16)
            select_warp_kernel<16><<<grid, 256, 0, st>>>(a);
        else if (widest <= 32 * 32)
            select_warp_kernel<32><<<grid, 256, 0, st>>>(a);
        else
            select_warp_kernel<64><<<grid, 256, 0, st>>>(a);
        return launch_check("select_warp_kernel");
    }
    const size_t smem = size_t(widest) * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(select_kernel)");
    }
    select_kernel<<<dim3(unsigned(d.n_video), unsigned(n_heads)), kSelectThreads, smem, static_cast<cudaStream_t>(stream)>>>(a);
    return launch_check("select_kernel");
}

template <int D, int kQK, bool kDirect = false>
static int launch_attend(DeviceState* ds, const AttendMaps& maps, const AttendArgs& a, cudaStream_t s) {
    using C = AttendCfg<D, kQK>;
    const int slot = kDirect ? 6 + (D == 128) : (D == 128) + 2 * kQK;
    if (!ds->attend_attr[slot]) {
        cudaError_t e = cudaFuncSetAttribute(attend_kernel<D, kQK, kDirect>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attend_kernel)");
        ds->attend_attr[slot] = true;
    }
    attend_kernel<D, kQK, kDirect><<<attend_grid(a.n_items, ds->sms), C::kThreads, C::kSmem, s>>>(maps, a);
    return launch_check("attend_kernel");
}

// Workspace of the paired attend, each region 256-aligned: the merged unit lists and their counts, the
// redo flags followed by the redo list's length (cleared together), and the redo list.
struct PairWorkspace {
    int32_t* units;
    int2* counts;
    int32_t* flags;
    int32_t* redo_count;
    int32_t* redo_items;
};
static int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }
// sizes from the layout's video tile count, list width and tile count
static int64_t pair_units_bytes(int64_t n_video, int64_t max_kept, int32_t n_heads) {
    return align256(int64_t(n_heads) * ((n_video + 1) / 2) * 2 * max_kept * 4);
}
static int64_t pair_counts_bytes(int64_t n_video, int32_t n_heads) {
    return align256(int64_t(n_heads) * ((n_video + 1) / 2) * 8);
}
static int64_t pair_flags_bytes(int64_t n_tiles, int32_t n_heads) { return align256(int64_t(n_heads) * n_tiles * 4); }
static int64_t pair_workspace_total(int64_t n_video, int64_t max_kept, int64_t n_tiles, int32_t n_heads) {
    return pair_units_bytes(n_video, max_kept, n_heads) + pair_counts_bytes(n_video, n_heads) +
           2 * pair_flags_bytes(n_tiles, n_heads) + 256;
}
static PairWorkspace pair_workspace(int64_t n_video, int64_t max_kept, int64_t n_tiles, int32_t n_heads, void* base) {
    char* p = static_cast<char*>(base);
    const int64_t ub = pair_units_bytes(n_video, max_kept, n_heads), cb = pair_counts_bytes(n_video, n_heads);
    const int64_t fb = pair_flags_bytes(n_tiles, n_heads);
    return {reinterpret_cast<int32_t*>(p), reinterpret_cast<int2*>(p + ub), reinterpret_cast<int32_t*>(p + ub + cb),
            reinterpret_cast<int32_t*>(p + ub + cb + fb), reinterpret_cast<int32_t*>(p + ub + cb + fb + 256)};
}

extern "C" size_t veda_attend_paired_workspace_bytes(const veda_layout* layout, int32_t n_heads) {
    if (!layout || n_heads <= 0) return 0;
    const veda_layout_desc& d = layout->desc;
    return size_t(pair_workspace_total(d.n_video, d.max_kept, d.n_tiles, n_heads));
}

// The paired attend: clear the redo flags, merge each pair's lists into units, run the paired kernel, then
// the single-tile kernel over the query tiles it flagged (an empty pass when none is).
template <int D, int kQK, bool kDirect>
static int launch_paired(DeviceState* ds, const AttendMaps& maps, AttendArgs a, const int32_t* kept_idx,
                         const int32_t* kept_cnt, void* workspace, cudaStream_t s) {
    const PairWorkspace ws = pair_workspace(a.n_video, a.max_kept, a.n_tiles, a.n_heads, workspace);
    cudaError_t e = cudaMemsetAsync(ws.flags, 0, size_t(pair_flags_bytes(a.n_tiles, a.n_heads)) + 256, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(redo flags)");
    PairUnitsArgs u{};
    u.kept_idx = kept_idx;
    u.kept_cnt = kept_cnt;
    u.n_video = a.n_video;
    u.max_kept = a.max_kept;
    u.n_tiles = a.n_tiles;
    u.n_heads = a.n_heads;
    u.n_pairs = (a.n_video + 1) / 2;
    u.units = ws.units;
    u.counts = ws.counts;
    u.err = a.err;
    const int64_t warps = int64_t(u.n_heads) * u.n_pairs;
    if (warps > 0) {
        // each warp stages its two lists in shared memory: up to 8 warps per block within 48 KB, else one
        // warp per block with the opt-in size (lists of up to ~29,000 tiles)
        const int64_t per_warp = 8 * int64_t(std::max(u.max_kept, 1));
        const int wpb = int(std::max<int64_t>(1, std::min<int64_t>(8, 49152 / per_warp)));
        const int64_t smem = per_warp * wpb;
        if (smem > 227 * 1024)
            return fail(VEDA_ERR_UNSUPPORTED, "veda_attend_paired: kept lists too wide for the list merge");
        if (smem > 49152) {
            e = cudaFuncSetAttribute(pair_units_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(pair_units_kernel)");
        }
        pair_units_kernel<<<unsigned((warps + wpb - 1) / wpb), unsigned(32 * wpb), size_t(smem), s>>>(u);
        if (int rc = launch_check("pair_units_kernel")) return rc;
    }
    PairArgs p{};
    p.units = ws.units;
    p.counts = ws.counts;
    p.ok_list = a.ok_list;
    p.valid_count = a.valid_count;
    p.perm = a.perm;
    p.heads = a.heads;
    p.out = a.out;
    p.out_s0 = a.out_s0;
    p.out_s1 = a.out_s1;
    p.n_slots = a.n_slots;
    p.max_kept = a.max_kept;
    p.n_ok = a.n_ok;
    p.n_tiles = a.n_tiles;
    p.n_video = a.n_video;
    p.n_global = a.n_global;
    p.n_heads = a.n_heads;
    p.h_total = a.h_total;
    p.n_pairs = (a.n_video + 1) / 2;
    p.n_gpairs = (a.n_global + 1) / 2;
    p.n_items = a.n_heads * (p.n_pairs + p.n_gpairs);
    p.scale_log2 = a.scale_log2;
    p.timeout_ns = a.timeout_ns;
    p.err = a.err;
    p.hold_q = a.hold_q;
    p.tile_coord = a.tile_coord;
    p.tile_mask = a.tile_mask;
    p.n_map_spans = a.n_map_spans;
    p.scales_q = a.scales_q;
    p.scales_k = a.scales_k;
    p.q_row_sq = a.q_row_sq;
    p.k_max_sq = a.k_max_sq;
    p.seq_len = a.seq_len;
    p.redo_flags = ws.flags;
    p.redo_items = ws.redo_items;
    p.redo_count = ws.redo_count;
    using C = PairCfg<D, kQK>;
    const int slot = (D == 128) + 2 * kDirect + 4 * kQK;
    if (!ds->pair_attr[slot]) {
        e = cudaFuncSetAttribute(attend_pair_kernel<D, kQK, kDirect>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attend_pair_kernel)");
        ds->pair_attr[slot] = true;
    }
    attend_pair_kernel<D, kQK, kDirect><<<attend_grid(p.n_items, ds->sms), C::kThreads, C::kSmem, s>>>(maps, p);
    if (int rc = launch_check("attend_pair_kernel")) return rc;
    // the redo pass over the listed items (at most n_items); CTAs past the list's length return at once
    a.redo_items = ws.redo_items;
    a.redo_count = ws.redo_count;
    a.hold_q = 0;
    return launch_attend<D, kQK, kDirect>(ds, maps, a, s);
}

// The launch arguments both attend entry points share: lists, layout tables, output, limits and the wait
// settings (tile tables and scales are left empty; each caller sets what its variant reads).
static AttendArgs attend_args(const veda_layout_desc& d, const DeviceCopy* dc, const DeviceState* ds,
                              const int32_t* kept_idx, const int32_t* kept_cnt, void* out,
                              const int64_t out_strides[3], int32_t h_total, const int32_t* heads, int32_t n_heads,
                              int32_t dim) {
    AttendArgs a{};
    a.kept_idx = kept_idx;
    a.kept_cnt = kept_cnt;
    a.ok_list = dc->ok_list;
    a.valid_count = dc->valid_count;
    a.perm = dc->perm;
    a.heads = heads;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.out_s0 = out_strides[0];
    a.out_s1 = out_strides[1];
    a.n_slots = d.n_slots;
    a.max_kept = d.max_kept;
    a.n_ok = d.n_kv_ok;
    a.n_tiles = d.n_tiles;
    a.n_video = d.n_video;
    a.n_global = d.n_global;
    a.n_heads = n_heads;
    a.h_total = h_total;
    a.n_items = n_heads * d.n_tiles;
    a.scale_log2 = float((1.0 / std::sqrt(double(dim))) * 1.4426950408889634);
    a.timeout_ns = g_timeout_ns.load();
    a.err = ds->err;
    a.hold_q = t_hold_next_attend ? 1 : 0;
    t_hold_next_attend = false;
    a.scales_q = nullptr;
    a.scales_k = nullptr;
    a.tile_coord = nullptr;
    a.tile_mask = nullptr;
    a.n_map_spans = 1;
    a.q_row_sq = nullptr;
    a.k_max_sq = nullptr;
    a.seq_len = d.seq_len;
    return a;
}

static int attend_common(const veda_layout* layout, const void* q, const void* k, const float* sq, const float* sk,
                         const void* v_t, int32_t n_heads, int32_t dim, const int32_t* kept_idx,
                         const int32_t* kept_cnt, void* out, const int64_t out_strides[3], int32_t h_total,
                         const int32_t* heads, void* stream, int qk, const float* q_row_sq = nullptr,
                         const float* k_max_sq = nullptr, void* pair_ws = nullptr) {
    const bool fp8 = qk != kQKBf16;  // 8-bit Q/K codes (e4m3 or int8)
    const char* who = qk == kQKI8 ? (pair_ws ? "veda_attend_int8_paired" : "veda_attend_int8")
                      : fp8       ? (pair_ws ? "veda_attend_fp8_paired" : "veda_attend_fp8")
                      : pair_ws   ? "veda_attend_paired"
                                  : "veda_attend";
    if (!layout || !q || !k || !v_t || !kept_idx || !kept_cnt || !out || !heads || (fp8 && (!sq || !sk)))
        return fail(VEDA_ERR_INVALID, std::string(who) + ": NULL argument");
    if (fp8 ? dim != 128 : (dim != 64 && dim != 128))
        return fail(VEDA_ERR_INVALID, std::string(who) + (fp8 ? ": head_dim must be 128" : ": head_dim must be 64 or 128"));
    if (n_heads <= 0 || h_total <= 0) return fail(VEDA_ERR_INVALID, std::string(who) + ": head counts must be positive");
    if (int rc = check_strided(out_strides, out, who)) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v_t))
        return fail(VEDA_ERR_INVALID, std::string(who) + ": tile-ordered inputs need 16-byte alignment");
    const veda_layout_desc& d = layout->desc;
    if (int64_t(n_heads) * d.n_slots >= (int64_t(1) << 31))
        return fail(VEDA_ERR_UNSUPPORTED, std::string(who) + ": n_heads * N must stay below 2^31 rows");
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const DeviceCopy* dc;
    if (int rc = device_copy(layout, &dc)) return rc;
    AttendMaps maps;
    std::memset(&maps, 0, sizeof maps);
    const int64_t rows = int64_t(n_heads) * d.n_slots;
    if (int rc = make_tile_map(&maps.q[0], q, rows, dim, fp8)) return rc;
    if (int rc = make_tile_map(&maps.k[0], k, rows, dim, fp8)) return rc;
    if (int rc = make_tile_map(&maps.v[0], v_t, rows, dim)) return rc;
    AttendArgs a = attend_args(d, dc, ds, kept_idx, kept_cnt, out, out_strides, h_total, heads, n_heads, dim);
    a.scales_q = sq;
    a.scales_k = sk;
    if (q_row_sq && k_max_sq) {  // the logit bound (bf16 Q/K only; the 8-bit variants keep the per-tile max)
        a.q_row_sq = q_row_sq;
        a.k_max_sq = k_max_sq;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pair_ws) {
        // the logit bound for the 8-bit codes comes from the bf16 norms: the codes' logits differ from the
        // bf16 ones by the quantisation error, far inside the reference's 2^64 headroom
        a.q_row_sq = q_row_sq;
        a.k_max_sq = k_max_sq;
        if (qk == kQKI8) return launch_paired<128, kQKI8, false>(ds, maps, a, kept_idx, kept_cnt, pair_ws, s);
        if (qk == kQKE4M3) return launch_paired<128, kQKE4M3, false>(ds, maps, a, kept_idx, kept_cnt, pair_ws, s);
        return dim == 128 ? launch_paired<128, kQKBf16, false>(ds, maps, a, kept_idx, kept_cnt, pair_ws, s)
                          : launch_paired<64, kQKBf16, false>(ds, maps, a, kept_idx, kept_cnt, pair_ws, s);
    }
    if (qk == kQKI8) return launch_attend<128, kQKI8>(ds, maps, a, s);
    if (qk == kQKE4M3) return launch_attend<128, kQKE4M3>(ds, maps, a, s);
    return dim == 128 ? launch_attend<128, kQKBf16>(ds, maps, a, s) : launch_attend<64, kQKBf16>(ds, maps, a, s);
}

extern "C" int veda_attend(const veda_layout* layout, const void* q_t, const void* k_t, const void* v_t,
                           int32_t n_heads, int32_t dim, const int32_t* kept_idx, const int32_t* kept_cnt, void* out,
                           const int64_t out_strides[3], int32_t h_total, const int32_t* heads,
                           const float* q_row_sq, const float* k_max_sq, void* stream) {
    clear_error();
    return attend_common(layout, q_t, k_t, nullptr, nullptr, v_t, n_heads, dim, kept_idx, kept_cnt, out, out_strides,
                         h_total, heads, stream, kQKBf16, q_row_sq, k_max_sq);
}

// Checks shared by the paired entry points: the norms of the bound and an aligned workspace.
static int check_paired(const char* who, const veda_layout* layout, int32_t n_heads, const float* q_row_sq,
                        const float* k_max_sq, const void* workspace, size_t workspace_bytes) {
    if (!q_row_sq || !k_max_sq)
        return fail(VEDA_ERR_INVALID, std::string(who) + ": the paired kernel needs q_row_sq and k_max_sq (veda_pool)");
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0)
        return fail(VEDA_ERR_INVALID, std::string(who) + ": workspace must be a 256-byte aligned device buffer");
    if (layout && n_heads > 0 && workspace_bytes < veda_attend_paired_workspace_bytes(layout, n_heads))
        return fail(VEDA_ERR_INVALID, std::string(who) + ": workspace smaller than veda_attend_paired_workspace_bytes");
    return VEDA_OK;
}

extern "C" int veda_attend_paired(const veda_layout* layout, const void* q_t, const void* k_t, const void* v_t,
                                  int32_t n_heads, int32_t dim, const int32_t* kept_idx, const int32_t* kept_cnt,
                                  void* out, const int64_t out_strides[3], int32_t h_total, const int32_t* heads,
                                  const float* q_row_sq, const float* k_max_sq, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    clear_error();
    if (int rc = check_paired("veda_attend_paired", layout, n_heads, q_row_sq, k_max_sq, workspace, workspace_bytes))
        return rc;
    return attend_common(layout, q_t, k_t, nullptr, nullptr, v_t, n_heads, dim, kept_idx, kept_cnt, out, out_strides,
                         h_total, heads, stream, kQKBf16, q_row_sq, k_max_sq, workspace);
}

static_assert(kMapSets == kMaxDirectSpans + 1, "one map set per tiled span plus the global set");

// 5D map over a packed [S, H_total, D] tensor viewed as the boxes of one tiled span: dims (D, heads, w, h,
// t) from the span's first row, box (64, 1, sw, sh, st); positions outside the grid read as zeros.
static int make_span_map(CUtensorMap* m, const void* x, const int64_t st[3], int32_t h_total, int dim,
                         const DirectSpan& sp) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const char* base = static_cast<const char*>(x) + sp.start * st[0] * 2;
    cuuint64_t gdim[5] = {cuuint64_t(dim), cuuint64_t(h_total), cuuint64_t(sp.w), cuuint64_t(sp.h), cuuint64_t(sp.t)};
    cuuint64_t gstride[4] = {cuuint64_t(st[1]) * 2, cuuint64_t(st[0]) * 2, cuuint64_t(st[0]) * 2 * cuuint64_t(sp.w),
                             cuuint64_t(st[0]) * 2 * cuuint64_t(sp.w) * cuuint64_t(sp.h)};
    cuuint32_t box[5] = {64, 1, cuuint32_t(sp.sw), cuuint32_t(sp.sh), cuuint32_t(sp.st)};
    cuuint32_t estride[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<char*>(base), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled (span box) failed (" + std::to_string(int(r)) + ")");
    return VEDA_OK;
}

// 3D map over rows [0, rows) of a packed [S, H_total, D] tensor: dims (D, heads, rows), box (64, 1, 128).
static int make_row_map(CUtensorMap* m, const void* x, const int64_t st[3], int32_t h_total, int dim, int64_t rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t gdim[3] = {cuuint64_t(dim), cuuint64_t(h_total), cuuint64_t(std::max<int64_t>(rows, 1))};
    cuuint64_t gstride[2] = {cuuint64_t(st[1]) * 2, cuuint64_t(st[0]) * 2};
    cuuint32_t box[3] = {64, 1, 128};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(VEDA_ERR_CUDA, "cuTensorMapEncodeTiled (global rows) failed (" + std::to_string(int(r)) + ")");
    return VEDA_OK;
}

static int attend_direct_impl(const veda_layout* layout, const void* q, const int64_t q_strides[3], const void* k,
                              const int64_t k_strides[3], const void* v, const int64_t v_strides[3], int32_t h_total,
                              int32_t dim, const int32_t* heads, int32_t n_heads, const int32_t* kept_idx,
                              const int32_t* kept_cnt, void* out, const int64_t out_strides[3], const float* q_row_sq,
                              const float* k_max_sq, void* pair_ws, void* stream) {
    const char* who = pair_ws ? "veda_attend_direct_paired" : "veda_attend_direct";
    if (!layout || !q || !k || !v || !kept_idx || !kept_cnt || !out || !heads)
        return fail(VEDA_ERR_INVALID, std::string(who) + ": NULL argument");
    if (dim != 64 && dim != 128) return fail(VEDA_ERR_INVALID, std::string(who) + ": head_dim must be 64 or 128");
    if (n_heads <= 0 || h_total <= 0) return fail(VEDA_ERR_INVALID, std::string(who) + ": head counts must be positive");
    if (int rc = check_strided(q_strides, q, "veda_attend_direct q")) return rc;
    if (int rc = check_strided(k_strides, k, "veda_attend_direct k")) return rc;
    if (int rc = check_strided(v_strides, v, "veda_attend_direct v")) return rc;
    if (int rc = check_strided(out_strides, out, "veda_attend_direct out")) return rc;
    if (!layout->direct_ok)
        return fail(VEDA_ERR_UNSUPPORTED, std::string(who) + ": " + layout->direct_why + "; use veda_gather + veda_attend");
    const veda_layout_desc& d = layout->desc;
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const DeviceCopy* dc;
    if (int rc = device_copy(layout, &dc)) return rc;
    AttendMaps maps;
    std::memset(&maps, 0, sizeof maps);
    const int n_spans = int(layout->spans.size());
    for (int i = 0; i < n_spans; ++i) {
        const DirectSpan& sp = layout->spans[size_t(i)];
        if (int rc = make_span_map(&maps.q[i], q, q_strides, h_total, dim, sp)) return rc;
        if (int rc = make_span_map(&maps.k[i], k, k_strides, h_total, dim, sp)) return rc;
        if (int rc = make_span_map(&maps.v[i], v, v_strides, h_total, dim, sp)) return rc;
    }
    if (d.n_global > 0) {
        // rows past the last global row read as zeros, which masks the tail of a partial last tile
        int64_t end = 0;
        for (int64_t i = d.n_video; i < d.n_tiles; ++i) {
            const int32_t c = layout->valid_count[size_t(i)];
            if (c > 0) end = std::max<int64_t>(end, int64_t(layout->perm[size_t(i * kTile + c - 1)]) + 1);
        }
        if (int rc = make_row_map(&maps.q[kGlobalMapSet], q, q_strides, h_total, dim, end)) return rc;
        if (int rc = make_row_map(&maps.k[kGlobalMapSet], k, k_strides, h_total, dim, end)) return rc;
        if (int rc = make_row_map(&maps.v[kGlobalMapSet], v, v_strides, h_total, dim, end)) return rc;
    }
    AttendArgs a = attend_args(d, dc, ds, kept_idx, kept_cnt, out, out_strides, h_total, heads, n_heads, dim);
    a.perm = dc->box_perm;  // box order: packed row of each box position
    a.tile_coord = reinterpret_cast<const int4*>(dc->tile_coord);
    a.tile_mask = reinterpret_cast<const uint4*>(dc->tile_mask);
    a.n_map_spans = n_spans;
    if (q_row_sq && k_max_sq) {
        a.q_row_sq = q_row_sq;
        a.k_max_sq = k_max_sq;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pair_ws)
        return dim == 128 ? launch_paired<128, kQKBf16, true>(ds, maps, a, kept_idx, kept_cnt, pair_ws, s)
                          : launch_paired<64, kQKBf16, true>(ds, maps, a, kept_idx, kept_cnt, pair_ws, s);
    return dim == 128 ? launch_attend<128, kQKBf16, true>(ds, maps, a, s) : launch_attend<64, kQKBf16, true>(ds, maps, a, s);
}

extern "C" int veda_attend_direct(const veda_layout* layout, const void* q, const int64_t q_strides[3], const void* k,
                                  const int64_t k_strides[3], const void* v, const int64_t v_strides[3],
                                  int32_t h_total, int32_t dim, const int32_t* heads, int32_t n_heads,
                                  const int32_t* kept_idx, const int32_t* kept_cnt, void* out,
                                  const int64_t out_strides[3], const float* q_row_sq, const float* k_max_sq,
                                  void* stream) {
    clear_error();
    return attend_direct_impl(layout, q, q_strides, k, k_strides, v, v_strides, h_total, dim, heads, n_heads, kept_idx,
                              kept_cnt, out, out_strides, q_row_sq, k_max_sq, nullptr, stream);
}

extern "C" int veda_attend_direct_paired(const veda_layout* layout, const void* q, const int64_t q_strides[3],
                                         const void* k, const int64_t k_strides[3], const void* v,
                                         const int64_t v_strides[3], int32_t h_total, int32_t dim,
                                         const int32_t* heads, int32_t n_heads, const int32_t* kept_idx,
                                         const int32_t* kept_cnt, void* out, const int64_t out_strides[3],
                                         const float* q_row_sq, const float* k_max_sq, void* workspace,
                                         size_t workspace_bytes, void* stream) {
    clear_error();
    if (int rc = check_paired("veda_attend_direct_paired", layout, n_heads, q_row_sq, k_max_sq, workspace,
                              workspace_bytes))
        return rc;
    return attend_direct_impl(layout, q, q_strides, k, k_strides, v, v_strides, h_total, dim, heads, n_heads, kept_idx,
                              kept_cnt, out, out_strides, q_row_sq, k_max_sq, workspace, stream);
}

extern "C" int veda_attend_fp8(const veda_layout* layout, const void* q_codes, const void* k_codes,
                               const float* scales_q, const float* scales_k, const void* v_t, int32_t n_heads,
                               int32_t dim, const int32_t* kept_idx, const int32_t* kept_cnt, void* out,
                               const int64_t out_strides[3], int32_t h_total, const int32_t* heads, void* stream) {
    clear_error();
    return attend_common(layout, q_codes, k_codes, scales_q, scales_k, v_t, n_heads, dim, kept_idx, kept_cnt, out,
                         out_strides, h_total, heads, stream, kQKE4M3);
}

extern "C" int veda_attend_int8(const veda_layout* layout, const void* q_codes, const void* k_codes,
                                const float* scales_q, const float* scales_k, const void* v_t, int32_t n_heads,
                                int32_t dim, const int32_t* kept_idx, const int32_t* kept_cnt, void* out,
                                const int64_t out_strides[3], int32_t h_total, const int32_t* heads, void* stream) {
    clear_error();
    return attend_common(layout, q_codes, k_codes, scales_q, scales_k, v_t, n_heads, dim, kept_idx, kept_cnt, out,
                         out_strides, h_total, heads, stream, kQKI8);
}

extern "C" int veda_attend_fp8_paired(const veda_layout* layout, const void* q_codes, const void* k_codes,
                                      const float* scales_q, const float* scales_k, const void* v_t, int32_t n_heads,
                                      int32_t dim, const int32_t* kept_idx, const int32_t* kept_cnt, void* out,
                                      const int64_t out_strides[3], int32_t h_total, const int32_t* heads,
                                      const float* q_row_sq, const float* k_max_sq, void* workspace,
                                      size_t workspace_bytes, void* stream) {
    clear_error();
    if (int rc = check_paired("veda_attend_fp8_paired", layout, n_heads, q_row_sq, k_max_sq, workspace,
                              workspace_bytes))
        return rc;
    return attend_common(layout, q_codes, k_codes, scales_q, scales_k, v_t, n_heads, dim, kept_idx, kept_cnt, out,
                         out_strides, h_total, heads, stream, kQKE4M3, q_row_sq, k_max_sq, workspace);
}

extern "C" int veda_attend_int8_paired(const veda_layout* layout, const void* q_codes, const void* k_codes,
                                       const float* scales_q, const float* scales_k, const void* v_t, int32_t n_heads,
                                       int32_t dim, const int32_t* kept_idx, const int32_t* kept_cnt, void* out,
                                       const int64_t out_strides[3], int32_t h_total, const int32_t* heads,
                                       const float* q_row_sq, const float* k_max_sq, void* workspace,
                                       size_t workspace_bytes, void* stream) {
    clear_error();
    if (int rc = check_paired("veda_attend_int8_paired", layout, n_heads, q_row_sq, k_max_sq, workspace,
                              workspace_bytes))
        return rc;
    return attend_common(layout, q_codes, k_codes, scales_q, scales_k, v_t, n_heads, dim, kept_idx, kept_cnt, out,
                         out_strides, h_total, heads, stream, kQKI8, q_row_sq, k_max_sq, workspace);
}

static int quantize_codes(const char* who, int code, const veda_layout* layout, const void* x_t, int32_t n_heads,
                          int32_t dim, void* codes, float* scales, void* stream) {
    clear_error();
    if (!layout || !x_t || !codes || !scales) return fail(VEDA_ERR_INVALID, std::string(who) + ": NULL argument");
    if (dim != 64 && dim != 128) return fail(VEDA_ERR_INVALID, std::string(who) + ": head_dim must be 64 or 128");
    if (n_heads <= 0) return fail(VEDA_ERR_INVALID, std::string(who) + ": n_heads must be positive");
    if (!aligned16(x_t) || !aligned16(codes) || !aligned16(scales))
        return fail(VEDA_ERR_INVALID, std::string(who) + ": buffers need 16-byte alignment");
    DeviceState* ds;
    if (int rc = device_state(&ds)) return rc;
    const DeviceCopy* dc;
    if (int rc = device_copy(layout, &dc)) return rc;
    QuantArgs a;
    a.x_t = static_cast<const __nv_bfloat16*>(x_t);
    a.valid_count = dc->valid_count;
    a.codes = static_cast<uint8_t*>(codes);
    a.scales = scales;
    a.n_slots = layout->desc.n_slots;
    a.n_tiles = layout->desc.n_tiles;
    dim3 grid(unsigned(layout->desc.n_tiles), unsigned(n_heads));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (code == kCodeI8) {
        if (dim == 128)
            quantize_kernel<128, kCodeI8><<<grid, 256, 0, s>>>(a);
        else
            quantize_kernel<64, kCodeI8><<<grid, 256, 0, s>>>(a);
    } else {
        if (dim == 128)
            quantize_kernel<128, kCodeE4M3><<<grid, 256, 0, s>>>(a);
        else
            quantize_kernel<64, kCodeE4M3><<<grid, 256, 0, s>>>(a);
    }
    return launch_check("quantize_kernel");
}

extern "C" int veda_quantize_fp8(const veda_layout* layout, const void* x_t, int32_t n_heads, int32_t dim,
                                 void* codes, float* scales, void* stream) {
    return quantize_codes("veda_quantize_fp8", kCodeE4M3, layout, x_t, n_heads, dim, codes, scales, stream);
}

extern "C" int veda_quantize_int8(const veda_layout* layout, const void* x_t, int32_t n_heads, int32_t dim,
                                  void* codes, float* scales, void* stream) {
    return quantize_codes("veda_quantize_int8", kCodeI8, layout, x_t, n_heads, dim, codes, scales, stream);
}

extern "C" int veda_sync_status(void* stream) {
    clear_error();
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int bits = 0;
    e = cudaMemcpyFromSymbol(&bits, g_err, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (bits) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_err, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    }
    if (bits & kErrTimeout) return fail(VEDA_ERR_TIMEOUT, "a bounded device wait expired; the kernel stopped early");
    if (bits & kErrBadList) return fail(VEDA_ERR_BAD_LIST, "a kept list was out of range or not ascending");
    if (bits & kErrBadHead) return fail(VEDA_ERR_INVALID, "a head index was outside [0, H_total)");
    if (bits & kErrLayout) return fail(VEDA_ERR_CUDA, "attend kernel: shared memory base was not 1024-byte aligned");
    return VEDA_OK;
}
