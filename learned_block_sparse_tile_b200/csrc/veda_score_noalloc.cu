// veda_score_noalloc: the tile-pair logits of veda_score for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc, or any allocator, at the moment they need the scores: plugin hosts
// whose device memory is owned and budgeted by the host application's own pool (a plugin may not grow it),
// and real-time loops where an allocation is not allowed because it can block on, or synchronise with,
// the device. veda_score asks its caller for a workspace; this entry point instead keeps that scratch (the
// projected query and key features and the transposed projections) in one fixed array in this library's
// device memory, and the caller passes only its inputs and outputs.
//
// The scratch is a file-scope __device__ array of kScratchFloats floats (4 MiB). Every GPU that loads
// the library holds it until the process exits. All calls on a device share it; it keeps whatever the
// last call left there. Nothing in it must start at zero: each head chunk's projections are written in
// full before the scores read them. Calls whose kernels overlap on the GPU (for example on two streams
// at once) race on the array and give wrong results; serialise them.
//
// The first call on a device looks up the array's device address (cudaGetSymbolAddress) and keeps it for
// the life of the process; make that first call before any stream capture. The kept address belongs to
// the device's current context: after cudaDeviceReset (or any teardown of the primary context) it is
// stale, so this entry point must not be called again in that process.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <string>

#include "veda_internal.h"

namespace {

constexpr size_t kScratchFloats = size_t(1) << 20;  // 4 MiB per GPU

// In host code this name is only a host-side stand-in for the array: handing it to a kernel would fault
// (or, where the GPU can reach host memory, use the wrong memory). Host code uses the device address
// that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) float g_score_scratch[kScratchFloats];

std::mutex g_mu;
float* g_scratch_addr[veda::kMaxDevices];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" int veda_score_noalloc(const veda_layout* layout, const float* feats_q, const float* feats_k,
                                  int32_t n_heads, int32_t dim, const float* proj_q, const float* proj_k,
                                  float* scores, void* stream) {
    veda::clear_error();
    if (!layout || !feats_q || !feats_k || !proj_q || !proj_k || !scores)
        return veda::fail(VEDA_ERR_INVALID, "veda_score_noalloc: NULL argument");
    if (dim != 64 && dim != 128) return veda::fail(VEDA_ERR_INVALID, "veda_score_noalloc: head_dim must be 64 or 128");
    if (n_heads <= 0) return veda::fail(VEDA_ERR_INVALID, "veda_score_noalloc: n_heads must be positive");
    if (!aligned16(feats_q) || !aligned16(feats_k) || !aligned16(proj_q) || !aligned16(proj_k) || !aligned16(scores))
        return veda::fail(VEDA_ERR_INVALID, "veda_score_noalloc: buffers need 16-byte alignment");
    const int64_t nv = layout->desc.n_video;
    const size_t per_head = size_t(veda::score_scratch_per_head(nv, dim));
    if (per_head > kScratchFloats)
        return veda::fail(VEDA_ERR_UNSUPPORTED,
                          "veda_score_noalloc: one head needs 2 * n_video * head_dim + 6 * head_dim^2 = " +
                              std::to_string(per_head) +
                              " floats of scratch but the static scratch holds " + std::to_string(kScratchFloats) +
                              " (4 MiB); use veda_score with a caller-provided workspace");
    if (int rc = veda_device_check()) return rc;

    // set-up, once per device, with that device current: the device address of the scratch array
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return veda::fail(VEDA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    if (dev < 0 || dev >= veda::kMaxDevices)
        return veda::fail(VEDA_ERR_UNSUPPORTED, "device ordinal beyond the library's table");
    float* base = nullptr;
    {
        std::lock_guard<std::mutex> g(g_mu);
        if (!g_scratch_addr[dev]) {
            float* p = nullptr;
            e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_score_scratch);
            if (e != cudaSuccess)
                return veda::fail(VEDA_ERR_CUDA, std::string("cudaGetSymbolAddress(score scratch): ") + cudaGetErrorString(e));
            g_scratch_addr[dev] = p;
        }
        base = g_scratch_addr[dev];
    }

    // heads in chunks that fit the scratch; kernels of one call run in stream order, so a chunk's scores
    // have read the scratch before the next chunk's projections overwrite it
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int chunk = int(kScratchFloats / per_head);
    for (int h0 = 0; h0 < n_heads; h0 += chunk) {
        const int hc = std::min(chunk, n_heads - h0);
        float* qh = base;
        float* kh = qh + int64_t(hc) * nv * dim;
        float* pt_q = kh + int64_t(hc) * nv * dim;
        float* pt_k = pt_q + int64_t(hc) * 3 * dim * dim;
        if (int rc = veda::launch_score_gemms(feats_q + int64_t(h0) * nv * 3 * dim, feats_k + int64_t(h0) * nv * 3 * dim,
                                              proj_q + int64_t(h0) * 3 * dim * dim, proj_k + int64_t(h0) * 3 * dim * dim,
                                              qh, kh, pt_q, pt_k, scores + int64_t(h0) * nv * nv, int(nv), dim, hc, s))
            return rc;
    }
    return VEDA_OK;
}
