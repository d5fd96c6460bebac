// moe_route_noalloc: the router without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they route:
// code that runs while a stream is being captured into a CUDA graph, an
// inference-engine plugin whose enqueue step is not allowed to allocate, or a
// latency-critical loop that cannot pay for cudaMalloc's implicit device
// synchronisation.  This entry point serves them by keeping the router's only
// scratch buffer (the fp32 logits) in a fixed-size array in device memory that
// belongs to the library itself.  The array is statically sized, so every GPU
// that loads the library holds it until the process exits.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace {

// Logits scratch shared by every call of moe_route_noalloc in the process.
static __device__ __align__(256) float g_route_scratch[MOE_ROUTE_NOALLOC_MAX_LOGITS];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device.  The name g_route_scratch means a host-side shadow in host code,
// so its device address must come from cudaGetSymbolAddress.
cudaError_t scratch_for_current_device(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int moe_route_noalloc(const uint16_t* x, int T, int H, const float* w_router,
                                 const float* bias, const moe_router_cfg* cfg, int32_t* topk_idx,
                                 float* topk_w, moe_stream_t stream) {
    const int rc = moe::check_cfg(cfg);  // the same limits as moe_route
    if (rc) return rc;
    const int E = cfg->n_expert;
    if (T < 0 || H <= 0 || H % 32) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (static_cast<long long>(T) * E > MOE_ROUTE_NOALLOC_MAX_LOGITS) return MOE_ETOO_LARGE;
    if (!x || !w_router || !bias || !topk_idx || !topk_w || !aligned16(x) || !aligned16(w_router) ||
        !aligned16(bias) || !aligned16(topk_idx) || !aligned16(topk_w))
        return MOE_EINVAL;
    float* logits = nullptr;
    if (scratch_for_current_device(&logits) != cudaSuccess) return MOE_ECUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // Every logit is written before it is read, so nothing needs clearing.
    if (moe::launch_router_logits(x, T, H, w_router, E, logits, st) != cudaSuccess) return MOE_ECUDA;
    if (moe::launch_router_select(logits, T, bias, *cfg, topk_idx, topk_w, nullptr, st) != cudaSuccess)
        return MOE_ECUDA;
    return MOE_OK;
}
