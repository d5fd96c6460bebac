// Router: noaux_tc sigmoid routing with renormalised, scaled gate weights.
//
// [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", section "구현된 주요 기능",
// router bullet: DeepSeek-V3-style sigmoid router, noaux_tc,
// routed_scaling_factor.  The reading implemented (DeepSeek-V3's published
// routing): sigmoid scores; a correction bias added for choosing only; group
// score = sum of the two largest biased scores; keep topk_group groups; keep
// top_k experts of kept groups; weights = unbiased scores renormalised over
// the chosen experts, times routed_scaling_factor.
//
// Logits are accumulated in fp64 (bf16 x fp32 products are exact in fp64)
// and rounded once to fp32, so the chosen indices do not depend on the
// summation order used here.
#include "common.cuh"
#include "kernels.cuh"
#include "router_select.cuh"

namespace moe {
namespace {

constexpr int kLogitWarps = 4;

// One warp per (expert, chunk of TT tokens): each lane streams 16-byte pieces
// of the expert's router row and keeps TT fp64 partial sums.
template <int TT>
__global__ void __launch_bounds__(kLogitWarps * 32)
k_router_logits(const uint16_t* __restrict__ x, const float* __restrict__ w, int T, int H, int E,
                float* __restrict__ logits) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * kLogitWarps + warp;
    const int t0 = blockIdx.y * TT;
    if (e >= E) return;
    double acc[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0.0;
    const float4* w4 = reinterpret_cast<const float4*>(w + static_cast<size_t>(e) * H);
    const int n4 = H >> 2;
#pragma unroll 2
    for (int j = lane; j < n4; j += 32) {
        const float4 wv = __ldg(w4 + j);
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t0 + t < T) {
                const uint2 xv = __ldg(reinterpret_cast<const uint2*>(x + static_cast<size_t>(t0 + t) * H) + j);
                acc[t] = fma(static_cast<double>(bf16_bits_to_f32(static_cast<uint16_t>(xv.x))), static_cast<double>(wv.x), acc[t]);
                acc[t] = fma(static_cast<double>(bf16_bits_to_f32(static_cast<uint16_t>(xv.x >> 16))), static_cast<double>(wv.y), acc[t]);
                acc[t] = fma(static_cast<double>(bf16_bits_to_f32(static_cast<uint16_t>(xv.y))), static_cast<double>(wv.z), acc[t]);
                acc[t] = fma(static_cast<double>(bf16_bits_to_f32(static_cast<uint16_t>(xv.y >> 16))), static_cast<double>(wv.w), acc[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
        const double s = warp_sum_f64(acc[t]);
        if (lane == 0 && t0 + t < T) logits[static_cast<size_t>(t0 + t) * E + e] = __double2float_rn(s);
    }
}

constexpr int kSelectWarps = 4;

// One warp per token.  Shared memory per warp: s[E], b[E].
__global__ void __launch_bounds__(kSelectWarps * 32)
k_router_select(const float* __restrict__ logits, int T, const float* __restrict__ bias, int E,
                int G, int TG, int K, float rsf, float top_p, int32_t* __restrict__ topk_idx,
                float* __restrict__ topk_w, int32_t* status) {
    extern __shared__ float sm[];
    __shared__ int chosen[kSelectWarps][32];
    const int warp = threadIdx.x >> 5;
    const int t = blockIdx.x * kSelectWarps + warp;
    if (t >= T) return;
    float* s = sm + static_cast<size_t>(warp) * 2 * E;
    const float* lg = logits + static_cast<size_t>(t) * E;
    select_token_warp([lg](int e) { return lg[e]; }, bias, E, G, TG, K, rsf, top_p, s, s + E,
                      chosen[warp], topk_idx + static_cast<size_t>(t) * K,
                      topk_w + static_cast<size_t>(t) * K, status);
}

}  // namespace

cudaError_t launch_router_logits(const uint16_t* x, int T, int H, const float* w, int E,
                                 float* logits, cudaStream_t st) {
    const dim3 block(kLogitWarps * 32);
    const int gx = (E + kLogitWarps - 1) / kLogitWarps;
    if (T <= 1) {
        k_router_logits<1><<<dim3(gx, T), block, 0, st>>>(x, w, T, H, E, logits);
    } else if (T <= 4) {
        k_router_logits<4><<<dim3(gx, 1), block, 0, st>>>(x, w, T, H, E, logits);
    } else {
        k_router_logits<8><<<dim3(gx, (T + 7) / 8), block, 0, st>>>(x, w, T, H, E, logits);
    }
    return counted(cudaGetLastError());
}

cudaError_t launch_router_select(const float* logits, int T, const float* bias,
                                 const moe_router_cfg& c, int32_t* idx, float* w, int32_t* status,
                                 cudaStream_t st) {
    const size_t smem = sizeof(float) * 2 * static_cast<size_t>(c.n_expert) * kSelectWarps;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(k_router_select), smem);
    if (e != cudaSuccess) return e;
    k_router_select<<<(T + kSelectWarps - 1) / kSelectWarps, kSelectWarps * 32, smem, st>>>(
        logits, T, bias, c.n_expert, c.n_group, c.topk_group, c.top_k, c.routed_scaling_factor, c.top_p, idx, w,
        status);
    return counted(cudaGetLastError());
}

}  // namespace moe
