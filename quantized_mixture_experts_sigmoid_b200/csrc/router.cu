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
#pragma unroll 8  // eight 16-byte loads of the row in flight per lane
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

// Batches (T >= kTiledMinT): a register-blocked fp64 GEMM.  A CTA computes
// 64 tokens x 64 experts, each thread 4 x 4 of them; x and W pass through
// shared memory in chunks of 16 along H, converted to fp64 once (double
// buffered).  Every logit is accumulated by one thread in ascending h, the
// order of the plain definition, so the fp64 sum is that of the definition.
// The W chunk is stored with each thread's expert pairs side by side across
// threads ([pair][thread][2]), so a warp's 16-byte loads of it are contiguous.
constexpr int kTiledMinT = 32;
constexpr int kTM = 64, kTN = 64, kKC = 16, kTiledThreads = 256;
static_assert(kTM == 64 && kTN == 64 && kTiledThreads == 256 && kKC % 4 == 0,
              "thread (ty, tx) = (tid / 16, tid % 16) owns tokens 4 ty.. and experts 4 tx..; the loader covers 64 rows");

__global__ void __launch_bounds__(kTiledThreads)
k_router_logits_tiled(const uint16_t* __restrict__ x, const float* __restrict__ w, int T, int H, int E,
                      float* __restrict__ logits) {
    __shared__ __align__(16) double xs[2][kKC][kTM];  // [stage][h][token]
    __shared__ __align__(16) double wsm[2][kKC][kTN]; // [stage][h][expert pair half][thread][2]
    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * kTM, e0 = blockIdx.y * kTN;
    const int ty = tid >> 4, tx = tid & 15;  // tokens 4 ty .. 4 ty + 3, experts 4 tx .. 4 tx + 3
    // loader: 64 rows x 16 values per operand per chunk; thread tid loads row tid / 4,
    // values 4 (tid % 4) .. + 3 of x and of W
    const int lr = tid >> 2, lc = (tid & 3) * 4;
    const bool xin = t0 + lr < T, win = e0 + lr < E;
    const uint16_t* xrow = x + static_cast<size_t>(xin ? t0 + lr : 0) * H + lc;
    const float* wrow = w + static_cast<size_t>(win ? e0 + lr : 0) * H + lc;
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    uint2 xr = xin ? __ldg(reinterpret_cast<const uint2*>(xrow)) : make_uint2(0, 0);
    float4 wr = win ? __ldg(reinterpret_cast<const float4*>(wrow)) : make_float4(0.f, 0.f, 0.f, 0.f);
    const int nk = H / kKC;
    for (int kc = 0; kc < nk; ++kc) {
        const int st = kc & 1;
        xs[st][lc + 0][lr] = static_cast<double>(bf16_bits_to_f32(static_cast<uint16_t>(xr.x)));
        xs[st][lc + 1][lr] = static_cast<double>(bf16_bits_to_f32(static_cast<uint16_t>(xr.x >> 16)));
        xs[st][lc + 2][lr] = static_cast<double>(bf16_bits_to_f32(static_cast<uint16_t>(xr.y)));
        xs[st][lc + 3][lr] = static_cast<double>(bf16_bits_to_f32(static_cast<uint16_t>(xr.y >> 16)));
        const int wc = ((lr & 3) >> 1) * (kTN / 2) + (lr >> 2) * 2 + (lr & 1);  // expert lr of the tile
        wsm[st][lc + 0][wc] = static_cast<double>(wr.x);
        wsm[st][lc + 1][wc] = static_cast<double>(wr.y);
        wsm[st][lc + 2][wc] = static_cast<double>(wr.z);
        wsm[st][lc + 3][wc] = static_cast<double>(wr.w);
        __syncthreads();
        if (kc + 1 < nk) {  // the next chunk's values, in flight during this chunk's products
            xr = xin ? __ldg(reinterpret_cast<const uint2*>(xrow + (kc + 1) * kKC)) : make_uint2(0, 0);
            wr = win ? __ldg(reinterpret_cast<const float4*>(wrow + (kc + 1) * kKC)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kKC; ++k) {
            const double2 a01 = *reinterpret_cast<const double2*>(&xs[st][k][4 * ty]);
            const double2 a23 = *reinterpret_cast<const double2*>(&xs[st][k][4 * ty + 2]);
            const double2 b01 = *reinterpret_cast<const double2*>(&wsm[st][k][2 * tx]);
            const double2 b23 = *reinterpret_cast<const double2*>(&wsm[st][k][kTN / 2 + 2 * tx]);
            const double a[4] = {a01.x, a01.y, a23.x, a23.y}, bb[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], bb[j], acc[i][j]);
        }
        // the stage written next iteration was read two chunks ago: one barrier per chunk suffices
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + 4 * ty + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + 4 * tx + j;
            if (e < E) logits[static_cast<size_t>(t) * E + e] = __double2float_rn(acc[i][j]);
        }
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
    } else if (T >= kTiledMinT && H % kKC == 0) {
        k_router_logits_tiled<<<dim3((T + kTM - 1) / kTM, (E + kTN - 1) / kTN), kTiledThreads, 0, st>>>(
            x, w, T, H, E, logits);
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
