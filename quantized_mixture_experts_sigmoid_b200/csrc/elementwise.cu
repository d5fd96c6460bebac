// Q8_0 activation quantiser and the weighted combine.
//
// Q8_0: [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", section "구현된 주요
// 기능", integer-dot bullet (Q8_0-style int8 activations).  Blocks of 32, one
// fp32 scale d = max|v| / 127, q = round(v / d) half away from zero.
// Combine: same section, router bullet (shared expert, routed_scaling_factor):
// out = shared + sum_k w_k * y_k in fp32, slot order, then bf16 or fp32.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

// One warp per 32-value block, one value per lane.
template <bool BF16>
__global__ void __launch_bounds__(256)
k_q8_0(const void* __restrict__ v, long nblocks, int8_t* __restrict__ q, float* __restrict__ d) {
    const int lane = threadIdx.x & 31;
    const long gw = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long nw = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
    for (long b = gw; b < nblocks; b += nw) {
        float x;
        if (BF16) {
            x = bf16_bits_to_f32(static_cast<const uint16_t*>(v)[b * 32 + lane]);
        } else {
            x = static_cast<const float*>(v)[b * 32 + lane];
        }
        float db;
        const int8_t qq = q8_0_lane(x, &db);
        q[b * 32 + lane] = qq;
        if (lane == 0) d[b] = db;
    }
}

// out[t][c] = shared[t][c] + sum_k w[t][k] * y[t][k][c] in slot order, slots of
// weight 0 skipped (empty slots: their y is never written); four columns per thread.
template <bool BF16_OUT>
__global__ void __launch_bounds__(256)
k_combine(const float* __restrict__ y, const float* __restrict__ w, const float* __restrict__ sy,
          int T, int K, int H, void* __restrict__ out) {
    const int h4 = H >> 2;
    const long n = static_cast<long>(T) * h4;
    for (long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<long>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>(i / h4), c4 = static_cast<int>(i % h4);
        float4 o = sy ? reinterpret_cast<const float4*>(sy + static_cast<size_t>(t) * H)[c4]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < K; ++k) {
            const float wk = w[static_cast<size_t>(t) * K + k];
            if (wk == 0.0f) continue;  // an empty slot: its y is not read
            const float4 yk = reinterpret_cast<const float4*>(y + (static_cast<size_t>(t) * K + k) * H)[c4];
            o.x = __fadd_rn(o.x, __fmul_rn(wk, yk.x));
            o.y = __fadd_rn(o.y, __fmul_rn(wk, yk.y));
            o.z = __fadd_rn(o.z, __fmul_rn(wk, yk.z));
            o.w = __fadd_rn(o.w, __fmul_rn(wk, yk.w));
        }
        if (BF16_OUT) {
            uint2 pk;
            pk.x = static_cast<uint32_t>(f32_to_bf16_bits(o.x)) | (static_cast<uint32_t>(f32_to_bf16_bits(o.y)) << 16);
            pk.y = static_cast<uint32_t>(f32_to_bf16_bits(o.z)) | (static_cast<uint32_t>(f32_to_bf16_bits(o.w)) << 16);
            reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + static_cast<size_t>(t) * H)[c4] = pk;
        } else {
            reinterpret_cast<float4*>(static_cast<float*>(out) + static_cast<size_t>(t) * H)[c4] = o;
        }
    }
}

int grid_cap(long work, int per_block) {
    long g = (work + per_block - 1) / per_block;
    if (g > 148L * 16) g = 148L * 16;
    return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_q8_0(const void* v, bool bf16, long rows, int n, int8_t* q, float* d,
                        cudaStream_t st) {
    const long nblocks = rows * (n / 32);
    if (nblocks == 0) return cudaSuccess;
    const int g = grid_cap(nblocks, 8);
    if (bf16) {
        k_q8_0<true><<<g, 256, 0, st>>>(v, nblocks, q, d);
    } else {
        k_q8_0<false><<<g, 256, 0, st>>>(v, nblocks, q, d);
    }
    return counted(cudaGetLastError());
}

cudaError_t launch_combine(const float* y, const float* w, const float* shared_y, int T, int K,
                           int H, void* out, int out_dtype, cudaStream_t st) {
    const long n = static_cast<long>(T) * (H / 4);
    if (n == 0) return cudaSuccess;
    const int g = grid_cap(n, 256);
    if (out_dtype == MOE_OUT_BF16) {
        k_combine<true><<<g, 256, 0, st>>>(y, w, shared_y, T, K, H, out);
    } else {
        k_combine<false><<<g, 256, 0, st>>>(y, w, shared_y, T, K, H, out);
    }
    return counted(cudaGetLastError());
}

}  // namespace moe
