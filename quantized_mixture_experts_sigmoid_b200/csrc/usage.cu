// Expert-usage histogram and the hot-expert order.
//
// [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", section "Learning cache와
// 하드웨어별 기대치": the engine records the experts routing actually picks
// and, at start-up, pins the most used ones in spare RAM (the yodev.dev page
// names the same switches: STATS to record, PIN to pin).  Here the record is a
// per-layer device histogram that routed batches add to, and the pin order is
// that histogram ranked: most used first, ties to the lower expert index.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kUsageThreads = 256;
constexpr int kRankThreads = 1024;

// usage[e] += number of (token, slot) entries routed to e; empty slots (-1)
// and indices outside [0, E) add nothing.
__global__ void __launch_bounds__(kUsageThreads)
k_usage_accumulate(const int32_t* __restrict__ idx, long n, int E, uint32_t* __restrict__ usage) {
    for (long i = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<long>(gridDim.x) * blockDim.x) {
        const int e = idx[i];
        if (e >= 0 && e < E) atomicAdd(usage + e, 1u);
    }
}

// order[r] = the expert of rank r: rank of e = number of experts used more
// often, or as often with a lower index.  One CTA, the counts in shared memory.
__global__ void __launch_bounds__(kRankThreads)
k_usage_rank(const uint32_t* __restrict__ usage, int E, int32_t* __restrict__ order) {
    __shared__ uint32_t u[1024];
    for (int e = threadIdx.x; e < E; e += kRankThreads) u[e] = usage[e];
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kRankThreads) {
        const uint32_t me = u[e];
        int r = 0;
        for (int f = 0; f < E; ++f) r += u[f] > me || (u[f] == me && f < e);
        order[r] = e;
    }
}

}  // namespace

cudaError_t launch_usage_accumulate(const int32_t* idx, long n, int E, uint32_t* usage, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int grid = static_cast<int>(std::min<long>(148, (n + kUsageThreads - 1) / kUsageThreads));
    k_usage_accumulate<<<grid, kUsageThreads, 0, st>>>(idx, n, E, usage);
    return counted(cudaGetLastError());
}

cudaError_t launch_usage_rank(const uint32_t* usage, int E, int32_t* order, cudaStream_t st) {
    k_usage_rank<<<1, kRankThreads, 0, st>>>(usage, E, order);
    return counted(cudaGetLastError());
}

}  // namespace moe
