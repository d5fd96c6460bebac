// Batch union: distinct experts of a batch, their token counts and the
// (token, slot) pairs grouped by expert.
//
// [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", section "구현된 주요 기능",
// batch-union bullet: in prefill and MTP verification every distinct expert
// of the batch is read once and applied to all positions routed to it.  The
// lists built here let every later kernel walk experts, not tokens.
//
// An index of -1 is an empty slot (dropped by adaptive top-p, or a token the
// router could not route): it has no pair.  Any other index outside [0, E)
// records MOE_EDEVICE_INDEX and is left out too, and so is a repeat of an
// expert earlier in the same row (rows must be distinct; a repeat would
// otherwise take the same pair position as its first entry and leave a hole in
// the lists, which later kernels would read as a token).  The pair lists hold the
// valid pairs first (offsets[n_unique] of them); the rest of the T*K entries
// get token 0, slot -1, so a pass that walks all T*K rows reads valid rows.
//
// One CTA: a shared-memory histogram, a block scan for the compacted expert
// list and CSR offsets, then a stable counting sort of the T*K entries in
// chunks of 256 tokens, ranked with per-expert token bitmaps so the pair order
// (expert ascending, token ascending) is deterministic.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace {

constexpr int kUnionThreads = 256;
constexpr int kChunk = 256;              // tokens per placement round
constexpr int kChunkWords = kChunk / 32; // bitmap words per expert

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Whether entry k of a row of top_k indices repeats an earlier entry of the row.
__device__ __forceinline__ bool repeats_earlier(const int32_t* __restrict__ row, int k, int e) {
    for (int j = 0; j < k; ++j)
        if (row[j] == e) return true;
    return false;
}

__global__ void __launch_bounds__(kUnionThreads)
k_union(const int32_t* __restrict__ idx, int T, int K, int E, int32_t* __restrict__ n_unique,
        int32_t* __restrict__ uniq, int32_t* __restrict__ offsets, int32_t* __restrict__ pair_tok,
        int32_t* __restrict__ pair_slot, int32_t* __restrict__ counts, int32_t* status) {
    extern __shared__ int32_t sm[];
    int32_t* cnt = sm;                                           // [E]
    int32_t* cursor = cnt + E;                                   // [E]
    uint32_t* bm = reinterpret_cast<uint32_t*>(cursor + E);      // [E][kChunkWords]
    __shared__ int32_t wc[kUnionThreads / 32], wp[kUnionThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    for (int e = tid; e < E; e += kUnionThreads) cnt[e] = 0;
    __syncthreads();
    const long n = static_cast<long>(T) * K;
    for (long i = tid; i < n; i += kUnionThreads) {
        const int e = idx[i];
        const long t = i / K;
        const int k = static_cast<int>(i - t * K);
        if (e >= 0 && e < E && !repeats_earlier(idx + t * K, k, e)) {
            atomicAdd(&cnt[e], 1);
        } else if (e != -1) {
            record_status(status, MOE_EDEVICE_INDEX);
        }
    }
    __syncthreads();

    // block scan: each thread owns a contiguous run of experts
    const int per = (E + kUnionThreads - 1) / kUnionThreads;
    const int e0 = tid * per, e1 = min(E, e0 + per);
    int csum = 0, psum = 0;
    for (int e = e0; e < e1; ++e) {
        csum += cnt[e];
        psum += cnt[e] > 0;
    }
    const int ci = warp_incl_scan(csum, lane), pi = warp_incl_scan(psum, lane);
    if (lane == 31) {
        wc[warp] = ci;
        wp[warp] = pi;
    }
    __syncthreads();
    int cbase = 0, pbase = 0, ctot = 0, ptot = 0;
    for (int w = 0; w < kUnionThreads / 32; ++w) {
        if (w < warp) {
            cbase += wc[w];
            pbase += wp[w];
        }
        ctot += wc[w];
        ptot += wp[w];
    }
    int c = cbase + ci - csum, p = pbase + pi - psum;
    for (int e = e0; e < e1; ++e) {
        cursor[e] = c;
        if (counts) counts[e] = cnt[e];
        if (cnt[e] > 0) {
            uniq[p] = e;
            offsets[p] = c;
            ++p;
        }
        c += cnt[e];
    }
    if (tid == 0) {
        *n_unique = ptot;
        offsets[ptot] = ctot;
    }
    for (long i = ctot + tid; i < n; i += kUnionThreads) {
        pair_tok[i] = 0;
        pair_slot[i] = -1;
    }
    __syncthreads();

    // stable placement, chunk by chunk
    for (int base = 0; base < T; base += kChunk) {
        for (int i = tid; i < E * kChunkWords; i += kUnionThreads) bm[i] = 0;
        __syncthreads();
        const int t = base + tid;
        const uint32_t mybit = 1u << lane;
        if (t < T) {
            for (int k = 0; k < K; ++k) {
                const int e = idx[static_cast<size_t>(t) * K + k];
                if (e >= 0 && e < E) atomicOr(&bm[e * kChunkWords + warp], mybit);
            }
        }
        __syncthreads();
        if (t < T) {
            for (int k = 0; k < K; ++k) {
                const int e = idx[static_cast<size_t>(t) * K + k];
                if (e < 0 || e >= E || repeats_earlier(idx + static_cast<size_t>(t) * K, k, e)) continue;
                const uint32_t* row = bm + e * kChunkWords;
                int rank = __popc(row[warp] & (mybit - 1u));
                for (int w = 0; w < warp; ++w) rank += __popc(row[w]);
                const int pos = cursor[e] + rank;
                pair_tok[pos] = t;
                pair_slot[pos] = k;
            }
        }
        __syncthreads();
        for (int e = tid; e < E; e += kUnionThreads) {
            int s = 0;
            for (int w = 0; w < kChunkWords; ++w) s += __popc(bm[e * kChunkWords + w]);
            cursor[e] += s;
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_union(const int32_t* idx, int T, int K, int E, int32_t* n_unique, int32_t* uniq,
                         int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot, int32_t* counts,
                         int32_t* status, cudaStream_t st) {
    const size_t smem = sizeof(int32_t) * static_cast<size_t>(E) * (2 + kChunkWords);
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(k_union), smem);
    if (e != cudaSuccess) return e;
    k_union<<<1, kUnionThreads, smem, st>>>(idx, T, K, E, n_unique, uniq, offsets, pair_tok,
                                             pair_slot, counts, status);
    return counted(cudaGetLastError());
}

}  // namespace moe
