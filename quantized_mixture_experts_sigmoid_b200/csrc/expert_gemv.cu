// Quantised SwiGLU experts over a batch union: the general (GEMV-style) path.
//
// [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", section "구현된 주요 기능":
// int8 / packed int4 / packed int2 weights with per-row scales and
// dequant-on-use, an integer-dot kernel against Q8_0 int8 activations, and
// batch-union MoE (each distinct expert applied to all its positions).
//
// up/gate kernel: one CTA per (32-row block of h, distinct expert).  It
// stages the Q8_0 activations of up to TC of the expert's tokens in shared
// memory, streams the 32 gate rows and 32 up rows (integer dot per block,
// fp32 promotion), applies SwiGLU and quantises the 32 h values of each token
// to one Q8_0 block, written by pair index.
// down kernel: one CTA per (32 output rows, distinct expert); it streams the
// rows against the staged Q8_0(h) of the expert's pairs and writes y by
// (token, slot).
#include "common.cuh"
#include "kernels.cuh"
#include "quant.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUgRows = 32;    // h rows per up/gate CTA
constexpr int kDownRows = 32;  // output rows per down CTA
constexpr int kUgTok = 8;      // tokens staged per pass (up/gate)
constexpr int kDownTok = 16;   // pairs staged per pass (down)

struct ExpertRange {
    int e, p0, p1;
};

__device__ __forceinline__ bool expert_range(const UnionView& un, int u, int T, ExpertRange& r) {
    if (un.uniq) {
        if (u >= *un.n_unique) return false;
        r.e = un.uniq[u];
        r.p0 = un.offsets[u];
        r.p1 = un.offsets[u + 1];
    } else {
        r.e = 0;
        r.p0 = 0;
        r.p1 = T;
    }
    return true;
}

template <int QT, int TC>
__global__ void __launch_bounds__(kThreads)
k_up_gate(const uint8_t* __restrict__ w_gate, const uint8_t* __restrict__ w_up,
          const float* __restrict__ s_gate, const float* __restrict__ s_up, int H, int I,
          const int8_t* __restrict__ qx, const float* __restrict__ dx, int T, UnionView un,
          int8_t* __restrict__ qh, float* __restrict__ dh) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int nb = H / 32;
    uint4* a0 = reinterpret_cast<uint4*>(smem);
    uint4* a1 = a0 + TC * nb;
    float* ad = reinterpret_cast<float*>(a1 + TC * nb);
    int32_t* as = reinterpret_cast<int32_t*>(ad + TC * nb);
    float* gbuf = reinterpret_cast<float*>(as + TC * nb);
    float* ubuf = gbuf + TC * kUgRows;

    ExpertRange er;
    if (!expert_range(un, blockIdx.y, T, er)) return;
    const int r0 = blockIdx.x * kUgRows;
    const size_t rb = static_cast<size_t>(H) * QT / 8;
    const uint8_t* Wg = w_gate + (static_cast<size_t>(er.e) * I + r0) * rb;
    const uint8_t* Wu = w_up + (static_cast<size_t>(er.e) * I + r0) * rb;
    const float* sg = s_gate + static_cast<size_t>(er.e) * I + r0;
    const float* su = s_up + static_cast<size_t>(er.e) * I + r0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int pc = er.p0; pc < er.p1; pc += TC) {
        const int nt = min(TC, er.p1 - pc);
        for (int i = 0; i < nt; ++i) {
            const int tok = un.uniq ? un.pair_tok[pc + i] : pc + i;
            stage_act_row<QT>(qx + static_cast<size_t>(tok) * H, dx + static_cast<size_t>(tok) * nb,
                              nb, a0 + i * nb, a1 + i * nb, ad + i * nb, as + i * nb, threadIdx.x,
                              kThreads);
        }
        __syncthreads();
        for (int j = warp; j < 2 * kUgRows; j += kWarps) {
            const uint8_t* row = j < kUgRows ? Wg + j * rb : Wu + (j - kUgRows) * rb;
            float acc[TC];
#pragma unroll
            for (int t = 0; t < TC; ++t) acc[t] = 0.0f;
#pragma unroll 2
            for (int b = lane; b < nb; b += 32) {
                const WBlock<QT> w = load_wblock<QT>(row, b);
#pragma unroll
                for (int t = 0; t < TC; ++t) {
                    if (t < nt) {
                        const int isum = block_dot<QT>(w, a0[t * nb + b], a1[t * nb + b], as[t * nb + b]);
                        acc[t] = fmaf(static_cast<float>(isum), ad[t * nb + b], acc[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < TC; ++t) {
                if (t < nt) {
                    const float v = warp_sum_f32(acc[t]);
                    if (lane == 0) {
                        if (j < kUgRows) {
                            gbuf[t * kUgRows + j] = __fmul_rn(v, sg[j]);
                        } else {
                            ubuf[t * kUgRows + j - kUgRows] = __fmul_rn(v, su[j - kUgRows]);
                        }
                    }
                }
            }
        }
        __syncthreads();
        for (int t = warp; t < nt; t += kWarps) {
            const float h = swiglu(gbuf[t * kUgRows + lane], ubuf[t * kUgRows + lane]);
            float db;
            const int8_t q = q8_0_lane(h, &db);
            const size_t p = static_cast<size_t>(pc + t);
            qh[p * I + r0 + lane] = q;
            if (lane == 0) dh[p * (I / 32) + blockIdx.x] = db;
        }
        __syncthreads();
    }
}

template <int QT, int TC>
__global__ void __launch_bounds__(kThreads)
k_down(const uint8_t* __restrict__ w_down, const float* __restrict__ s_down, int H, int I,
       const int8_t* __restrict__ qh, const float* __restrict__ dh, int T, int K, UnionView un,
       float* __restrict__ y_pairs) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int nb = I / 32;
    uint4* a0 = reinterpret_cast<uint4*>(smem);
    uint4* a1 = a0 + TC * nb;
    float* ad = reinterpret_cast<float*>(a1 + TC * nb);
    int32_t* as = reinterpret_cast<int32_t*>(ad + TC * nb);

    ExpertRange er;
    if (!expert_range(un, blockIdx.y, T, er)) return;
    const int c0 = blockIdx.x * kDownRows;
    const size_t rb = static_cast<size_t>(I) * QT / 8;
    const uint8_t* Wd = w_down + (static_cast<size_t>(er.e) * H + c0) * rb;
    const float* sd = s_down + static_cast<size_t>(er.e) * H + c0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int pc = er.p0; pc < er.p1; pc += TC) {
        const int nt = min(TC, er.p1 - pc);
        for (int i = 0; i < nt; ++i) {
            const size_t p = static_cast<size_t>(pc + i);
            stage_act_row<QT>(qh + p * I, dh + p * nb, nb, a0 + i * nb, a1 + i * nb, ad + i * nb,
                              as + i * nb, threadIdx.x, kThreads);
        }
        __syncthreads();
        for (int j = warp; j < kDownRows; j += kWarps) {
            const uint8_t* row = Wd + j * rb;
            float acc[TC];
#pragma unroll
            for (int t = 0; t < TC; ++t) acc[t] = 0.0f;
#pragma unroll 2
            for (int b = lane; b < nb; b += 32) {
                const WBlock<QT> w = load_wblock<QT>(row, b);
#pragma unroll
                for (int t = 0; t < TC; ++t) {
                    if (t < nt) {
                        const int isum = block_dot<QT>(w, a0[t * nb + b], a1[t * nb + b], as[t * nb + b]);
                        acc[t] = fmaf(static_cast<float>(isum), ad[t * nb + b], acc[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < TC; ++t) {
                if (t < nt) {
                    const float v = warp_sum_f32(acc[t]);
                    if (lane == 0) {
                        const int p = pc + t;
                        const int tok = un.uniq ? un.pair_tok[p] : p;
                        const int slot = un.uniq ? un.pair_slot[p] : 0;
                        y_pairs[(static_cast<size_t>(tok) * K + slot) * H + c0 + j] = __fmul_rn(v, sd[j]);
                    }
                }
            }
        }
        __syncthreads();
    }
}

template <int QT>
cudaError_t up_gate_qt(const moe_experts& ex, const int8_t* qx, const float* dx, int T,
                       const UnionView& un, int8_t* qh, float* dh, cudaStream_t st) {
    const int nb = ex.hidden / 32;
    const size_t smem = static_cast<size_t>(kUgTok) * nb * 40 + 2 * kUgTok * kUgRows * sizeof(float);
    auto kern = k_up_gate<QT, kUgTok>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(ex.inter / kUgRows, un.max_unique);
    kern<<<grid, kThreads, smem, st>>>(ex.w_gate, ex.w_up, ex.s_gate, ex.s_up, ex.hidden, ex.inter,
                                       qx, dx, T, un, qh, dh);
    return counted(cudaGetLastError());
}

template <int QT>
cudaError_t down_qt(const moe_experts& ex, const int8_t* qh, const float* dh, int T, int K,
                    const UnionView& un, float* y, cudaStream_t st) {
    const int nb = ex.inter / 32;
    const size_t smem = static_cast<size_t>(kDownTok) * nb * 40;
    auto kern = k_down<QT, kDownTok>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(ex.hidden / kDownRows, un.max_unique);
    kern<<<grid, kThreads, smem, st>>>(ex.w_down, ex.s_down, ex.hidden, ex.inter, qh, dh, T, K, un, y);
    return counted(cudaGetLastError());
}

}  // namespace

cudaError_t launch_expert_up_gate(const moe_experts& ex, const int8_t* qx, const float* dx, int T,
                                  const UnionView& un, int8_t* qh, float* dh, cudaStream_t st) {
    if (un.max_unique <= 0) return cudaSuccess;
    switch (ex.qtype) {
        case MOE_Q_INT4: return up_gate_qt<4>(ex, qx, dx, T, un, qh, dh, st);
        case MOE_Q_INT8: return up_gate_qt<8>(ex, qx, dx, T, un, qh, dh, st);
        case MOE_Q_INT2: return up_gate_qt<2>(ex, qx, dx, T, un, qh, dh, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_expert_down(const moe_experts& ex, const int8_t* qh, const float* dh, int T,
                               int top_k, const UnionView& un, float* y, cudaStream_t st) {
    if (un.max_unique <= 0) return cudaSuccess;
    switch (ex.qtype) {
        case MOE_Q_INT4: return down_qt<4>(ex, qh, dh, T, top_k, un, y, st);
        case MOE_Q_INT8: return down_qt<8>(ex, qh, dh, T, top_k, un, y, st);
        case MOE_Q_INT2: return down_qt<2>(ex, qh, dh, T, top_k, un, y, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
