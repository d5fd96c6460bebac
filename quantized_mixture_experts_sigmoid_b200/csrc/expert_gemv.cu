// Quantised SwiGLU experts over a batch union: the general (GEMV-style) path.
//
// [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", section "구현된 주요 기능":
// int8 / packed int4 / packed int2 weights with per-row scales and
// dequant-on-use, an integer-dot kernel against Q8_0 int8 activations, and
// batch-union MoE (each distinct expert applied to all its positions).
//
// Every weight row is consumed by one lane, which folds the row's 32-code
// blocks in ascending order with one fp32 fused multiply-add per block: the
// quantised dot of the layer's definition, bit for bit (a one-ulp difference in
// h could flip a Q8_0 code of h).  The CTA's weight rows pass through shared
// memory in chunks, loaded with coalesced 16-byte (int2: 8-byte) reads one
// chunk ahead in registers: a lane streaming its own row through L1 would need
// more L1 than the SM has beside the staging buffers.  With grouped weight
// scales ([MO] "int4 양자화 (Quantization)의 품질 비용") block b's factor is
// d_b * s[g(b)], rounded once, and the row has no separate scale.
//
// up/gate kernel: one CTA per (group of h rows, distinct expert).  It stages
// the Q8_0 activations of a pass's tokens in shared memory; warp w takes the
// gate (w even) or up (w odd) rows of its 32-row group, lane r row r, for its
// tokens; then SwiGLU and Q8_0 of each token's 32 h values give one Q8_0 block,
// written by pair index.
// down kernel: one CTA per (group of output rows, distinct expert); warp w
// takes its rows and pairs, lane r output row r; y is written by (token, slot).
// The CTA geometry (how many rows, how many tokens a pass) is narrow or wide,
// below.  A shared expert of the routed experts' shape can ride along as grid
// row 0 of both launches.
#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"
#include "quant.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTpw = 2;  // tokens (pairs) per warp and pass

// CTA geometry.  Narrow: the 8 warps split into 4 token groups of 2 (up/gate:
// 32 h rows; down: 8 groups over 32 output rows), for experts that see many
// tokens.  Wide: every warp takes its own 32 rows (up/gate: 128 h rows; down:
// 256 output rows) and the CTA two tokens a pass, for batches whose experts
// see one or two tokens each: then no warp idles while the others compute.
template <bool W>
struct UgGeom {
    static constexpr int kRq = W ? 4 : 1;              // 32-row groups of h per CTA
    static constexpr int kTg = 4 / kRq;                // token groups
    static constexpr int kRows = 32 * kRq;             // h rows per CTA
    static constexpr int kTok = kTg * kTpw;            // tokens staged per pass
};
template <bool W>
struct DownGeom {
    static constexpr int kRd = W ? 8 : 1;              // 32-row groups of output per CTA
    static constexpr int kPg = kWarps / kRd;           // pair groups
    static constexpr int kRows = 32 * kRd;             // output rows per CTA
    static constexpr int kTok = kPg * kTpw;            // pairs staged per pass
};

// Chunk c of NR weight rows (a row's bytes kBytesPerRow per chunk: kChunkBlocks
// blocks), staged through registers into shared memory rows of kStride bytes.
// Thread tid takes pieces tid, tid + kThreads, ... in row-major order, so a
// warp reads contiguous bytes of a row.  Pieces past the end of a row (a last,
// partial chunk) read nothing.
template <int QT, int NR, int kBytesPerRow>
struct WeightChunk {
    static constexpr int kPiece = QT == 2 ? 8 : 16;           // one int2 block, or 16 bytes
    static constexpr int kChunkBytes = kBytesPerRow;
    static constexpr int kChunkBlocks = kChunkBytes / (4 * QT);
    static constexpr int kStride = kChunkBytes + kPiece;       // padded: conflict-free lane-per-row reads
    static constexpr int kPieces = kChunkBytes / kPiece;       // pieces per row per chunk
    static constexpr int kPerThread = NR * kPieces / kThreads;
    static constexpr int kBytes = NR * kStride;                // shared memory
    static_assert(NR * kPieces % kThreads == 0 && kChunkBytes % (4 * QT) == 0, "whole pieces and blocks");
    using Piece = typename std::conditional<QT == 2, uint2, uint4>::type;
    Piece v[kPerThread];

    template <class RowPtr>
    __device__ __forceinline__ void load(const RowPtr& row_ptr, size_t row_bytes, int c) {
#pragma unroll
        for (int j = 0; j < kPerThread; ++j) {
            const int u = j * kThreads + static_cast<int>(threadIdx.x);
            const int r = u / kPieces, pc = u % kPieces;
            const size_t off = static_cast<size_t>(c) * kChunkBytes + static_cast<size_t>(pc) * kPiece;
            v[j] = off < row_bytes ? __ldg(reinterpret_cast<const Piece*>(row_ptr(r) + off)) : Piece{};
        }
    }
    __device__ __forceinline__ void store(uint8_t* dst) const {
#pragma unroll
        for (int j = 0; j < kPerThread; ++j) {
            const int u = j * kThreads + static_cast<int>(threadIdx.x);
            const int r = u / kPieces, pc = u % kPieces;
            *reinterpret_cast<Piece*>(dst + r * kStride + pc * kPiece) = v[j];
        }
    }
};
// Narrow CTAs stage 32 blocks of a row per chunk; wide ones (four or eight
// times the rows) 256 bytes of a row.
template <int QT, int NR, bool W>
using ChunkOf = WeightChunk<QT, NR, W ? 256 : 32 * 4 * QT>;

template <int QT>
__device__ __forceinline__ WBlock<QT> wblock_staged(const uint8_t* row, int i) {
    WBlock<QT> r;
    if constexpr (QT == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(row + 8 * i);
        r.w[0] = v.x;
        r.w[1] = v.y;
    } else {
#pragma unroll
        for (int h = 0; h < QT / 4; ++h) {
            const uint4 v = *reinterpret_cast<const uint4*>(row + 16 * (QT / 4 * i + h));
            r.w[4 * h] = v.x; r.w[4 * h + 1] = v.y; r.w[4 * h + 2] = v.z; r.w[4 * h + 3] = v.w;
        }
    }
    return r;
}

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

// Lane-per-row quantised dots of one weight row against TPW staged activation
// rows (t0 .. t0 + nt - 1 of the staging area), blocks b0 .. b0 + nbc - 1 of
// the row (its staged chunk `row`): blocks ascending, one fused multiply-add
// per block, accumulated into acc (the sums before any per-row scale).  sg:
// the row's grouped scales (gpb blocks per group), or null for per-row scales.
template <int QT, int TPW>
__device__ __forceinline__ void row_dots_chunk(const uint8_t* row, int b0, int nbc, int nb, const uint4* a0,
                                               const uint4* a1, const float* ad, const int32_t* as, int t0,
                                               int nt, const float* sg, int gpb, float (&acc)[TPW]) {
#pragma unroll 4
    for (int i = 0; i < nbc; ++i) {
        const int b = b0 + i;
        const WBlock<QT> w = wblock_staged<QT>(row, i);
        const float gw = sg ? __ldg(sg + b / gpb) : 1.0f;
#pragma unroll
        for (int t = 0; t < TPW; ++t) {
            if (t < nt) {
                const int q = (t0 + t) * nb + b;
                const float f = sg ? __fmul_rn(ad[q], gw) : ad[q];
                acc[t] = fmaf(static_cast<float>(block_dot<QT>(w, a0[q], a1[q], as[q])), f, acc[t]);
            }
        }
    }
}

template <int QT, bool W>
__global__ void __launch_bounds__(kThreads, QT == 4 ? 2 : 1)  // int4: two CTAs an SM (measured 3% faster)
k_up_gate(const uint8_t* __restrict__ w_gate, const uint8_t* __restrict__ w_up,
          const float* __restrict__ s_gate, const float* __restrict__ s_up, int H, int I, int gs,
          const int8_t* __restrict__ qx, const float* __restrict__ dx, int T, UnionView un,
          int8_t* __restrict__ qh, float* __restrict__ dh, SharedUpGate sx) {
    using Geo = UgGeom<W>;
    using Chunk = ChunkOf<QT, 2 * Geo::kRows, W>;  // the CTA's gate rows, then its up rows
    extern __shared__ __align__(16) uint8_t smem[];
    const int nb = H / 32;
    uint8_t* wsm = smem;
    uint4* a0 = reinterpret_cast<uint4*>(smem + Chunk::kBytes);
    uint4* a1 = a0 + Geo::kTok * nb;
    float* ad = reinterpret_cast<float*>(a1 + Geo::kTok * nb);
    int32_t* as = reinterpret_cast<int32_t*>(ad + Geo::kTok * nb);
    float* gbuf = reinterpret_cast<float*>(as + Geo::kTok * nb);
    float* ubuf = gbuf + Geo::kTok * Geo::kRows;

    // grid row 0 is the shared expert when it rides along (all T tokens), the
    // others the union's experts
    const bool shared = sx.w_gate && blockIdx.y == 0;
    ExpertRange er;
    if (shared) {
        er = ExpertRange{0, 0, T};
        w_gate = sx.w_gate; w_up = sx.w_up; s_gate = sx.s_gate; s_up = sx.s_up; qh = sx.qh; dh = sx.dh;
    } else if (!expert_range(un, blockIdx.y - (sx.w_gate ? 1 : 0), T, er)) {
        return;
    }
    const bool dense = shared || !un.uniq;  // rows are tokens, not union pairs
    const int r0 = blockIdx.x * Geo::kRows;
    const size_t rb = static_cast<size_t>(H) * QT / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m = warp & 1, g = warp >> 1, rq = g % Geo::kRq, tg = g / Geo::kRq;  // gate / up; rows; tokens
    const int hr = rq * 32 + lane;  // this lane's h row within the CTA
    const size_t row = static_cast<size_t>(er.e) * I + r0 + hr;
    const uint8_t* gate0 = w_gate + (static_cast<size_t>(er.e) * I + r0) * rb;
    const uint8_t* up0 = w_up + (static_cast<size_t>(er.e) * I + r0) * rb;
    const auto row_ptr = [&](int r) { return r < Geo::kRows ? gate0 + r * rb : up0 + (r - Geo::kRows) * rb; };
    const uint8_t* wrow = wsm + (m * Geo::kRows + hr) * Chunk::kStride;
    const int nchunks = (nb + Chunk::kChunkBlocks - 1) / Chunk::kChunkBlocks;
    const float* sbase = m == 0 ? s_gate : s_up;
    const float* sg = gs ? sbase + row * (H / gs) : nullptr;  // grouped: the row's scales
    const float srow = gs ? 1.0f : __ldg(sbase + row);
    float* dst = m == 0 ? gbuf : ubuf;

    for (int pc = er.p0; pc < er.p1; pc += Geo::kTok) {
        const int nt = min(Geo::kTok, er.p1 - pc);
        for (int i = 0; i < nt; ++i) {
            const int tok = dense ? pc + i : un.pair_tok[pc + i];
            stage_act_row<QT>(qx + static_cast<size_t>(tok) * H, dx + static_cast<size_t>(tok) * nb,
                              nb, a0 + i * nb, a1 + i * nb, ad + i * nb, as + i * nb, threadIdx.x,
                              kThreads);
        }
        const int t0 = tg * kTpw, ntw = min(kTpw, nt - t0);
        float acc[kTpw];
#pragma unroll
        for (int t = 0; t < kTpw; ++t) acc[t] = 0.0f;
        Chunk wc;
        wc.load(row_ptr, rb, 0);
        for (int c = 0; c < nchunks; ++c) {
            __syncthreads();  // activations staged; the previous chunk consumed
            wc.store(wsm);
            __syncthreads();
            if (c + 1 < nchunks) wc.load(row_ptr, rb, c + 1);  // in flight while this chunk is used
            const int b0 = c * Chunk::kChunkBlocks;
            if (ntw > 0)
                row_dots_chunk<QT, kTpw>(wrow, b0, min(Chunk::kChunkBlocks, nb - b0), nb, a0, a1, ad, as, t0, ntw,
                                         sg, gs / 32, acc);
        }
        if (ntw > 0) {
#pragma unroll
            for (int t = 0; t < kTpw; ++t)
                if (t < ntw) dst[(t0 + t) * Geo::kRows + hr] = gs ? acc[t] : __fmul_rn(acc[t], srow);
        }
        __syncthreads();
        // SwiGLU and Q8_0 of each token's 32-row groups of h (one warp a group)
        for (int i = warp; i < nt * Geo::kRq; i += kWarps) {
            const int t = i / Geo::kRq, q = i % Geo::kRq;
            const float h = swiglu(gbuf[t * Geo::kRows + q * 32 + lane], ubuf[t * Geo::kRows + q * 32 + lane]);
            float db;
            const int8_t qv = q8_0_lane(h, &db);
            const size_t p = static_cast<size_t>(pc + t);
            qh[p * I + r0 + q * 32 + lane] = qv;
            if (lane == 0) dh[p * (I / 32) + r0 / 32 + q] = db;
        }
        __syncthreads();
    }
}

template <int QT, bool W>
__global__ void __launch_bounds__(kThreads, QT == 4 ? 2 : 1)  // int4: two CTAs an SM (measured 3% faster)
k_down(const uint8_t* __restrict__ w_down, const float* __restrict__ s_down, int H, int I, int gs,
       const int8_t* __restrict__ qh, const float* __restrict__ dh, int T, int K, UnionView un,
       float* __restrict__ y_pairs, SharedDown sx) {
    using Geo = DownGeom<W>;
    using Chunk = ChunkOf<QT, Geo::kRows, W>;
    extern __shared__ __align__(16) uint8_t smem[];
    const int nb = I / 32;
    uint8_t* wsm = smem;
    uint4* a0 = reinterpret_cast<uint4*>(smem + Chunk::kBytes);
    uint4* a1 = a0 + Geo::kTok * nb;
    float* ad = reinterpret_cast<float*>(a1 + Geo::kTok * nb);
    int32_t* as = reinterpret_cast<int32_t*>(ad + Geo::kTok * nb);

    // grid row 0 is the shared expert when it rides along (all T tokens, one slot)
    const bool shared = sx.w_down && blockIdx.y == 0;
    ExpertRange er;
    if (shared) {
        er = ExpertRange{0, 0, T};
        w_down = sx.w_down; s_down = sx.s_down; qh = sx.qh; dh = sx.dh; y_pairs = sx.y; K = 1;
    } else if (!expert_range(un, blockIdx.y - (sx.w_down ? 1 : 0), T, er)) {
        return;
    }
    const bool dense = shared || !un.uniq;  // rows are tokens, not union pairs
    const int c0 = blockIdx.x * Geo::kRows;
    const size_t rb = static_cast<size_t>(I) * QT / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rg = warp % Geo::kRd, pg = warp / Geo::kRd;  // rows; pairs
    const int orow = rg * 32 + lane;  // this lane's output row within the CTA
    const size_t row = static_cast<size_t>(er.e) * H + c0 + orow;
    const uint8_t* down0 = w_down + (static_cast<size_t>(er.e) * H + c0) * rb;
    const auto row_ptr = [&](int r) { return down0 + r * rb; };
    const uint8_t* wrow = wsm + orow * Chunk::kStride;
    const int nchunks = (nb + Chunk::kChunkBlocks - 1) / Chunk::kChunkBlocks;
    const float* sg = gs ? s_down + row * (I / gs) : nullptr;  // grouped: the row's scales
    const float srow = gs ? 1.0f : __ldg(s_down + row);

    for (int pc = er.p0; pc < er.p1; pc += Geo::kTok) {
        const int nt = min(Geo::kTok, er.p1 - pc);
        for (int i = 0; i < nt; ++i) {
            const size_t p = static_cast<size_t>(pc + i);
            stage_act_row<QT>(qh + p * I, dh + p * nb, nb, a0 + i * nb, a1 + i * nb, ad + i * nb,
                              as + i * nb, threadIdx.x, kThreads);
        }
        const int t0 = pg * kTpw, ntw = min(kTpw, nt - t0);
        float acc[kTpw];
#pragma unroll
        for (int t = 0; t < kTpw; ++t) acc[t] = 0.0f;
        Chunk wc;
        wc.load(row_ptr, rb, 0);
        for (int c = 0; c < nchunks; ++c) {
            __syncthreads();  // activations staged; the previous chunk consumed
            wc.store(wsm);
            __syncthreads();
            if (c + 1 < nchunks) wc.load(row_ptr, rb, c + 1);
            const int b0 = c * Chunk::kChunkBlocks;
            if (ntw > 0)
                row_dots_chunk<QT, kTpw>(wrow, b0, min(Chunk::kChunkBlocks, nb - b0), nb, a0, a1, ad, as, t0, ntw,
                                         sg, gs / 32, acc);
        }
        if (ntw > 0) {
#pragma unroll
            for (int t = 0; t < kTpw; ++t) {
                if (t < ntw) {
                    const int p = pc + t0 + t;
                    const int tok = dense ? p : un.pair_tok[p];
                    const int slot = dense ? 0 : un.pair_slot[p];
                    y_pairs[(static_cast<size_t>(tok) * K + slot) * H + c0 + orow] = gs ? acc[t] : __fmul_rn(acc[t], srow);
                }
            }
        }
        __syncthreads();
    }
}

template <int QT, bool W>
cudaError_t up_gate_qt(const moe_experts& ex, const int8_t* qx, const float* dx, int T,
                       const UnionView& un, int8_t* qh, float* dh, const SharedUpGate& sx, cudaStream_t st) {
    using Geo = UgGeom<W>;
    const int nb = ex.hidden / 32;
    const size_t smem = ChunkOf<QT, 2 * Geo::kRows, W>::kBytes + static_cast<size_t>(Geo::kTok) * nb * 40 +
                        2 * Geo::kTok * Geo::kRows * sizeof(float);
    auto kern = k_up_gate<QT, W>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(ex.inter / Geo::kRows, un.max_unique + (sx.w_gate ? 1 : 0));
    kern<<<grid, kThreads, smem, st>>>(ex.w_gate, ex.w_up, ex.s_gate, ex.s_up, ex.hidden, ex.inter,
                                       ex.group_size, qx, dx, T, un, qh, dh, sx);
    return counted(cudaGetLastError());
}

template <int QT, bool W>
cudaError_t down_qt(const moe_experts& ex, const int8_t* qh, const float* dh, int T, int K,
                    const UnionView& un, float* y, const SharedDown& sx, cudaStream_t st) {
    using Geo = DownGeom<W>;
    const int nb = ex.inter / 32;
    const size_t smem = ChunkOf<QT, Geo::kRows, W>::kBytes + static_cast<size_t>(Geo::kTok) * nb * 40;
    auto kern = k_down<QT, W>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(ex.hidden / Geo::kRows, un.max_unique + (sx.w_down ? 1 : 0));
    kern<<<grid, kThreads, smem, st>>>(ex.w_down, ex.s_down, ex.hidden, ex.inter, ex.group_size, qh, dh, T, K,
                                       un, y, sx);
    return counted(cudaGetLastError());
}

}  // namespace

cudaError_t launch_expert_up_gate(const moe_experts& ex, const int8_t* qx, const float* dx, int T,
                                  const UnionView& un, int tok_per_expert, int8_t* qh, float* dh,
                                  const SharedUpGate& sx, cudaStream_t st) {
    if (un.max_unique <= 0 && !sx.w_gate) return cudaSuccess;
    const bool wide = tok_per_expert <= kTpw && ex.inter % UgGeom<true>::kRows == 0;
    switch (ex.qtype) {
        case MOE_Q_INT4: return wide ? up_gate_qt<4, true>(ex, qx, dx, T, un, qh, dh, sx, st)
                                     : up_gate_qt<4, false>(ex, qx, dx, T, un, qh, dh, sx, st);
        case MOE_Q_INT8: return wide ? up_gate_qt<8, true>(ex, qx, dx, T, un, qh, dh, sx, st)
                                     : up_gate_qt<8, false>(ex, qx, dx, T, un, qh, dh, sx, st);
        case MOE_Q_INT2: return wide ? up_gate_qt<2, true>(ex, qx, dx, T, un, qh, dh, sx, st)
                                     : up_gate_qt<2, false>(ex, qx, dx, T, un, qh, dh, sx, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_expert_down(const moe_experts& ex, const int8_t* qh, const float* dh, int T,
                               int top_k, const UnionView& un, int tok_per_expert, float* y,
                               const SharedDown& sx, cudaStream_t st) {
    if (un.max_unique <= 0 && !sx.w_down) return cudaSuccess;
    const bool wide = tok_per_expert <= kTpw && ex.hidden % DownGeom<true>::kRows == 0;
    switch (ex.qtype) {
        case MOE_Q_INT4: return wide ? down_qt<4, true>(ex, qh, dh, T, top_k, un, y, sx, st)
                                     : down_qt<4, false>(ex, qh, dh, T, top_k, un, y, sx, st);
        case MOE_Q_INT8: return wide ? down_qt<8, true>(ex, qh, dh, T, top_k, un, y, sx, st)
                                     : down_qt<8, false>(ex, qh, dh, T, top_k, un, y, sx, st);
        case MOE_Q_INT2: return wide ? down_qt<2, true>(ex, qh, dh, T, top_k, un, y, sx, st)
                                     : down_qt<2, false>(ex, qh, dh, T, top_k, un, y, sx, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
