// Batch-union expert FFN on the 5th-generation tensor cores (tcgen05), for
// batches whose experts see many tokens (prefill, long verify).
//
// The layer of [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", section
// "구현된 주요 기능" (batch-union MoE over packed int4 experts with per-row
// scales, against Q8_0 activations), with each unique expert's weights read
// once per 128-token tile and applied to every pair routed to it.
//
// Arithmetic, exactly the quantised dot's: for every 32-block b the integer
// dot isum_b of the activation codes with the weight codes, then
// acc = fma(isum_b, d_b, acc) in ascending b (fp32, one rounding per block),
// then times the row scale.  The tensor cores produce the isum_b:
// both operands are the integer codes written as fp16 (exact: |q| <= 127 and
// the int4 weight codes), one 32-element block per pair of K = 16 MMAs; the
// fp32 accumulator of a block holds an integer below 2^15 (exact).  Each
// block's result lands in its own TMEM slot; the two blocks of a 64-K stage
// form a slot pair, and the ring holds two pairs.  One tcgen05.commit per
// stage (on the stage's `empty` barrier) tells both the producer that the
// stage's shared memory is free and the epilogue that the pair's results are
// in TMEM; the epilogue warps fold them into per-thread fp32 accumulators in
// block order (packed f32x2 fused multiply-add).  Up/gate then applies SwiGLU
// and Q8_0 to h (the codes written as fp16 for the down GEMM); down writes the
// fp32 output per (token, slot).  The result is the same, bit for bit, as the
// plain definition above evaluated one row at a time.
//
// Operand order along K.  Inside every group of 8 consecutive K positions
// both operands hold the elements in the order 0 4 1 5 2 6 3 7: the order in
// which the int4 conversion below produces them from one 32-bit word of packed
// codes.  The activation rows are written in that order by k_gather_codes (x)
// and by the up/gate epilogue (h).  A permutation inside a 32-block leaves its
// integer dot unchanged.
//
// Kernel roles (one persistent CTA per SM, 16 warps):
//   warp 0       producer: tensor-TMA tiles of the activation codes (rows in
//                union order, contiguous) and of the packed weight rows;
//   warp 1       MMA issuer (one lane); owns the TMEM allocation;
//   warps 2-5    dequantise the packed int4 rows to fp16 in the swizzled
//                operand layout (one warp per SM sub-partition);
//   warps 6-7    idle;
//   warps 8-15   epilogue: warp 8 + h covers TMEM lanes 32 (h % 4) .. + 31 and
//                columns 64 (h / 4) .. + 63 of each ring slot.
// Six shared-memory stages of 64 K each.  Every wait is bounded; on timeout
// the kernel records MOE_EDEVICE_TIMEOUT, drains what it issued and exits.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sm100_async.cuh"
#include "sm100_tc.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;            // rows (tokens or pairs) per tile = TMEM lanes
constexpr int kBN = 128;            // MMA columns per tile
constexpr int kBK = 64;             // K per stage (one 128-byte swizzle atom of fp16) = 2 blocks
constexpr int kStagesG = 6;
constexpr int kRing = 4;            // TMEM slots of block results (kRing x kBN columns)
constexpr int kPairs = kRing / 2;   // slot pairs: the two blocks of one stage
constexpr int kThreadsG = 512;
constexpr int kWarpProducer = 0, kWarpMma = 1, kWarpXform0 = 2, kXformWarps = 4, kWarpEpi0 = 8, kEpiWarps = 8;
// Register split: the CTA is launched with kLaunchRegs per thread (checked on
// the host); warpgroups 0-1 (producer, MMA, dequantisers) lower their limit to
// kRegsLow and the epilogue warpgroups 2-3 raise theirs to kRegsHigh, which
// uses exactly the launched total: 2 x kRegsLow + 2 x kRegsHigh = 4 x kLaunchRegs.
constexpr int kLaunchRegs = 128, kRegsLow = 48, kRegsHigh = 208;
static_assert(2 * kRegsLow + 2 * kRegsHigh == 4 * kLaunchRegs, "register split must use the launched total");
static_assert(kWarpEpi0 == 8 && kEpiWarps == 8, "epilogue = warpgroups 2 and 3");
constexpr long kGemmWait = 1L << 26;            // polls of the final drain waits
constexpr uint64_t kGemmWaitNs = 2000000000ull;  // pipeline waits give up after 2 s
constexpr int kTileBytes = kBM * kBK * 2;    // one 128 x 64 fp16 operand tile (16 KiB)
constexpr int kPackedBytes = kBN * kBK / 2;  // the stage's packed int4 weight rows (4 KiB)
constexpr int kStageBytesG = 2 * kTileBytes + kPackedBytes;
constexpr int kMaxItems = 1040;              // routed experts + shared expert
constexpr int kRowClasses = kBM / 16;        // activation tiles of 16, 32, .., 128 rows

// Activation-row tensor maps, one per tile height: a tile whose item has fewer
// than 128 rows left loads only round_up(rows, 16) of them (the MMA's other
// rows are stale and their results are discarded).
struct RowMaps {
    CUtensorMap m[kRowClasses];
};

struct GemmSmem {
    uint8_t* stage;       // [kStagesG][kStageBytesG], 1024-byte aligned: A | B | packed
    uint64_t* full;       // [kStagesG] activation and weight bytes landed
    uint64_t* bready;     // [kStagesG] weights dequantised
    uint64_t* empty;      // [kStagesG] MMAs done with the stage
    uint64_t* rempty;     // [kPairs] slot pair read out by every epilogue warp
    uint64_t* mma_done;   // every MMA of this CTA has completed
    uint32_t* tmem_base;
    int* item_tile0;      // [kMaxItems + 1] first tile of each expert item
};

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Pipeline wait: polls without sleeping (try_wait suspends in hardware), so a
// phase that completes is seen at once; gives up after kGemmWaitNs, or after
// `polls` polls when the workspace's test limit is set (nonzero).
__device__ __forceinline__ bool gwait(uint64_t* bar, uint32_t parity, int32_t* status, uint32_t polls) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (polls != 0 && i >= polls) break;
        if ((i & 255u) == 0 && globaltimer_ns() - t0 > kGemmWaitNs) break;
    }
    record_status(status, MOE_EDEVICE_TIMEOUT);
    return false;
}

// Expert item i: routed unique expert i (< U) or the shared expert (i == U).
struct Item {
    int row0;     // first A row: union position (routed) or P + token 0 (shared)
    int rows;     // pairs of the item
    int e;        // expert index in the stacked matrices (0 for the shared one)
    int shared;
};

__device__ __forceinline__ Item item_of(const GemmParams& p, int U, int i) {
    Item it;
    if (i < U) {
        it.row0 = p.offsets[i];
        it.rows = p.offsets[i + 1] - it.row0;
        it.e = p.uniq[i];
        it.shared = 0;
    } else {
        it.row0 = p.P;
        it.rows = p.T;
        it.e = 0;
        it.shared = 1;
    }
    return it;
}

// Tile t -> (item, n tile, m tile), m fastest so consecutive tiles share weights.
__device__ __forceinline__ void tile_of(const GemmSmem& s, int n_items, int n_tiles_n, int t, int& item, int& nt,
                                        int& mt) {
    int lo = 0, hi = n_items - 1;
    while (lo < hi) {  // last item whose first tile <= t
        const int mid = (lo + hi + 1) >> 1;
        if (s.item_tile0[mid] <= t) lo = mid; else hi = mid - 1;
    }
    item = lo;
    const int local = t - s.item_tile0[lo];
    const int mtiles = (s.item_tile0[lo + 1] - s.item_tile0[lo]) / n_tiles_n;
    nt = local / mtiles;
    mt = local % mtiles;
}

// 8 packed int4 codes (offset binary, element 2j in the low nibble of byte j)
// -> 8 fp16 values q = u - 8 in the order 0 4 1 5 2 6 3 7.  Masking a nibble
// into the mantissa of fp16 1024 gives 1024 + u (low nibble of a 16-bit half)
// or 1024 + 16 u (high nibble); 1024 + u - 1032 and (1024 + 16 u) / 16 - 72
// are exact.
__device__ __forceinline__ uint4 int4x8_to_f16(uint32_t w) {
    const uint32_t ex = 0x64006400u;
    const uint32_t e04 = (w & 0x000F000Fu) | ex, e15 = (w & 0x00F000F0u) | ex;
    w >>= 8;
    const uint32_t e26 = (w & 0x000F000Fu) | ex, e37 = (w & 0x00F000F0u) | ex;
    const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));      // 1032
    const __half2 sixteenth = __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00));  // 1/16
    const __half2 m72 = __halves2half2(__ushort_as_half(0xD480), __ushort_as_half(0xD480));        // -72
    uint4 r;
    __half2 h;
    h = __hsub2(*reinterpret_cast<const __half2*>(&e04), off); r.x = *reinterpret_cast<uint32_t*>(&h);
    h = __hfma2(*reinterpret_cast<const __half2*>(&e15), sixteenth, m72); r.y = *reinterpret_cast<uint32_t*>(&h);
    h = __hsub2(*reinterpret_cast<const __half2*>(&e26), off); r.z = *reinterpret_cast<uint32_t*>(&h);
    h = __hfma2(*reinterpret_cast<const __half2*>(&e37), sixteenth, m72); r.w = *reinterpret_cast<uint32_t*>(&h);
    return r;
}

// Byte offset of 16-byte chunk c of row r in a K-major 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// acc = fma(v, d, acc) for a pair of lanes: the quantised dot's block step
// (one rounding), as a packed f32x2 fused multiply-add.
__device__ __forceinline__ void fold2(float2& acc, uint32_t v0, uint32_t v1, float d) {
    float2 v = make_float2(__uint_as_float(v0), __uint_as_float(v1));
    float2 dd = make_float2(d, d);
    asm volatile("fma.rn.f32x2 %0, %1, %2, %0;"
                 : "+l"(reinterpret_cast<uint64_t&>(acc))
                 : "l"(reinterpret_cast<uint64_t&>(v)), "l"(reinterpret_cast<uint64_t&>(dd)));
}

// Q8_0 of 32 values held by one thread, same arithmetic as q8_0_lane; the codes
// are returned as fp16 pairs (exact) for the down GEMM, each group of 8 in the
// order 0 4 1 5 2 6 3 7.
__device__ __forceinline__ float q8_0_thread_f16(const float (&v)[32], uint32_t (&codes)[16]) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const float d = __fdiv_rn(amax, 127.0f);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int e = 8 * (j >> 2) + (j & 3);  // group element pair (e, e + 4)
        float q[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            q[i] = 0.0f;
            if (d != 0.0f) q[i] = fminf(fmaxf(roundf(__fdiv_rn(v[e + 4 * i], d)), -127.0f), 127.0f);
        }
        const __half2 h = __floats2half2_rn(q[0], q[1]);
        codes[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return d;
}

template <int MODE>
__global__ void __launch_bounds__(kThreadsG, 1)
    k_moe_gemm(const __grid_constant__ GemmParams p, const __grid_constant__ RowMaps tm_a,
               const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1,
               const __grid_constant__ CUtensorMap tm_b0s, const __grid_constant__ CUtensorMap tm_b1s) {
    extern __shared__ __align__(1024) uint8_t gsm_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the workspace's test limit on pipeline waits (0: none; the final drains ignore it)
    const uint32_t wl = static_cast<uint32_t>(ld_relaxed_gpu(p.wait_limit));
    GemmSmem s;
    {
        const uintptr_t base = (reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~static_cast<uintptr_t>(1023);
        s.stage = reinterpret_cast<uint8_t*>(base);
        uint64_t* bars = reinterpret_cast<uint64_t*>(s.stage + kStagesG * kStageBytesG);
        s.full = bars;
        s.bready = bars + kStagesG;
        s.empty = bars + 2 * kStagesG;
        s.rempty = bars + 3 * kStagesG;
        s.mma_done = s.rempty + kPairs;
        s.tmem_base = reinterpret_cast<uint32_t*>(s.mma_done + 1);
        s.item_tile0 = reinterpret_cast<int*>(s.tmem_base + 4);
    }
    // up/gate: tile columns = 64 h indices x (gate, up); down: 128 output columns
    const int nout = MODE == kGemmUpGate ? p.I : p.H;     // weight rows per expert matrix
    const int kdim = MODE == kGemmUpGate ? p.H : p.I;     // contraction length
    const int cols_per_tile = MODE == kGemmUpGate ? kBN / 2 : kBN;
    const int n_tiles_n = (nout + cols_per_tile - 1) / cols_per_tile;
    const int ksteps = kdim / kBK;
    const int nblk = kdim / 32;
    const int U = *p.n_unique;
    const int n_items = U + (p.has_shared ? 1 : 0);
    if (tid == 0) {
        for (int i = 0; i < kStagesG; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.bready[i], kXformWarps);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < kPairs; ++i) mbar_init(&s.rempty[i], kEpiWarps);
        mbar_init(s.mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 0) {  // first tile of every item (prefix over the items' tile counts)
        int carry = 0;
        for (int base = 0; base < n_items; base += 32) {
            const int i = base + lane;
            int cnt = 0;
            if (i < n_items) cnt = ((item_of(p, U, i).rows + kBM - 1) / kBM) * n_tiles_n;
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (i < n_items) s.item_tile0[i] = carry + incl - cnt;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s.item_tile0[n_items] = carry;
    }
    if (warp == kWarpMma) {
        tmem_alloc(s.tmem_base, kRing * kBN);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const int n_tiles = s.item_tile0[n_items];
    const uint32_t tmem = *s.tmem_base;

    if (warp >= kWarpEpi0) {
        regs_raise<kRegsHigh>();
        // ------------------------------------------------------------ epilogue
        const int eh = warp - kWarpEpi0;            // 0..7
        const int q = warp & 3;                     // TMEM lane quarter of this warp
        const int half = eh >> 2;                   // columns 64 half .. 64 half + 63 of each slot
        const int r = q * 32 + lane;                // tile row (token / pair) of this thread
        int stage = 0, pair = 0;                    // the MMA issuer's stage / slot-pair sequence
        uint32_t phase = 0, rphase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            int item, nt, mt;
            tile_of(s, n_items, n_tiles_n, t, item, nt, mt);
            const Item it = item_of(p, U, item);
            const int rows = min(kBM, it.rows - mt * kBM);
            const int pr = it.row0 + mt * kBM + r;  // A row (union position or P + token)
            const bool valid = r < rows;
            int arow = 0, tok = 0, slot_k = 0;
            if (valid) {
                tok = it.shared ? pr - p.P : p.pair_tok[pr];
                slot_k = it.shared ? 0 : p.pair_slot[pr];
                arow = MODE == kGemmUpGate ? tok : pr;
            }
            // the two block scales of each k step (nblk is even), prefetched kPre steps ahead
            const float2* d2 = reinterpret_cast<const float2*>(p.a_scales + static_cast<size_t>(arow) * nblk);
            float2 acc[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i] = make_float2(0.0f, 0.0f);
            constexpr int kPre = 4;
            float2 dq[kPre];
#pragma unroll
            for (int j = 0; j < kPre; ++j) dq[j] = j < ksteps ? __ldg(d2 + j) : make_float2(0.0f, 0.0f);
            // Per stage: wait for the MMAs' commit on the stage's `empty` barrier,
            // load the pair's two block results, release the pair, fold both.
            const uint32_t lane_off = half * 64 + (static_cast<uint32_t>(q * 32) << 16);
            for (int ks0 = 0; ks0 < ksteps && ok; ks0 += kPre) {
#pragma unroll
                for (int j = 0; j < kPre; ++j) {
                    const int ks = ks0 + j;
                    if (ks >= ksteps || !ok) continue;
                    const float2 dk = dq[j];
                    if (ks + kPre < ksteps) dq[j] = __ldg(d2 + ks + kPre);
                    if (!gwait(&s.empty[stage], phase, p.status, wl)) {
                        ok = false;
                        continue;
                    }
                    tc_fence_after_sync();
                    const uint32_t ta = tmem + pair * 2 * kBN + lane_off;
                    uint32_t va[32], vb[32], vc[32], vd[32];
                    tmem_ld32_async(ta, va);
                    tmem_ld32_async(ta + 32, vb);
                    tmem_ld32_async(ta + kBN, vc);
                    tmem_ld32_async(ta + kBN + 32, vd);
                    tmem_wait_ld();
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.rempty[pair]);
#pragma unroll
                    for (int i = 0; i < 16; ++i) fold2(acc[i], va[2 * i], va[2 * i + 1], dk.x);
#pragma unroll
                    for (int i = 0; i < 16; ++i) fold2(acc[16 + i], vb[2 * i], vb[2 * i + 1], dk.x);
#pragma unroll
                    for (int i = 0; i < 16; ++i) fold2(acc[i], vc[2 * i], vc[2 * i + 1], dk.y);
#pragma unroll
                    for (int i = 0; i < 16; ++i) fold2(acc[16 + i], vd[2 * i], vd[2 * i + 1], dk.y);
                    if (++stage == kStagesG) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++pair == kPairs) {
                        pair = 0;
                        rphase ^= 1u;
                    }
                }
            }
            if (!ok || !valid) continue;
            const int c0 = nt * cols_per_tile + half * (MODE == kGemmUpGate ? 32 : 64);
            if (c0 >= nout) continue;
            if (MODE == kGemmUpGate) {
                // acc[0..15] gate, acc[16..31] up, for h indices c0 .. c0 + 31
                const float* sg = it.shared ? p.s_a_sh : p.s_a + static_cast<size_t>(it.e) * nout;
                const float* su = it.shared ? p.s_b_sh : p.s_b + static_cast<size_t>(it.e) * nout;
                float h[32];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float g0 = __fmul_rn(acc[i].x, __ldg(sg + c0 + 2 * i));
                    const float g1 = __fmul_rn(acc[i].y, __ldg(sg + c0 + 2 * i + 1));
                    const float u0 = __fmul_rn(acc[16 + i].x, __ldg(su + c0 + 2 * i));
                    const float u1 = __fmul_rn(acc[16 + i].y, __ldg(su + c0 + 2 * i + 1));
                    h[2 * i] = swiglu(g0, u0);
                    h[2 * i + 1] = swiglu(g1, u1);
                }
                uint32_t codes[16];
                const float d = q8_0_thread_f16(h, codes);
                uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(p.h_codes) + static_cast<size_t>(pr) * nout + c0);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    dst[j] = make_uint4(codes[4 * j], codes[4 * j + 1], codes[4 * j + 2], codes[4 * j + 3]);
                p.h_scales[static_cast<size_t>(pr) * (nout / 32) + c0 / 32] = d;
            } else {
                const float* sd = it.shared ? p.s_a_sh : p.s_a + static_cast<size_t>(it.e) * nout;
                float* yrow = it.shared ? p.ys + static_cast<size_t>(tok) * nout
                                        : p.y + (static_cast<size_t>(tok) * p.K + slot_k) * nout;
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float4 o;
                    o.x = __fmul_rn(acc[i].x, __ldg(sd + c0 + 2 * i));
                    o.y = __fmul_rn(acc[i].y, __ldg(sd + c0 + 2 * i + 1));
                    o.z = __fmul_rn(acc[i + 1].x, __ldg(sd + c0 + 2 * i + 2));
                    o.w = __fmul_rn(acc[i + 1].y, __ldg(sd + c0 + 2 * i + 3));
                    *reinterpret_cast<float4*>(yrow + c0 + 2 * i) = o;
                }
            }
        }
    } else {
        regs_lower<kRegsLow>();
        if (warp == kWarpProducer) {
            // ------------------------------------------------------------ producer
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            long issued = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                int item, nt, mt;
                tile_of(s, n_items, n_tiles_n, t, item, nt, mt);
                const Item it = item_of(p, U, item);
                const int r0 = it.row0 + mt * kBM;
                const int rcls = (min(kBM, it.rows - mt * kBM) + 15) / 16 - 1;  // tile height class
                const uint32_t a_bytes = static_cast<uint32_t>(rcls + 1) * 16u * kBK * 2u;
                const CUtensorMap* b0 = it.shared ? &tm_b0s : &tm_b0;
                const CUtensorMap* b1 = it.shared ? &tm_b1s : &tm_b1;
                const int wr = (it.shared ? 0 : it.e * nout) + nt * cols_per_tile;
                for (int ks = 0; ks < ksteps; ++ks) {
                    if (!gwait(&s.empty[stage], phase ^ 1u, p.status, wl)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = s.stage + stage * kStageBytesG;
                    uint8_t* a = st;
                    uint8_t* packed = st + 2 * kTileBytes;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&s.full[stage], a_bytes + kPackedBytes);
                        tma_load_2d(a, &tm_a.m[rcls], ks * kBK, r0, &s.full[stage]);
                        if (MODE == kGemmUpGate) {  // gate rows then up rows, 64 each
                            tma_load_2d(packed, b0, ks * (kBK / 2), wr, &s.full[stage]);
                            tma_load_2d(packed + kPackedBytes / 2, b1, ks * (kBK / 2), wr, &s.full[stage]);
                        } else {
                            tma_load_2d(packed, b0, ks * (kBK / 2), wr, &s.full[stage]);
                        }
                    }
                    __syncwarp();
                    ++issued;
                    if (++stage == kStagesG) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // drain: every copy issued into this CTA's shared memory has landed
            if (lane == 0) {
                for (int st = 0; st < kStagesG; ++st) {
                    const long uses = issued / kStagesG + (st < issued % kStagesG ? 1 : 0);
                    if (uses > 0) mbar_wait(&s.full[st], static_cast<uint32_t>((uses - 1) & 1), kGemmWait);
                }
            }
            __syncwarp();
        } else if (warp == kWarpMma) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                int stage = 0, pair = 0;
                uint32_t phase = 0, rphase = 0;
                bool ok = true;
                const uint32_t idesc = umma_idesc_f16(kBM, kBN);
                // descriptors of stage 0; a stage or K offset adds (bytes >> 4) to the
                // start-address field (all addresses stay below 256 KiB)
                const uint64_t adesc0 = umma_desc_sw128(s.stage, 0);
                const uint64_t bdesc0 = umma_desc_sw128(s.stage + kTileBytes, 0);
                for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                    for (int ks = 0; ks < ksteps && ok; ++ks) {
                        if (!gwait(&s.full[stage], phase, p.status, wl) || !gwait(&s.bready[stage], phase, p.status, wl)) {
                            ok = false;
                            break;
                        }
                        if (!gwait(&s.rempty[pair], rphase ^ 1u, p.status, wl)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint64_t soff = static_cast<uint64_t>((stage * kStageBytesG) >> 4);
                        const uint64_t ad = adesc0 + soff, bd = bdesc0 + soff;
                        const uint32_t d = tmem + pair * 2 * kBN;
                        // block 0 (K 0..31 of the stage) into the pair's first slot, block 1 into the second
                        umma_f16(d, ad, bd, idesc, false);
                        umma_f16(d, ad + 2, bd + 2, idesc, true);
                        umma_f16(d + kBN, ad + 4, bd + 4, idesc, false);
                        umma_f16(d + kBN, ad + 6, bd + 6, idesc, true);
                        // one commit: the stage's shared memory is free (producer) and the
                        // pair's results are in TMEM (epilogue)
                        umma_commit(&s.empty[stage]);
                        if (++pair == kPairs) {
                            pair = 0;
                            rphase ^= 1u;
                        }
                        if (++stage == kStagesG) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
                // every MMA issued by this thread has completed before TMEM is freed
                umma_commit(s.mma_done);
                mbar_wait(s.mma_done, 0, kGemmWait);
            }
            __syncwarp();
        } else if (warp < kWarpXform0 + kXformWarps) {
            // ------------------------------------------------------------ dequantise weights
            const int xt = tid - kWarpXform0 * 32;  // 0 .. 32 kXformWarps - 1
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                for (int ks = 0; ks < ksteps; ++ks) {
                    if (!gwait(&s.full[stage], phase, p.status, wl)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = s.stage + stage * kStageBytesG;
                    uint8_t* b = st + kTileBytes;
                    const uint8_t* packed = st + 2 * kTileBytes;
                    // B row br <- packed row: up/gate interleaves [gate 32 | up 32 | gate 32 | up 32]
                    // so that each epilogue warp's 64 columns hold gate and up of the same 32 h
                    for (int task = xt; task < kBN * 2; task += 32 * kXformWarps) {
                        const int br = task >> 1, hv = task & 1;  // hv: chunks 0-3 or 4-7 of the row
                        int src_row = br;
                        if (MODE == kGemmUpGate) src_row = ((br >> 5) & 1) * 64 + (br & 31) + ((br >> 6) << 5);
                        const uint4 w = reinterpret_cast<const uint4*>(packed + src_row * (kBK / 2))[hv];
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            *reinterpret_cast<uint4*>(b + sw128_off(br, 4 * hv + c)) = int4x8_to_f16(ws[c]);
                    }
                    // orders the dequantised weights before the MMAs (async proxy)
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.bready[stage]);
                    if (++stage == kStagesG) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kRing * kBN);
    }
}

// The up/gate GEMM's activation rows: row r < P is the Q8_0 codes of token
// pair_tok[r] (union order), row P + t those of token t (shared expert); codes
// as fp16 (exact), each group of 8 in the order 0 4 1 5 2 6 3 7.  One thread
// per group of 8.
__global__ void k_gather_codes(const int8_t* __restrict__ q, int H, int P, size_t rows,
                               const int32_t* __restrict__ pair_tok, __half* __restrict__ out) {
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int g = H / 8;
    if (i >= rows * g) return;
    const size_t r = i / g;
    const int c = static_cast<int>(i - r * g);
    const int tok = r < static_cast<size_t>(P) ? __ldg(pair_tok + r) : static_cast<int>(r - P);
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(q + static_cast<size_t>(tok) * H) + c);
    auto code = [&](int e) { return static_cast<float>(static_cast<int8_t>(((e < 4 ? raw.x : raw.y) >> (8 * (e & 3))) & 0xFF)); };
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __half2 h = __floats2half2_rn(code(j), code(j + 4));
        o[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
}

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D map over a row-major [rows][cols] matrix of `esize`-byte elements.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(esize)};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t gemm_smem_bytes() {
    return 1024 + static_cast<size_t>(kStagesG) * kStageBytesG + 256 + sizeof(int) * (kMaxItems + 8);
}

}  // namespace

bool tc_gemm_supported(const moe_experts& r, const moe_experts* s, int E) {
    if (r.qtype != MOE_Q_INT4 || (s && (s->qtype != MOE_Q_INT4 || s->inter != r.inter || s->hidden != r.hidden)))
        return false;
    if (r.group_size || (s && s->group_size)) return false;  // per-row scales only (the epilogue's fold)
    if (r.hidden % kBK || r.inter % kBK) return false;  // whole K stages; 64-column output halves
    if (E + 1 > kMaxItems) return false;
    return true;
}

cudaError_t launch_gather_codes(const int8_t* q, int H, int P, int rows, const int32_t* pair_tok, __half* out,
                                cudaStream_t st) {
    const size_t n8 = static_cast<size_t>(rows) * (H / 8);
    if (n8 == 0) return cudaSuccess;
    const int threads = 256;
    k_gather_codes<<<static_cast<unsigned>((n8 + threads - 1) / threads), threads, 0, st>>>(q, H, P, rows, pair_tok,
                                                                                            out);
    return counted(cudaGetLastError());
}

cudaError_t launch_moe_gemm(int mode, const GemmParams& p, const GemmOperands& o, cudaStream_t st) {
    RowMaps a;
    CUtensorMap b0, b1, b0s, b1s;
    const int K = mode == kGemmUpGate ? p.H : p.I;  // contraction
    const int nout = mode == kGemmUpGate ? p.I : p.H;
    const uint32_t brows = mode == kGemmUpGate ? kBN / 2 : kBN;
    bool ok = make_map(&b0, o.w0, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, static_cast<uint64_t>(o.n_expert) * nout,
                       kBK / 2, brows, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (ok && p.has_shared)
        ok = make_map(&b0s, o.w0s, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, nout, kBK / 2, brows,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    else
        b0s = b0;
    if (ok && mode == kGemmUpGate) {
        ok = make_map(&b1, o.w1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, static_cast<uint64_t>(o.n_expert) * nout,
                      kBK / 2, brows, CU_TENSOR_MAP_SWIZZLE_NONE);
        if (ok && p.has_shared)
            ok = make_map(&b1s, o.w1s, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, nout, kBK / 2, brows,
                          CU_TENSOR_MAP_SWIZZLE_NONE);
        else
            b1s = b1;
    } else {
        b1 = b0;
        b1s = b0s;
    }
    for (int c = 0; c < kRowClasses && ok; ++c)
        ok = make_map(&a.m[c], p.a_codes, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, K, static_cast<uint64_t>(p.P + p.T), kBK,
                      16 * (c + 1), CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    static int sms[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && sms[dev] == 0) {
        e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    const int grid = (dev >= 0 && dev < 64) ? sms[dev] : 148;
    const size_t smem = gemm_smem_bytes();
    const void* kern = mode == kGemmUpGate ? reinterpret_cast<const void*>(k_moe_gemm<kGemmUpGate>)
                                           : reinterpret_cast<const void*>(k_moe_gemm<kGemmDown>);
    e = ensure_smem(kern, smem);
    if (e != cudaSuccess) return e;
    // the in-kernel register split assumes this launch size exactly
    cudaFuncAttributes fa{};
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    if (mode == kGemmUpGate)
        k_moe_gemm<kGemmUpGate><<<grid, kThreadsG, smem, st>>>(p, a, b0, b1, b0s, b1s);
    else
        k_moe_gemm<kGemmDown><<<grid, kThreadsG, smem, st>>>(p, a, b0, b1, b0s, b1s);
    return counted(cudaGetLastError());
}

}  // namespace moe
