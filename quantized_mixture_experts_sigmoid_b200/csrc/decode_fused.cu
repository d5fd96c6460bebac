// Fused, persistent routed-MoE layer for small batches (decode T = 1, MTP verify T <= 4).
//
// The whole layer of [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기",
// section "구현된 주요 기능" (DeepSeek-V3-style sigmoid router with noaux_tc and
// routed_scaling_factor, shared expert, batch-union MoE, int8 / packed int4 /
// packed int2 per-row-scaled weights with dequant-on-use, integer dot against
// Q8_0 activations) in one launch.  At these batch sizes the layer is a pure
// weight stream from HBM (176.5 MB per decode token for GLM-5.2's shape), so
// the design goal is to keep HBM busy from the first byte to the last.
//
// Roles (one CTA per SM):
//  * warp 17, the producer, streams weight rows into a shared-memory ring
//    with bulk copies (cp.async.bulk, non-multicast TMA) completing on
//    mbarriers;
//  * warps 0-15, the consumers, take one ring stage at a time and form the
//    integer dot products with dp4a;
//  * warp 16, the epilogue warp, finishes tiles handed over through a
//    double-buffered mbarrier queue (SwiGLU and Q8_0 of h for up/gate tiles;
//    completion counting and the combine for down tiles), so the consumers
//    never wait on fences or atomics.
//
// Work is one global ticket sequence claimed by the producers:
//      router rows | shared up/gate tiles | routed up/gate tiles |
//      shared down tiles | routed down tiles
// so every dependency points to an earlier ticket and every CTA sees its
// stages in that order.  After its last router row a producer queues a
// zero-byte route marker; at the marker the consumers wait until every logit
// of the batch has been counted, then compute the noaux_tc selection and the
// batch union themselves (all consumer threads, rank-based, in shared memory:
// every CTA reaches the same result) and hand it to their producer through an
// mbarrier.  Routing therefore costs one global round trip (the logit count)
// rather than a publish by one CTA and a read-back by all.  An up/gate tile is 32 rows of h for one expert; its epilogue
// writes Q8_0(h) as a pre-permuted activation record.  A down tile waits for
// its expert's h tiles, then copies the records of its pairs next to its
// weight stages.  The CTA that completes a row block of the output combines
// it (shared + sum_k w_k y_k in slot order), so the result is deterministic.
//
// NT is the compile-time token capacity: NT = 1 keeps the token's activations
// in registers; NT = 4 reads them from shared memory.
//
// Counters live in the caller's workspace; the last CTA to exit resets them.
// Every wait is bounded: on timeout the kernel records MOE_EDEVICE_TIMEOUT in
// the workspace status word, stops issuing copies, waits for those in flight
// and exits.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "quant.cuh"
#include "sm100_async.cuh"

namespace moe {
namespace {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kEpilogueWarp = kConsumerWarps;
constexpr int kProducerWarp = kConsumerWarps + 1;
constexpr int kThreadsF = (kConsumerWarps + 2) * 32;
constexpr int kMaxT = kFusedMaxTokens;
constexpr int kStageRows = 16;       // up/gate rows per stage (one per consumer warp)
constexpr int kUgTileRows = 32;      // one Q8_0 block of h
constexpr int kDownStagesPerTile = 2;
constexpr int kMaxRouterRows = 4;    // router rows per stage
constexpr int kMaxDownRowsPerWarp = 4;
constexpr int kActSlots = 2;
constexpr int kTaskSlots = 2;
constexpr int kScaleBytes = 256;     // room after each stage for its rows' fp32 scales
// Copies a producer keeps in flight.  Enough to cover HBM latency at full
// bandwidth; more only lengthens the memory queues, and every other request
// (logits, counters, instruction fetches) then waits behind them.
constexpr int kMaxInflight = 2;
constexpr int kRegChunksUg = 6;      // NT = 1: blocks of x per lane held in registers (H <= 6144)
constexpr int kRegChunksDown = 2;    // NT = 1: blocks of h per lane held in registers (I <= 2048)
constexpr long kProducerWait = 1L << 22;
constexpr long kConsumerWait = 1L << 24;
constexpr long kEpilogueWait = 1L << 25;
constexpr int kBarConsumers = 1;     // named barrier id of the consumer warps

enum : int { D_EXIT = 0, D_ROUTER = 1, D_UG = 2, D_DOWN = 3, D_ROUTE = 4 };
constexpr int kMaxPairs = kMaxT * 32;

struct Desc {
    int type;
    int e;          // expert index (routed) or 0 (shared); router: first expert row
    int cslot;      // h-completion counter slot: 0 shared, 1 + u routed
    int mat;        // 0 gate, 1 up, 2 down
    int row0;       // first row of this stage in its matrix
    int nrows;
    int first;
    int last;
    int blk;        // up/gate: h block index; down: row block index
    int aslot;
    int n_experts;  // shared + distinct routed experts (down tiles)
    int n_tok;
    int tok[kMaxT];
    int pair[kMaxT];
};

// A finished tile handed to the epilogue warp.
struct Task {
    int type;  // D_UG, D_DOWN or D_EXIT
    int n_tok, blk, cslot, n_experts;
    int pair[kMaxT];
};

struct Smem {
    uint8_t* ring;
    uint8_t* act;
    uint16_t* xs;    // bf16 x; reused as routing scratch once the router rows are done
    uint4* q0;
    uint4* q1;
    float* qd;
    int32_t* qs;
    float* bias;     // [E]
    Desc* desc;
    Task* task;      // [kTaskSlots]
    float* gbuf;     // [kTaskSlots][kMaxT][32]
    float* ubuf;     // [kTaskSlots][kMaxT][32]
    double* red;
    uint64_t* full;
    uint64_t* empty;
    uint64_t* afull;
    uint64_t* aempty;
    uint64_t* tfull;
    uint64_t* tfree;
    uint64_t* route_bar;  // consumers -> producer: routing of the batch is ready
    int* flag;
    int* chosen;     // [kMaxT][32] chosen experts per token, slot order
    int* ent;        // [kMaxPairs] union scratch
    uint32_t* bmap;  // [32]
    // routing of the batch, identical in every CTA
    float* rt_w;     // [kMaxPairs] gate weights by (token, slot)
    int* rt_pair_of; // [kMaxPairs] pair index by (token, slot)
    int* rt_uniq;    // [kMaxPairs] distinct experts ascending
    int* rt_off;     // [kMaxPairs + 1] pair offsets per distinct expert
    int* rt_ptok;    // [kMaxPairs] token of each pair
    int* rt_U;       // [1] number of distinct experts
    int* bpre;       // [33] prefix popcounts of the expert bitmap
    uint8_t* qscratch;  // [kConsumerWarps][256] Q8_0 staging (aliases the activation slots)
};

__host__ __device__ inline size_t a16(size_t v) { return (v + 15) & ~size_t(15); }

struct Layout {
    size_t ring, act, xs, qx, bias, desc, task, gbuf, red, bars, misc, total;
};

__host__ __device__ inline Layout layout_of(const FusedParams& p) {
    Layout L{};
    const size_t slot = static_cast<size_t>(p.stage_bytes) + kScaleBytes;
    const int nbH = p.H / 32;
    size_t o = 0;
    L.ring = o; o += a16(slot * p.nstage);
    // the activation slots (down tiles) double as Q8_0 staging before routing
    const size_t act = static_cast<size_t>(p.act_bytes) * kActSlots, qstage = static_cast<size_t>(kConsumerWarps) * 256;
    L.act = o; o += a16(act > qstage ? act : qstage);
    L.xs = o; o += a16(static_cast<size_t>(p.T) * p.H * 2);
    L.qx = o; o += a16(static_cast<size_t>(p.T) * nbH * 40);
    L.bias = o; o += a16(sizeof(float) * p.E);
    L.desc = o; o += a16(sizeof(Desc) * p.nstage);
    L.task = o; o += a16(sizeof(Task) * kTaskSlots);
    L.gbuf = o; o += a16(sizeof(float) * 2 * kTaskSlots * kMaxT * kUgTileRows);
    L.red = o; o += a16(sizeof(double) * kConsumerWarps * kMaxRouterRows * kMaxT);
    L.bars = o; o += a16(sizeof(uint64_t) * (2 * p.nstage + 2 * kActSlots + 2 * kTaskSlots + 1));
    L.misc = o; o += a16(sizeof(int) * (4 + 2 * kMaxPairs + 32 + 5 * kMaxPairs + 2 + 33));
    L.total = o;
    return L;
}

__device__ Smem carve(uint8_t* base, const FusedParams& p) {
    const Layout L = layout_of(p);
    const int nbH = p.H / 32;
    Smem s;
    s.ring = base + L.ring;
    s.act = base + L.act;
    s.xs = reinterpret_cast<uint16_t*>(base + L.xs);
    s.q0 = reinterpret_cast<uint4*>(base + L.qx);
    s.q1 = s.q0 + p.T * nbH;
    s.qd = reinterpret_cast<float*>(s.q1 + p.T * nbH);
    s.qs = reinterpret_cast<int32_t*>(s.qd + p.T * nbH);
    s.bias = reinterpret_cast<float*>(base + L.bias);
    s.desc = reinterpret_cast<Desc*>(base + L.desc);
    s.task = reinterpret_cast<Task*>(base + L.task);
    s.gbuf = reinterpret_cast<float*>(base + L.gbuf);
    s.ubuf = s.gbuf + kTaskSlots * kMaxT * kUgTileRows;
    s.red = reinterpret_cast<double*>(base + L.red);
    s.full = reinterpret_cast<uint64_t*>(base + L.bars);
    s.empty = s.full + p.nstage;
    s.afull = s.empty + p.nstage;
    s.aempty = s.afull + kActSlots;
    s.tfull = s.aempty + kActSlots;
    s.tfree = s.tfull + kTaskSlots;
    s.route_bar = s.tfree + kTaskSlots;
    s.flag = reinterpret_cast<int*>(base + L.misc);
    s.chosen = s.flag + 4;
    s.ent = s.chosen + kMaxPairs;
    s.bmap = reinterpret_cast<uint32_t*>(s.ent + kMaxPairs);
    s.rt_w = reinterpret_cast<float*>(s.bmap + 32);
    s.rt_pair_of = reinterpret_cast<int*>(s.rt_w + kMaxPairs);
    s.rt_uniq = s.rt_pair_of + kMaxPairs;
    s.rt_off = s.rt_uniq + kMaxPairs;
    s.rt_ptok = s.rt_off + kMaxPairs + 1;
    s.rt_U = s.rt_ptok + kMaxPairs;
    s.bpre = s.rt_U + 1;
    s.qscratch = s.act;
    return s;
}

template <int QT>
__device__ __forceinline__ WBlock<QT> load_wblock_smem(const uint8_t* row, int b) {
    WBlock<QT> r;
    if constexpr (QT == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(row + 8 * b);
        r.w[0] = v.x;
        r.w[1] = v.y;
    } else if constexpr (QT == 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + 16 * b);
        r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
    } else {
        const uint4 v0 = *reinterpret_cast<const uint4*>(row + 32 * b);
        const uint4 v1 = *reinterpret_cast<const uint4*>(row + 32 * b + 16);
        r.w[0] = v0.x; r.w[1] = v0.y; r.w[2] = v0.z; r.w[3] = v0.w;
        r.w[4] = v1.x; r.w[5] = v1.y; r.w[6] = v1.z; r.w[7] = v1.w;
    }
    return r;
}

__device__ __forceinline__ void consumers_sync() { named_bar_sync(kBarConsumers, kConsumers); }

// Element of a 32-block that byte i of permuted activation word w holds,
// matching the field order in which block_dot<QT> presents weight codes.
template <int QT>
__host__ __device__ constexpr int perm_src(int w, int i) {
    return QT == 4 ? 8 * (w >> 1) + 2 * i + (w & 1) : QT == 2 ? 16 * (w >> 2) + 4 * i + (w & 3) : 4 * w + i;
}

// Lane l holds code q of element l of a block; returns permuted word (l & 7).
template <int QT>
__device__ __forceinline__ uint32_t perm_word(int q, int lane) {
    const int w = lane & 7;
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        word |= (static_cast<uint32_t>(__shfl_sync(0xffffffffu, q, perm_src<QT>(w, i))) & 0xFFu) << (8 * i);
    return word;
}

// ------------------------------------------------------------------ producer
template <int QT>
__device__ void producer(const FusedParams& p, const Smem& s) {
    const size_t slot_bytes = static_cast<size_t>(p.stage_bytes) + kScaleBytes;
    const uint64_t pol = l2_evict_first_policy();
    const int nrt = p.n_rt, nug = p.n_ugt, nd = p.n_dt, hs = p.has_shared;
    const int P = p.T * p.K;
    const size_t rb_ug = static_cast<size_t>(p.H) * QT / 8, rb_d = static_cast<size_t>(p.I) * QT / 8;
    int stage = 0, aslot = 0;
    uint32_t sphase = 0, aphase = 0;
    long n_issued = 0, n_act = 0;
    int U = -1;
    bool ok = true, marked = false;

    auto acquire_stage = [&]() -> bool {
        if (n_issued >= kMaxInflight) {  // at most kMaxInflight copies in flight
            const long older = n_issued - kMaxInflight;
            if (!mbar_wait(&s.full[older % p.nstage], static_cast<uint32_t>((older / p.nstage) & 1),
                           kProducerWait))
                return false;
        }
        return mbar_wait(&s.empty[stage], sphase ^ 1u, kProducerWait);
    };
    auto advance = [&]() {
        ++n_issued;
        if (++stage == p.nstage) {
            stage = 0;
            sphase ^= 1u;
        }
    };
    auto issue = [&](const Desc& d, const void* w_src, uint32_t w_bytes, const void* s_src,
                     uint32_t s_bytes) -> bool {
        if (!acquire_stage()) return false;
        s.desc[stage] = d;
        uint8_t* dst = s.ring + stage * slot_bytes;
        mbar_arrive_expect_tx(&s.full[stage], w_bytes + s_bytes);
        bulk_g2s_hint(dst, w_src, w_bytes, &s.full[stage], pol);
        if (s_bytes) bulk_g2s(dst + p.stage_bytes, s_src, s_bytes, &s.full[stage]);
        advance();
        return true;
    };

    int next = atomicAdd(&p.sync->ticket, 1);
    while (ok) {
        const int cur = next;
        next = atomicAdd(&p.sync->ticket, 1);
        Desc d{};
        if (cur < nrt) {  // router rows e0 .. e0 + n - 1
            d.type = D_ROUTER;
            d.e = cur * p.rps;
            d.nrows = min(p.rps, p.E - d.e);
            ok = issue(d, p.w_router + static_cast<size_t>(d.e) * p.H, 4u * p.H * d.nrows, nullptr, 0);
            continue;
        }
        if (!marked) {  // router rows of this CTA are all queued: the consumers route next
            if (!acquire_stage()) {
                ok = false;
                break;
            }
            s.desc[stage].type = D_ROUTE;
            mbar_arrive(&s.full[stage]);
            advance();
            marked = true;
        }
        int t = cur - nrt;
        int kind, u, j;  // kind: 0 up/gate, 1 down; u = -1 shared
        if (hs && t < nug) {
            kind = 0; u = -1; j = t;
        } else {
            if (U < 0) {
                if (!mbar_wait(s.route_bar, 0, kProducerWait)) {
                    ok = false;
                    break;
                }
                U = *reinterpret_cast<volatile int*>(s.rt_U);
            }
            t -= hs * nug;
            if (t < U * nug) {
                kind = 0; u = t / nug; j = t % nug;
            } else {
                t -= U * nug;
                if (hs && t < nd) {
                    kind = 1; u = -1; j = t;
                } else {
                    t -= hs * nd;
                    if (t >= U * nd) break;  // no work left
                    kind = 1; u = t / nd; j = t % nd;
                }
            }
        }
        d.cslot = u < 0 ? 0 : 1 + u;
        d.n_experts = U + hs;
        if (u < 0) {
            d.e = 0;
            d.n_tok = p.T;
            for (int i = 0; i < p.T; ++i) {
                d.tok[i] = i;
                d.pair[i] = P + i;
            }
        } else {
            d.e = s.rt_uniq[u];
            const int p0 = s.rt_off[u], p1 = s.rt_off[u + 1];
            d.n_tok = p1 - p0;
            for (int i = 0; i < d.n_tok; ++i) {
                d.tok[i] = s.rt_ptok[p0 + i];
                d.pair[i] = p0 + i;
            }
        }
        const moe_experts& ex = u < 0 ? p.shared : p.routed;
        d.blk = j;
        if (kind == 0) {  // up/gate tile: rows 32j..32j+31 of gate, then of up
            d.type = D_UG;
            d.nrows = kStageRows;
            for (int m = 0; m < 2 && ok; ++m) {
                const uint8_t* wm = m == 0 ? ex.w_gate : ex.w_up;
                const float* sm = m == 0 ? ex.s_gate : ex.s_up;
                for (int q = 0; q < kUgTileRows / kStageRows && ok; ++q) {
                    d.mat = m;
                    d.row0 = j * kUgTileRows + q * kStageRows;
                    d.first = (m == 0 && q == 0);
                    d.last = (m == 1 && q == kUgTileRows / kStageRows - 1);
                    const size_t r = static_cast<size_t>(d.e) * p.I + d.row0;
                    ok = issue(d, wm + r * rb_ug, static_cast<uint32_t>(kStageRows * rb_ug), sm + r,
                               kStageRows * 4);
                }
            }
        } else {  // down tile: rows j*dr .. j*dr+dr-1, after the expert's h is complete
            d.type = D_DOWN;
            d.mat = 2;
            if (!mbar_wait(&s.aempty[aslot], aphase ^ 1u, kProducerWait) ||
                !wait_counter_geq(p.ug_done + d.cslot, nug, kProducerWait)) {
                ok = false;
                break;
            }
            fence_proxy_async_global();
            const uint32_t abytes = static_cast<uint32_t>(d.n_tok) * p.rec_bytes;
            mbar_arrive_expect_tx(&s.afull[aslot], abytes);
            bulk_g2s(s.act + static_cast<size_t>(aslot) * p.act_bytes,
                     p.qrec + static_cast<size_t>(d.pair[0]) * p.rec_bytes, abytes, &s.afull[aslot]);
            ++n_act;
            d.aslot = aslot;
            const int c_end = min(p.H, (j + 1) * p.dr);
            for (int c0 = j * p.dr; c0 < c_end && ok; c0 += p.sr_down) {
                d.row0 = c0;
                d.nrows = min(p.sr_down, c_end - c0);
                d.first = (c0 == j * p.dr);
                d.last = (c0 + p.sr_down >= c_end);
                const size_t r = static_cast<size_t>(d.e) * p.H + c0;
                ok = issue(d, ex.w_down + r * rb_d, static_cast<uint32_t>(d.nrows * rb_d), ex.s_down + r,
                           static_cast<uint32_t>(d.nrows * 4));
            }
            if (++aslot == kActSlots) {
                aslot = 0;
                aphase ^= 1u;
            }
        }
    }
    if (!ok) record_status(p.status, MOE_EDEVICE_TIMEOUT);
    // tell the consumers to stop (after the route marker, if none was queued yet)
    if (!marked && acquire_stage()) {
        s.desc[stage].type = D_ROUTE;
        mbar_arrive(&s.full[stage]);
        advance();
    }
    if (acquire_stage()) {
        s.desc[stage].type = D_EXIT;
        mbar_arrive(&s.full[stage]);
        advance();
    }
    // drain: wait until every copy issued into this CTA's shared memory has landed
    for (int st = 0; st < p.nstage; ++st) {
        const long uses = n_issued / p.nstage + (st < n_issued % p.nstage ? 1 : 0);
        if (uses > 0) mbar_wait(&s.full[st], static_cast<uint32_t>((uses - 1) & 1), kProducerWait);
    }
    for (int a = 0; a < kActSlots; ++a) {
        const long uses = n_act / kActSlots + (a < n_act % kActSlots ? 1 : 0);
        if (uses > 0) mbar_wait(&s.afull[a], static_cast<uint32_t>((uses - 1) & 1), kProducerWait);
    }
}

// ------------------------------------------------------------------ Q8_0 helpers
// Warp-collective: quantises one 32-value block held one value per lane to
// Q8_0 and stores it permuted for dp4a: words 0-3 to w_lo, 4-7 to w_hi, the
// scale and the block code sum.
template <int QT>
__device__ __forceinline__ void store_q8_block_warp(float v, uint32_t* w_lo, uint32_t* w_hi, float* d_out,
                                                    int32_t* sum_out) {
    const int lane = threadIdx.x & 31;
    float d;
    const int q = q8_0_lane(v, &d);
    const uint32_t word = perm_word<QT>(q, lane);
    const int sum = __reduce_add_sync(0xffffffffu, q);
    if (lane < 4) {
        w_lo[lane] = word;
    } else if (lane < 8) {
        w_hi[lane - 4] = word;
    }
    if (lane == 0) {
        *d_out = d;
        *sum_out = sum;
    }
}

// One thread: Q8_0 of 32 bf16 values (same arithmetic as q8_0_lane), stored
// permuted for dp4a.
template <int QT>
__device__ __forceinline__ void quantize_block_thread(const uint16_t* src, uint4* q0, uint4* q1, float* qd,
                                                      int32_t* qs) {
    float v[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint4 u = reinterpret_cast<const uint4*>(src)[c];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[8 * c + 2 * i] = bf16_bits_to_f32(static_cast<uint16_t>(w[i]));
            v[8 * c + 2 * i + 1] = bf16_bits_to_f32(static_cast<uint16_t>(w[i] >> 16));
        }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const float d = __fdiv_rn(amax, 127.0f);
    int q[32];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        int qi = 0;
        if (d != 0.0f) qi = static_cast<int>(fminf(fmaxf(roundf(__fdiv_rn(v[i], d)), -127.0f), 127.0f));
        q[i] = qi;
        sum += qi;
    }
    uint32_t o[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) word |= (static_cast<uint32_t>(q[perm_src<QT>(w, i)]) & 0xFFu) << (8 * i);
        o[w] = word;
    }
    *q0 = make_uint4(o[0], o[1], o[2], o[3]);
    *q1 = make_uint4(o[4], o[5], o[6], o[7]);
    *qd = d;
    *qs = sum;
}

// ------------------------------------------------------------------ consumers
// Q8_0 of every token's x (all consumer threads, four per 32-block), stored
// permuted for dp4a against qtype QT.  Same arithmetic as q8_0_lane.
template <int QT>
__device__ void quantize_x(const FusedParams& p, const Smem& s) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int nbH = p.H / 32, ntask = p.T * nbH * 4;
    uint8_t* scr = s.qscratch + (tid >> 5) * 256 + (lane >> 2) * 32;  // this lane group's block
    for (int base = 0; base < ntask; base += kConsumers) {
        const int task = base + tid;
        const bool active = task < ntask;
        const int blk = task >> 2, part = task & 3;
        float v[8];
        float amax = 0.0f;
        if (active) {
            const int t = blk / nbH, b = blk % nbH;
            const uint4 u = reinterpret_cast<const uint4*>(s.xs + static_cast<size_t>(t) * p.H + 32 * b)[part];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = bf16_bits_to_f32(static_cast<uint16_t>(w[i]));
                v[2 * i + 1] = bf16_bits_to_f32(static_cast<uint16_t>(w[i] >> 16));
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const float d = __fdiv_rn(amax, 127.0f);
        int sum = 0;
        uint32_t packed[2] = {0u, 0u};
        if (active) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                int qi = 0;
                if (d != 0.0f) qi = static_cast<int>(fminf(fmaxf(roundf(__fdiv_rn(v[i], d)), -127.0f), 127.0f));
                sum += qi;
                packed[i >> 2] |= (static_cast<uint32_t>(qi) & 0xFFu) << (8 * (i & 3));
            }
            *reinterpret_cast<uint2*>(scr + 8 * part) = make_uint2(packed[0], packed[1]);
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        __syncwarp();
        if (active) {
            uint32_t o[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int w = 2 * part + k;
                uint32_t word = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) word |= static_cast<uint32_t>(scr[perm_src<QT>(w, i)]) << (8 * i);
                o[k] = word;
            }
            uint32_t* dst = reinterpret_cast<uint32_t*>(part < 2 ? s.q0 + blk : s.q1 + blk) + 2 * (part & 1);
            *reinterpret_cast<uint2*>(dst) = make_uint2(o[0], o[1]);
            if (part == 0) {
                s.qd[blk] = d;
                s.qs[blk] = sum;
            }
        }
        __syncwarp();
    }
}

__device__ void consumer_init(const FusedParams& p, const Smem& s) {
    const int tid = threadIdx.x;
    const int n16 = p.T * p.H / 8;
    for (int i = tid; i < n16; i += kConsumers)
        reinterpret_cast<uint4*>(s.xs)[i] = reinterpret_cast<const uint4*>(p.x)[i];
    for (int e = tid; e < p.E; e += kConsumers) s.bias[e] = __ldg(p.bias + e);
    consumers_sync();
}

// One router stage: logits of rows e0 .. e0 + nrows - 1 for every token.
template <int NT>
__device__ void consume_router(const FusedParams& p, const Smem& s, int e0, int nrows, const uint8_t* sbuf) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h4 = p.H / 4;
    double acc[kMaxRouterRows][NT];
#pragma unroll
    for (int q = 0; q < kMaxRouterRows; ++q)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[q][t] = 0.0;
    for (int j = tid; j < h4; j += kConsumers) {
        double xv[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const int tt = t < p.T ? t : 0;
            const uint2 u = reinterpret_cast<const uint2*>(s.xs + static_cast<size_t>(tt) * p.H)[j];
            xv[t][0] = bf16_bits_to_f32(static_cast<uint16_t>(u.x));
            xv[t][1] = bf16_bits_to_f32(static_cast<uint16_t>(u.x >> 16));
            xv[t][2] = bf16_bits_to_f32(static_cast<uint16_t>(u.y));
            xv[t][3] = bf16_bits_to_f32(static_cast<uint16_t>(u.y >> 16));
        }
#pragma unroll
        for (int q = 0; q < kMaxRouterRows; ++q) {
            if (q < nrows) {
                const float4 wv = reinterpret_cast<const float4*>(sbuf + static_cast<size_t>(q) * 4 * p.H)[j];
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    acc[q][t] = fma(xv[t][0], static_cast<double>(wv.x), acc[q][t]);
                    acc[q][t] = fma(xv[t][1], static_cast<double>(wv.y), acc[q][t]);
                    acc[q][t] = fma(xv[t][2], static_cast<double>(wv.z), acc[q][t]);
                    acc[q][t] = fma(xv[t][3], static_cast<double>(wv.w), acc[q][t]);
                }
            }
        }
    }
#pragma unroll
    for (int q = 0; q < kMaxRouterRows; ++q)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (q < nrows) {
                const double v = warp_sum_f64(acc[q][t]);
                if (lane == 0) s.red[(warp * kMaxRouterRows + q) * kMaxT + t] = v;
            }
        }
    consumers_sync();
    if (tid < nrows * p.T) {
        const int q = tid / p.T, t = tid % p.T;
        double sum = 0.0;
        for (int w = 0; w < kConsumerWarps; ++w) sum += s.red[(w * kMaxRouterRows + q) * kMaxT + t];
        p.logits[static_cast<size_t>(t) * p.E + e0 + q] = __double2float_rn(sum);
        red_release_add_gpu(&p.sync->router_done, 1);  // one count per logit
    }
}

// Selection and union for the whole batch, computed by all consumer threads
// of every CTA into shared memory once every logit has been counted.
// noaux_tc (DeepSeek-V3 routing, as [HN] "구현된 주요 기능" names it):
// s = sigmoid(logit), b = s + bias; group score = sum of the two largest b;
// keep topk_group groups; keep the top_k experts of kept groups by b; ties to
// the lower index.  A kept group / expert finds its rank by counting the
// candidates that order before it (vectorised scans over shared memory).
__device__ void route_cta(const FusedParams& p, const Smem& s) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T, K = p.K, E = p.E, G = p.G, TG = p.TG, gsz = E / G;
    float* sv = reinterpret_cast<float*>(s.xs);    // [T][E] unbiased scores
    float* bv = sv + T * E;                        // [T][E] biased scores
    float* gs = bv + T * E;                        // [T][G] group scores
    int* kg = reinterpret_cast<int*>(gs + T * G);  // [T][TG] kept groups (any order)
    int* ch = s.chosen;                            // [T][32] chosen experts, slot order
    int* bpre = s.bpre;
    const bool vec = (gsz % 4 == 0) && (E % 4 == 0);
    if (tid == 0) {
        bool okc = false;
        for (long i = 0; i < kConsumerWait; ++i) {
            if (ld_relaxed_gpu(&p.sync->router_done) >= T * E) {
                okc = ld_acquire_gpu(&p.sync->router_done) >= T * E;
                break;
            }
            __nanosleep(32);
        }
        if (!okc) record_status(p.status, MOE_EDEVICE_TIMEOUT);
    }
    consumers_sync();
    for (int i = tid; i < T * E; i += kConsumers) {
        const int e = i % E;
        const double l = static_cast<double>(__ldcg(p.logits + i));
        const float sc = __double2float_rn(1.0 / (1.0 + exp(-l)));
        sv[i] = sc;
        bv[i] = __fadd_rn(sc, s.bias[e]);
    }
    for (int i = tid; i < T * 32; i += kConsumers) ch[i] = -1;
    if (tid < 32) s.bmap[tid] = 0;
    consumers_sync();
    // group scores: one warp per (token, group); lane-local top-2, then a warp merge
    for (int pg = warp; pg < T * G; pg += kConsumerWarps) {
        const int t = pg / G, g = pg % G;
        const float* bg = bv + t * E + g * gsz;
        float m1 = -INFINITY, m2 = -INFINITY;
        for (int e = lane; e < gsz; e += 32) {
            const float v = bg[e];
            if (v > m1) {
                m2 = m1;
                m1 = v;
            } else if (v > m2) {
                m2 = v;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float o1 = __shfl_xor_sync(0xffffffffu, m1, o), o2 = __shfl_xor_sync(0xffffffffu, m2, o);
            const float n1 = fmaxf(m1, o1);
            m2 = fmaxf(fminf(m1, o1), fmaxf(m2, o2));
            m1 = n1;
        }
        if (lane == 0) gs[pg] = __fadd_rn(m1, m2);
    }
    consumers_sync();
    // kept groups: rank each group's score among its token's groups
    for (int i = tid; i < T * G; i += kConsumers) {
        const int t = i / G, g = i % G;
        const float v = gs[i];
        int r = 0;
        for (int g2 = 0; g2 < G; ++g2) {
            const float w = gs[t * G + g2];
            r += (w > v) || (w == v && g2 < g);
        }
        if (r < TG) kg[t * TG + r] = g;
    }
    consumers_sync();
    // experts: rank each expert of a kept group among all experts of kept groups
    for (int i = tid; i < T * E; i += kConsumers) {
        const int t = i / E, e = i % E, ge = e / gsz;
        bool kept = false;
        for (int j = 0; j < TG; ++j) kept |= kg[t * TG + j] == ge;
        if (!kept) continue;
        const float v = bv[i];
        int r = 0;
        for (int j = 0; j < TG; ++j) {
            const int base = kg[t * TG + j] * gsz;
            const float* bg = bv + t * E + base;
            if (vec) {
                const float4* bg4 = reinterpret_cast<const float4*>(bg);
#pragma unroll 4
                for (int q = 0; q < gsz / 4; ++q) {
                    const float4 w = bg4[q];
                    const int x = base + 4 * q;
                    r += (w.x > v) | ((w.x == v) & (x < e));
                    r += (w.y > v) | ((w.y == v) & (x + 1 < e));
                    r += (w.z > v) | ((w.z == v) & (x + 2 < e));
                    r += (w.w > v) | ((w.w == v) & (x + 3 < e));
                }
            } else {
                for (int q = 0; q < gsz; ++q) r += (bg[q] > v) | ((bg[q] == v) & (base + q < e));
            }
        }
        if (r < K) ch[t * 32 + r] = e;
    }
    consumers_sync();
    // per token (warp t, lane k = slot): guard, gate weight, entry, bitmap
    if (warp < T) {
        const int t = warp;
        int e = lane < K ? ch[t * 32 + lane] : 0;
        if (lane < K && (e < 0 || e >= E)) {  // only reachable with NaN scores
            record_status(p.status, MOE_EDEVICE_INDEX);
            e = 0;
        }
        const float sk = lane < K ? sv[t * E + e] : 0.0f;
        float den = 0.0f;  // sum in slot order, as the definition orders it
        for (int j = 0; j < K; ++j) den = __fadd_rn(den, __shfl_sync(0xffffffffu, sk, j));
        if (lane < K) {
            ch[t * 32 + lane] = e;
            s.rt_w[t * K + lane] = __fmul_rn(__fdiv_rn(sk, den), p.rsf);
            s.ent[t * K + lane] = e;
            atomicOr(&s.bmap[e >> 5], 1u << (e & 31));
        }
    }
    consumers_sync();
    if (warp == 0) {  // exclusive prefix of the bitmap's popcounts
        const int c = __popc(s.bmap[lane]);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n2 = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n2;
        }
        bpre[lane] = incl - c;
        if (lane == 31) bpre[32] = incl;
    }
    consumers_sync();
    // union of the T*K entries: (expert ascending, token ascending) positions
    const int n = T * K;
    for (int i = tid; i < n; i += kConsumers) {
        const int t = i / K, e = s.ent[i];
        int before = 0, same_before = 0, first = 1;
        for (int jx = 0, tj = 0, kj = 0; jx < n; ++jx) {  // tj = jx / K without a division
            const int ej = s.ent[jx];
            before += ej < e;
            same_before += (ej == e) & (tj < t);
            first &= !((ej == e) & (jx < i));
            if (++kj == K) {
                kj = 0;
                ++tj;
            }
        }
        const int rank = bpre[e >> 5] + __popc(s.bmap[e >> 5] & ((1u << (e & 31)) - 1u));
        const int pos = before + same_before;
        s.rt_ptok[pos] = t;
        s.rt_pair_of[i] = pos;
        if (first) {
            s.rt_uniq[rank] = e;
            s.rt_off[rank] = before;
        }
    }
    if (tid == 0) {
        const int U = bpre[32];
        *s.rt_U = U;
        s.rt_off[U] = n;
    }
    consumers_sync();
    if (tid == 0) mbar_arrive(s.route_bar);
    // the routing outputs the caller can see, written once (off the critical path)
    if (blockIdx.x == 0) {
        for (int i = tid; i < n; i += kConsumers) {
            p.idx[i] = ch[(i / K) * 32 + (i % K)];
            p.w[i] = s.rt_w[i];
        }
    }
}

// Activations of one token for the blocks a lane owns (b = lane + 32 j), in registers.
template <int NC>
struct ActRegs {
    uint4 a0[NC];
    uint4 a1[NC];
};

// up/gate stage, NT = 1: the token's Q8_0(x) words are in registers.
template <int QT>
__device__ __forceinline__ void consume_ug_reg(const FusedParams& p, const Smem& s, float* dst, int row0,
                                               const uint8_t* sbuf, const ActRegs<kRegChunksUg>& ar) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nbH = p.H / 32;
    const size_t rb = static_cast<size_t>(p.H) * QT / 8;
    const uint8_t* wrow = sbuf + warp * rb;
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < kRegChunksUg; ++j) {
        const int b = lane + 32 * j;
        if (b < nbH) {
            const WBlock<QT> wb = load_wblock_smem<QT>(wrow, b);
            const int isum = block_dot<QT>(wb, ar.a0[j], ar.a1[j], s.qs[b]);
            acc = fmaf(static_cast<float>(isum), s.qd[b], acc);
        }
    }
    const float v = warp_sum_f32(acc);
    if (lane == 0) {
        const float* sc = reinterpret_cast<const float*>(sbuf + p.stage_bytes);
        dst[row0 % kUgTileRows + warp] = __fmul_rn(v, sc[warp]);
    }
}

// up/gate stage, NT > 1: activations read from the shared-memory cache.
template <int QT, int NT>
__device__ __forceinline__ void consume_ug_smem(const FusedParams& p, const Smem& s, const Desc& d, float* dst,
                                                const uint8_t* sbuf) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nbH = p.H / 32;
    const size_t rb = static_cast<size_t>(p.H) * QT / 8;
    const uint8_t* wrow = sbuf + warp * rb;
    const int n_tok = d.n_tok;
    int tok[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) tok[t] = t < n_tok ? d.tok[t] : 0;
    float acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.0f;
#pragma unroll 2
    for (int b = lane; b < nbH; b += 32) {
        const WBlock<QT> wb = load_wblock_smem<QT>(wrow, b);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < n_tok) {
                const int q = tok[t] * nbH + b;
                const int isum = block_dot<QT>(wb, s.q0[q], s.q1[q], s.qs[q]);
                acc[t] = fmaf(static_cast<float>(isum), s.qd[q], acc[t]);
            }
        }
    }
    const float* sc = reinterpret_cast<const float*>(sbuf + p.stage_bytes);
    const int r = d.row0 % kUgTileRows + warp;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (t < n_tok) {
            const float v = warp_sum_f32(acc[t]);
            if (lane == 0) dst[t * kUgTileRows + r] = __fmul_rn(v, sc[warp]);
        }
    }
}

// down stage, NT = 1: the pair's Q8_0(h) words are in registers (loaded per tile).
template <int QT>
__device__ __forceinline__ void consume_down_reg(const FusedParams& p, int row0, int nrows, int pair,
                                                 const uint8_t* sbuf, const ActRegs<kRegChunksDown>& ar,
                                                 const float* ad, const int32_t* as) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nbI = p.I / 32;
    const size_t rb = static_cast<size_t>(p.I) * QT / 8;
    const float* sc = reinterpret_cast<const float*>(sbuf + p.stage_bytes);
    float acc[kMaxDownRowsPerWarp];
#pragma unroll
    for (int k = 0; k < kMaxDownRowsPerWarp; ++k) {
        acc[k] = 0.0f;
        const int r = warp + kConsumerWarps * k;
        if (r < nrows) {
            const uint8_t* wrow = sbuf + r * rb;
#pragma unroll
            for (int j = 0; j < kRegChunksDown; ++j) {
                const int b = lane + 32 * j;
                if (b < nbI) {
                    const WBlock<QT> wb = load_wblock_smem<QT>(wrow, b);
                    const int isum = block_dot<QT>(wb, ar.a0[j], ar.a1[j], as[b]);
                    acc[k] = fmaf(static_cast<float>(isum), ad[b], acc[k]);
                }
            }
        }
    }
#pragma unroll
    for (int k = 0; k < kMaxDownRowsPerWarp; ++k) {
        const int r = warp + kConsumerWarps * k;
        if (r < nrows) {
            const float v = warp_sum_f32(acc[k]);
            if (lane == 0) p.y[static_cast<size_t>(pair) * p.H + row0 + r] = __fmul_rn(v, sc[r]);
        }
    }
}

// down stage, NT > 1: activations read from the tile's shared-memory slot.
template <int QT, int NT>
__device__ __forceinline__ void consume_down_smem(const FusedParams& p, const Smem& s, const Desc& d,
                                                  const uint8_t* sbuf) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nbI = p.I / 32;
    const size_t rb = static_cast<size_t>(p.I) * QT / 8;
    const uint8_t* act = s.act + static_cast<size_t>(d.aslot) * p.act_bytes;
    const float* sc = reinterpret_cast<const float*>(sbuf + p.stage_bytes);
    const int n_tok = d.n_tok, nrows = d.nrows, row0 = d.row0;
    int pair[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) pair[t] = d.pair[t];
    for (int r = warp; r < nrows; r += kConsumerWarps) {
        const uint8_t* wrow = sbuf + r * rb;
        float acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.0f;
#pragma unroll 2
        for (int b = lane; b < nbI; b += 32) {
            const WBlock<QT> wb = load_wblock_smem<QT>(wrow, b);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (t < n_tok) {
                    const uint8_t* rec = act + static_cast<size_t>(t) * p.rec_bytes;
                    const uint4 a0 = reinterpret_cast<const uint4*>(rec)[b];
                    const uint4 a1 = reinterpret_cast<const uint4*>(rec + p.I / 2)[b];
                    const float da = reinterpret_cast<const float*>(rec + p.I)[b];
                    const int as = reinterpret_cast<const int32_t*>(rec + p.I + nbI * 4)[b];
                    acc[t] = fmaf(static_cast<float>(block_dot<QT>(wb, a0, a1, as)), da, acc[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < n_tok) {
                const float v = warp_sum_f32(acc[t]);
                if (lane == 0) p.y[static_cast<size_t>(pair[t]) * p.H + row0 + r] = __fmul_rn(v, sc[r]);
            }
        }
    }
}

// Hands a finished tile (or the end) to the epilogue warp through task slot tb.
__device__ __forceinline__ void push_task(const Smem& s, int tb, const Desc* d, int type) {
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid == 0) {
        Task& tk = s.task[tb];
        tk.type = type;
        if (d) {
            tk.n_tok = d->n_tok;
            tk.blk = d->blk;
            tk.cslot = d->cslot;
            tk.n_experts = d->n_experts;
#pragma unroll
            for (int t = 0; t < kMaxT; ++t) tk.pair[t] = d->pair[t];
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.tfull[tb]);
}

template <int QT, int NT>
__device__ void consumer(const FusedParams& p, const Smem& s) {
    const int tid = threadIdx.x, lane = tid & 31;
    const size_t slot_bytes = static_cast<size_t>(p.stage_bytes) + kScaleBytes;
    consumer_init(p, s);
    int stage = 0, aslot = 0, tb = 0;
    uint32_t phase = 0, aphase = 0;
    uint32_t tph[kTaskSlots] = {0, 0};
    // Waits for the current stage; returns its type (D_EXIT on timeout).
    auto next_type = [&]() -> int {
        if (!mbar_wait(&s.full[stage], phase, kConsumerWait)) {
            record_status(p.status, MOE_EDEVICE_TIMEOUT);
            return D_EXIT;
        }
        return s.desc[stage].type;
    };
    auto release = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty[stage]);
        if (++stage == p.nstage) {
            stage = 0;
            phase ^= 1u;
        }
    };
    // Waits until the epilogue warp has finished with task slot tb.
    auto task_slot_free = [&]() -> bool {
        if (!mbar_wait(&s.tfree[tb], tph[tb] ^ 1u, kConsumerWait)) {
            record_status(p.status, MOE_EDEVICE_TIMEOUT);
            return false;
        }
        return true;
    };
    auto next_task = [&]() {
        tph[tb] ^= 1u;
        tb ^= 1;
    };
    int type = next_type();
    // phase A: router rows, then (at the route marker) Q8_0 of x and the routing
    while (type == D_ROUTER) {
        const int e0 = s.desc[stage].e, nrows = s.desc[stage].nrows;
        consume_router<NT>(p, s, e0, nrows, s.ring + stage * slot_bytes);
        release();
        type = next_type();
    }
    quantize_x<QT>(p, s);
    consumers_sync();
    if (type == D_ROUTE) {
        route_cta(p, s);
        release();
        type = next_type();
    }
    // phase B: up/gate tiles
    bool ok = true;
    {
        ActRegs<kRegChunksUg> ar;
        if constexpr (NT == 1) {
            const int nbH = p.H / 32;
#pragma unroll
            for (int j = 0; j < kRegChunksUg; ++j) {
                const int b = lane + 32 * j;
                ar.a0[j] = b < nbH ? s.q0[b] : make_uint4(0, 0, 0, 0);
                ar.a1[j] = b < nbH ? s.q1[b] : make_uint4(0, 0, 0, 0);
            }
        }
        while (type == D_UG) {
            const Desc& d = s.desc[stage];
            const uint8_t* sbuf = s.ring + stage * slot_bytes;
            if (d.first && !task_slot_free()) {
                ok = false;
                break;
            }
            float* dst = (d.mat == 0 ? s.gbuf : s.ubuf) + tb * kMaxT * kUgTileRows;
            if constexpr (NT == 1) {
                consume_ug_reg<QT>(p, s, dst, d.row0, sbuf, ar);
            } else {
                consume_ug_smem<QT, NT>(p, s, d, dst, sbuf);
            }
            if (d.last) {
                push_task(s, tb, &d, D_UG);
                next_task();
            }
            release();
            type = next_type();
        }
    }
    // phase C: down tiles
    if (ok) {
        ActRegs<kRegChunksDown> ar;
        const float* ad = nullptr;
        const int32_t* as = nullptr;
        while (type == D_DOWN) {
            const Desc& d = s.desc[stage];
            const uint8_t* sbuf = s.ring + stage * slot_bytes;
            if (d.first) {
                if (!mbar_wait(&s.afull[aslot], aphase, kConsumerWait)) {
                    record_status(p.status, MOE_EDEVICE_TIMEOUT);
                    break;
                }
                if constexpr (NT == 1) {
                    const uint8_t* rec = s.act + static_cast<size_t>(aslot) * p.act_bytes;
                    const int nbI = p.I / 32;
#pragma unroll
                    for (int j = 0; j < kRegChunksDown; ++j) {
                        const int b = lane + 32 * j;
                        ar.a0[j] = b < nbI ? reinterpret_cast<const uint4*>(rec)[b] : make_uint4(0, 0, 0, 0);
                        ar.a1[j] = b < nbI ? reinterpret_cast<const uint4*>(rec + p.I / 2)[b]
                                           : make_uint4(0, 0, 0, 0);
                    }
                    ad = reinterpret_cast<const float*>(rec + p.I);
                    as = reinterpret_cast<const int32_t*>(rec + p.I + nbI * 4);
                }
            }
            if constexpr (NT == 1) {
                consume_down_reg<QT>(p, d.row0, d.nrows, d.pair[0], sbuf, ar, ad, as);
            } else {
                consume_down_smem<QT, NT>(p, s, d, sbuf);
            }
            if (d.last) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.aempty[aslot]);
                if (++aslot == kActSlots) {
                    aslot = 0;
                    aphase ^= 1u;
                }
                if (!task_slot_free()) break;
                push_task(s, tb, &d, D_DOWN);
                next_task();
            }
            release();
            type = next_type();
        }
    }
    // hand the end to the epilogue warp
    if (task_slot_free()) push_task(s, tb, nullptr, D_EXIT);
}

// ------------------------------------------------------------------ epilogue warp
template <int QT>
__device__ void epilogue_warp(const FusedParams& p, const Smem& s) {
    const int lane = threadIdx.x & 31;
    const int nbI = p.I / 32;
    const int P = p.T * p.K;
    int tb = 0;
    uint32_t eph[kTaskSlots] = {0, 0};
    while (true) {
        if (!mbar_wait(&s.tfull[tb], eph[tb], kEpilogueWait)) {
            record_status(p.status, MOE_EDEVICE_TIMEOUT);
            break;
        }
        const Task& tk = s.task[tb];
        const int type = tk.type;
        if (type == D_EXIT) break;
        if (type == D_UG) {
            // SwiGLU + Q8_0 of the tile's 32 h rows for each token -> activation records
            const float* g = s.gbuf + tb * kMaxT * kUgTileRows;
            const float* u = s.ubuf + tb * kMaxT * kUgTileRows;
            for (int t = 0; t < tk.n_tok; ++t) {
                const float h = swiglu(g[t * kUgTileRows + lane], u[t * kUgTileRows + lane]);
                uint8_t* rec = p.qrec + static_cast<size_t>(tk.pair[t]) * p.rec_bytes;
                store_q8_block_warp<QT>(h, reinterpret_cast<uint32_t*>(rec + 16 * tk.blk),
                                        reinterpret_cast<uint32_t*>(rec + p.I / 2 + 16 * tk.blk),
                                        reinterpret_cast<float*>(rec + p.I) + tk.blk,
                                        reinterpret_cast<int32_t*>(rec + p.I + nbI * 4) + tk.blk);
            }
            fence_proxy_async_global();
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(p.ug_done + tk.cslot, 1);
        } else {
            // count the down tile for its row block; the CTA completing a block combines it
            const int blk = tk.blk, n_experts = tk.n_experts;
            int last = 0;
            if (lane == 0) {
                __threadfence();
                last = atomicAdd(p.rb_done + blk, 1) == n_experts - 1;
                if (last) __threadfence();
            }
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                const int c0 = blk * p.dr, nr = min(p.dr, p.H - c0);
                for (int i = lane; i < p.T * nr; i += 32) {
                    const int t = i / nr, c = c0 + i % nr;
                    float o = p.has_shared ? __ldcg(p.y + static_cast<size_t>(P + t) * p.H + c) : 0.0f;
                    for (int k = 0; k < p.K; ++k) {
                        const int pr = s.rt_pair_of[t * p.K + k];
                        const float wk = s.rt_w[t * p.K + k];
                        o = __fadd_rn(o, __fmul_rn(wk, __ldcg(p.y + static_cast<size_t>(pr) * p.H + c)));
                    }
                    if (p.out_bf16) {
                        static_cast<uint16_t*>(p.out)[static_cast<size_t>(t) * p.H + c] = f32_to_bf16_bits(o);
                    } else {
                        static_cast<float*>(p.out)[static_cast<size_t>(t) * p.H + c] = o;
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.tfree[tb]);
        eph[tb] ^= 1u;
        tb ^= 1;
    }
}

template <int QT, int NT>
__global__ void __launch_bounds__(kThreadsF, 1) k_decode_fused(const __grid_constant__ FusedParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const Smem s = carve(smem_raw, p);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // Touch every parameter word now, while the memory system is idle: a
    // constant-cache miss on a parameter first read in the middle of the
    // kernel would queue behind the weight stream.
    {
        const int* pw = reinterpret_cast<const int*>(&p);
        int acc = 0;
        for (int i = lane; i < static_cast<int>(sizeof(FusedParams) / 4); i += 32) acc ^= pw[i];
        if (acc == 0x7fffffff && tid == kThreadsF) s.flag[3] = acc;  // keeps the reads
    }
    if (tid == 0) {
        for (int i = 0; i < p.nstage; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], kConsumerWarps);
        }
        for (int i = 0; i < kActSlots; ++i) {
            mbar_init(&s.afull[i], 1);
            mbar_init(&s.aempty[i], kConsumerWarps);
        }
        for (int i = 0; i < kTaskSlots; ++i) {
            mbar_init(&s.tfull[i], kConsumerWarps);
            mbar_init(&s.tfree[i], 1);
        }
        mbar_init(s.route_bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == kProducerWarp) {
        if (lane == 0) producer<QT>(p, s);
    } else if (warp == kEpilogueWarp) {
        epilogue_warp<QT>(p, s);
    } else {
        consumer<QT, NT>(p, s);
    }
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(&p.sync->exit_count, 1) == static_cast<int>(gridDim.x) - 1) {
            // last CTA out: reset the counters for the next call on this workspace
            for (int i = 0; i <= p.E; ++i) p.ug_done[i] = 0;
            for (int i = 0; i < p.n_dt; ++i) p.rb_done[i] = 0;
            p.sync->ticket = 0;
            p.sync->router_done = 0;
            p.sync->route_ready = 0;
            p.sync->exit_count = 0;
            __threadfence();
        }
    }
}

template <int QT>
const void* fused_kernel(int nt) {
    return nt == 1 ? reinterpret_cast<const void*>(k_decode_fused<QT, 1>)
                   : reinterpret_cast<const void*>(k_decode_fused<QT, kMaxT>);
}

}  // namespace

bool fused_geometry(FusedParams& p, int qtype) {
    // the routing scratch (scores, biased scores, group scores and flags of
    // every token) reuses the bf16 copy of x: needs 6 E <= H
    if (p.T < 1 || p.T > kMaxT || p.K * p.T > 128 || 6 * p.E > p.H) return false;
    const size_t rb_ug = static_cast<size_t>(p.H) * qtype / 8, rb_d = static_cast<size_t>(p.I) * qtype / 8;
    size_t stage = std::max(static_cast<size_t>(4) * p.H, kStageRows * rb_ug);
    stage = (stage + 127) / 128 * 128;
    const int sr = static_cast<int>(stage / (kStageRows * rb_d)) * kStageRows;
    if (sr < kStageRows || sr > kConsumerWarps * kMaxDownRowsPerWarp || sr * 4 > kScaleBytes) return false;
    p.stage_bytes = static_cast<int>(stage);
    p.rps = std::min<int>(kMaxRouterRows, static_cast<int>(stage / (4 * static_cast<size_t>(p.H))));
    p.n_rt = (p.E + p.rps - 1) / p.rps;
    p.sr_down = sr;
    p.dr = sr * kDownStagesPerTile;
    p.n_ugt = p.I / kUgTileRows;
    p.n_dt = (p.H + p.dr - 1) / p.dr;
    p.rec_bytes = static_cast<int>(fused_record_bytes(p.I));
    p.act_bytes = static_cast<int>(a16(static_cast<size_t>(p.T) * p.rec_bytes));
    const bool regs_fit = p.H / 32 <= 32 * kRegChunksUg && p.I / 32 <= 32 * kRegChunksDown;
    p.nt = (p.T == 1 && regs_fit) ? 1 : kMaxT;
    const size_t cap = 227 * 1024;
    for (int ns = 8; ns >= 2; --ns) {
        p.nstage = ns;
        if (layout_of(p).total <= cap) return true;
    }
    return false;
}

size_t fused_smem_bytes(const FusedParams& p) { return layout_of(p).total; }

cudaError_t launch_decode_fused(const FusedParams& p, cudaStream_t st) {
    static int sms[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && sms[dev] == 0) {
        e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    const int grid = (dev >= 0 && dev < 64) ? sms[dev] : 148;
    const size_t smem = fused_smem_bytes(p);
    const void* kern;
    switch (p.routed.qtype) {
        case MOE_Q_INT4: kern = fused_kernel<4>(p.nt); break;
        case MOE_Q_INT8: kern = fused_kernel<8>(p.nt); break;
        case MOE_Q_INT2: kern = fused_kernel<2>(p.nt); break;
        default: return cudaErrorInvalidValue;
    }
    e = ensure_smem(kern, smem);
    if (e != cudaSuccess) return e;
    void* args[] = {const_cast<FusedParams*>(&p)};
    e = cudaLaunchKernel(kern, dim3(grid), dim3(kThreadsF), args, smem, st);
    if (e != cudaSuccess) return e;
    return counted(cudaGetLastError());
}

}  // namespace moe
