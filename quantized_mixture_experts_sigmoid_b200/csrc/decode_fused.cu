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
// Roles (one CTA per SM, 20 warps):
//  * warp 18, the producer, streams weight rows into a shared-memory ring
//    with bulk copies (cp.async.bulk, non-multicast TMA) completing on
//    mbarriers;
//  * warps 0-15, the consumers, take one ring stage at a time and form the
//    integer dot products with dp4a; once their router rows are done they
//    also route the batch (every CTA computes the same routing from the
//    published router scores, one expert per thread);
//  * warps 16-17, the epilogue warps, each finish the tiles handed over
//    through one task slot (SwiGLU and Q8_0 of h for up/gate tiles;
//    completion counting and the combine for down tiles), so the consumers
//    never wait on fences or atomics;
//  * warp 19, the helper, copies each down tile's activation records once
//    the expert's h is complete, so the producer never waits on another CTA.
//
// Work is one global ticket sequence claimed by the producers:
//      router rows | shared up/gate tiles | then, per distinct routed expert
//      u: its up/gate tiles, followed by the down tiles of expert u - 8; the
//      last routed experts' down tiles at the end, the shared expert's down
//      tiles before the very last expert's,
// so every dependency points to an earlier ticket, far enough back that it is
// usually complete when claimed.  The consumers that finish a router row
// publish its scores (sigmoid of the fp32-rounded logit) in 64-bit slots
// tagged with the launch number; every CTA's consumers poll those slots, so
// the data and its readiness arrive in one load.  A producer claims routed
// tiles once its CTA's consumers have routed.  An up/gate tile is 32 rows of h for one
// expert; its epilogue writes Q8_0(h) as a pre-permuted activation record.  A
// down tile's weight stages stream at once; its records follow when the
// expert's h tiles are all done.  The CTA that completes a row block of the
// output combines it (shared + sum_k w_k y_k in slot order), so the result is
// deterministic.
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
constexpr int kGroups = 2;  // consumer groups: ring stage n belongs to group n % kGroups
constexpr int kGroupWarps = kConsumerWarps / kGroups;
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kEpilogueWarps = 2;    // one per task slot
constexpr int kEpilogueWarp0 = kConsumerWarps;
constexpr int kProducerWarp = kEpilogueWarp0 + kEpilogueWarps;
constexpr int kHelperWarp = kProducerWarp + 1;  // routing, then the activation copies
constexpr int kThreadsF = (kHelperWarp + 1) * 32;
constexpr int kMaxT = kFusedMaxTokens;
constexpr int kStageRows = 16;       // up/gate rows per stage (two per warp of a group)
constexpr int kUgTileRows = 32;      // one Q8_0 block of h
constexpr int kDownStagesPerTile = 2;  // one per consumer group
constexpr int kMaxRouterRows = 4;    // router rows per stage
constexpr int kMaxDownRowsPerWarp = 8;
constexpr int kActSlots = 2;         // activation-record slots of their own
constexpr int kMaxActSlots = 6;      // with up to 4 more in the x cache, free once routed
constexpr int kTaskSlots = kEpilogueWarps;
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
// (The drains that wait for this CTA's own copies in flight keep kProducerWait
// whatever the test limit below says: a copy may not land after the exit.)
constexpr int kBarConsumers = 1;     // named barrier id of the consumer warps (group g: 2 + g)
static_assert(kStageRows == 2 * kGroupWarps, "an up/gate stage gives each warp of a group two rows");
static_assert(kDownStagesPerTile == kGroups && (2 * (kUgTileRows / kStageRows)) % kGroups == 0,
              "the stages of every tile reach every consumer group");
constexpr int kDownLag = 8;          // routed experts between an expert's up/gate and down tiles
constexpr int kMaxExpertsPerLane = 8; // warp routing: E <= 32 * 8

enum : int { D_EXIT = 0, D_ROUTER = 1, D_UG = 2, D_DOWN = 3, D_MARK = 4 };  // D_MARK: route now
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
    int sit;        // stage index within its tile
    int nst;        // stages in the tile (4 up/gate, 2 down: every group sees every tile)
    int aslot;
    int n_experts;  // shared + distinct routed experts (down tiles)
    int n_tok;
    int tok[kMaxT];
    int pair[kMaxT];
};

// A down tile's activation-record copy, posted by the producer and issued by
// the helper warp once the expert's h is complete.
struct ActReq {
    const uint8_t* src;
    uint32_t bytes;
    int cslot;
    int need;   // h tiles the expert must have finished
    int exit;
    int pad[2];
};

// A finished tile handed to an epilogue warp.
struct Task {
    int type;  // D_UG, D_DOWN or D_EXIT
    int n_tok, blk, cslot, n_experts;
    int pair[kMaxT];
};

using u64 = unsigned long long;

// Routing scratch, one half per token routed at the same time.  It lives in
// the x cache, which is free once Q8_0(x) is built.
struct alignas(16) RouteHalf {
    u64 cand[32 * kMaxExpertsPerLane];   // (key, complement of the index) of every expert
    float sc[32 * kMaxExpertsPerLane];   // scores s (unbiased)
    uint32_t part[kMaxExpertsPerLane][2];  // per warp of 32 experts: largest, second largest key
    int slot[kMaxExpertsPerLane];        // the expert of each slot
    uint32_t kept;                       // kept groups
    int nan;
};
// the rank scan reads cand as 16-byte pairs, in both halves
static_assert(sizeof(RouteHalf) % 16 == 0, "each half's cand array must stay 16-byte aligned");
struct RouteScratch {
    RouteHalf h[2];
    int pe[kMaxPairs];                   // expert of pair t K + k
    int bad[kMaxT];                      // token t had a NaN score
};

struct Smem {
    uint8_t* ring;
    uint8_t* act;
    uint16_t* xs;    // bf16 x; the routing scratch (RouteScratch) once Q8_0(x) is built
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
    uint64_t* route_bar;  // helper warp -> producer: routing of the batch is ready
    uint64_t* areq_full;  // [kMaxActSlots] producer -> helper: request posted
    uint64_t* areq_free;  // [kMaxActSlots] helper -> producer: request taken
    ActReq* areq;         // [kMaxActSlots]
    int* flag;
    uint32_t* tag;   // [1] this launch's score tag
    // routing of the batch, identical in every CTA
    float* rt_w;     // [kMaxPairs] gate weights by (token, slot)
    int* rt_pair_of; // [kMaxPairs] pair index by (token, slot)
    int* rt_uniq;    // [kMaxPairs] distinct experts ascending
    int* rt_off;     // [kMaxPairs + 1] pair offsets per distinct expert
    int* rt_ptok;    // [kMaxPairs] token of each pair
    int* rt_U;       // [1] number of distinct experts
};

__host__ __device__ inline size_t a16(size_t v) { return (v + 15) & ~size_t(15); }

struct Layout {
    size_t ring, act, xs, qx, bias, desc, task, areq, gbuf, red, bars, misc, total;
};

__host__ __device__ inline Layout layout_of(const FusedParams& p) {
    Layout L{};
    const size_t slot = static_cast<size_t>(p.stage_bytes) + kScaleBytes;
    const int nbH = p.H / 32;
    size_t o = 0;
    L.ring = o; o += a16(slot * p.nstage);
    L.act = o; o += a16(static_cast<size_t>(p.act_bytes) * kActSlots);
    L.xs = o; o += a16(std::max(static_cast<size_t>(p.T) * p.H * 2, sizeof(RouteScratch)));
    L.qx = o; o += a16(static_cast<size_t>(p.T) * nbH * 40);
    L.bias = o; o += a16(sizeof(float) * p.E);
    L.desc = o; o += a16(sizeof(Desc) * p.nstage);
    L.task = o; o += a16(sizeof(Task) * kTaskSlots);
    L.areq = o; o += a16(sizeof(ActReq) * kMaxActSlots);
    L.gbuf = o; o += a16(sizeof(float) * 2 * kTaskSlots * kMaxT * kUgTileRows);
    L.red = o; o += a16(sizeof(double) * kConsumerWarps * kMaxRouterRows * kMaxT);
    L.bars = o; o += a16(sizeof(uint64_t) * (2 * p.nstage + 4 * kMaxActSlots + 2 * kTaskSlots + 1));
    L.misc = o; o += a16(sizeof(int) * (4 + 4 + 5 * kMaxPairs + 2));
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
    s.areq = reinterpret_cast<ActReq*>(base + L.areq);
    s.gbuf = reinterpret_cast<float*>(base + L.gbuf);
    s.ubuf = s.gbuf + kTaskSlots * kMaxT * kUgTileRows;
    s.red = reinterpret_cast<double*>(base + L.red);
    s.full = reinterpret_cast<uint64_t*>(base + L.bars);
    s.empty = s.full + p.nstage;
    s.afull = s.empty + p.nstage;
    s.aempty = s.afull + kMaxActSlots;
    s.tfull = s.aempty + kMaxActSlots;
    s.tfree = s.tfull + kTaskSlots;
    s.route_bar = s.tfree + kTaskSlots;
    s.areq_full = s.route_bar + 1;
    s.areq_free = s.areq_full + kMaxActSlots;
    s.flag = reinterpret_cast<int*>(base + L.misc);
    s.tag = reinterpret_cast<uint32_t*>(s.flag + 4);
    s.rt_w = reinterpret_cast<float*>(s.tag + 4);
    s.rt_pair_of = reinterpret_cast<int*>(s.rt_w + kMaxPairs);
    s.rt_uniq = s.rt_pair_of + kMaxPairs;
    s.rt_off = s.rt_uniq + kMaxPairs;
    s.rt_ptok = s.rt_off + kMaxPairs + 1;
    s.rt_U = s.rt_ptok + kMaxPairs;
    return s;
}

// Activation-record slot i: the first kActSlots have their own region, the
// others sit in the x cache (neither x nor the routing scratch is read once
// the routing is done, and the first record copy follows it).
__device__ __forceinline__ uint8_t* act_slot(const FusedParams& p, const Smem& s, int i) {
    return i < kActSlots ? s.act + static_cast<size_t>(i) * p.act_bytes
                         : reinterpret_cast<uint8_t*>(s.xs) + static_cast<size_t>(i - kActSlots) * p.act_bytes;
}

// Poll limit of a wait: its default, or the workspace's test limit when that
// is set (nonzero) and smaller (see moe_workspace_set_wait_limit).
__device__ __forceinline__ long lim(const Smem& s, long dflt) {
    const long k = *reinterpret_cast<volatile const int*>(s.flag + 2);
    return k > 0 && k < dflt ? k : dflt;
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
__device__ __forceinline__ void group_sync(int g) { named_bar_sync(kBarConsumers + 1 + g, kGroupThreads); }

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

// Post-routing tile order: per routed expert r its up/gate tiles, followed by
// the down tiles of expert r - kDownLag; then the remaining routed experts'
// down tiles, with the shared expert's (whose h was finished first) placed
// before the last one to give that expert's h the most time.
struct Segments {
    int begin = 0, size = 0, kind = 0, u = 0;
    int r = 0, phase = 0, tail = -1, shared_left = 1;
    // Advances to the next non-empty segment; false when none is left.
    __device__ bool next(int U, int hs, int nug, int nd) {
        while (tail < 0) {
            if (phase == 0) {
                phase = 1;
                return set(0, r, nug);
            }
            phase = 0;
            const int rr = r++;
            if (r == U) tail = U > kDownLag ? U - kDownLag : 0;
            if (rr >= kDownLag) return set(1, rr - kDownLag, nd);
        }
        if (tail < U - 1) return set(1, tail++, nd);
        if (hs && shared_left) {
            shared_left = 0;
            return set(1, -1, nd);
        }
        if (tail == U - 1) return set(1, tail++, nd);
        size = 0;
        return false;
    }
    __device__ bool set(int k, int uu, int n) {
        kind = k;
        u = uu;
        size = n;
        return true;
    }
};

// ------------------------------------------------------------------ producer
template <int QT, bool G>
__device__ void producer(const FusedParams& p, const Smem& s) {
    const size_t slot_bytes = static_cast<size_t>(p.stage_bytes) + kScaleBytes;
    const uint64_t pol = l2_evict_first_policy();
    const int nrt = p.n_rt, nug = p.n_ugt, nd = p.n_dt, hs = p.has_shared;
    constexpr bool gs = G;  // grouped weight scales are read in place, not staged
    const int P = p.T * p.K;
    const size_t rb_ug = static_cast<size_t>(p.H) * QT / 8, rb_d = static_cast<size_t>(p.I) * QT / 8;
    int stage = 0, aslot = 0;
    uint32_t sphase = 0, aphase = 0;
    long n_issued = 0;
    int U = -1;
    bool ok = true;
    Segments seg;

    auto acquire_stage = [&]() -> bool {
        if (n_issued >= kMaxInflight) {  // at most kMaxInflight copies in flight
            const long older = n_issued - kMaxInflight;
            if (!mbar_wait(&s.full[older % p.nstage], static_cast<uint32_t>((older / p.nstage) & 1),
                           lim(s, kProducerWait)))
                return false;
        }
        return mbar_wait(&s.empty[stage], sphase ^ 1u, lim(s, kProducerWait));
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
        if (w_bytes == 0) {  // an empty stage (the short half of a ragged down tile)
            mbar_arrive(&s.full[stage]);
        } else {
            mbar_arrive_expect_tx(&s.full[stage], w_bytes + s_bytes);
            bulk_g2s_hint(dst, w_src, w_bytes, &s.full[stage], pol);
            if (s_bytes) bulk_g2s(dst + p.stage_bytes, s_src, s_bytes, &s.full[stage]);
        }
        advance();
        return true;
    };

    // One marker stage per consumer group, ahead of the first stage that is
    // not a router row: the consumers route when they reach it, so they never
    // wait for a stage that itself waits for the routing.
    bool marked = false;
    auto mark = [&]() -> bool {
        marked = true;
        for (int g = 0; g < kGroups; ++g) {
            if (!acquire_stage()) return false;
            s.desc[stage].type = D_MARK;
            mbar_arrive(&s.full[stage]);
            advance();
        }
        return true;
    };

    // The first ticket of CTA b is b: no round trip before the first copy,
    // and none of the workspace is touched, so it streams while the previous
    // grid in the stream finishes.  Later tickets come from the shared
    // counter, claimed once that grid has completed.
    int next = blockIdx.x;
    bool dep_done = false;
    while (ok) {
        if (next < 0) {
            grid_dependency_wait();
            dep_done = true;
            next = static_cast<int>(gridDim.x) + atomicAdd(&p.sync->ticket, 1);
        }
        const int cur = next;
        next = dep_done ? static_cast<int>(gridDim.x) + atomicAdd(&p.sync->ticket, 1) : -1;
        Desc d{};
        if (cur < nrt) {  // router rows e0 .. e0 + n - 1
            d.type = D_ROUTER;
            d.e = cur * p.rps;
            d.nrows = min(p.rps, p.E - d.e);
            ok = issue(d, p.w_router + static_cast<size_t>(d.e) * p.H, 4u * p.H * d.nrows, nullptr, 0);
            continue;
        }
        if (!marked && !mark()) {
            ok = false;
            break;
        }
        int t = cur - nrt;
        int kind, u, j;  // kind: 0 up/gate, 1 down; u = -1 shared
        if (hs && t < nug) {
            kind = 0; u = -1; j = t;
        } else {
            if (U < 0) {
                if (!mbar_wait(s.route_bar, 0, lim(s, kProducerWait))) {
                    ok = false;
                    break;
                }
                U = *reinterpret_cast<volatile int*>(s.rt_U);
            }
            t -= hs * nug;
            // walk the segment sequence forward to the segment holding ticket t
            while (t >= seg.begin + seg.size) {
                seg.begin += seg.size;
                if (!seg.next(U, hs, nug, nd)) break;
            }
            if (t >= seg.begin + seg.size) break;  // no work left
            kind = seg.kind; u = seg.u; j = t - seg.begin;
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
            d.nst = 2 * (kUgTileRows / kStageRows);
            for (int m = 0; m < 2 && ok; ++m) {
                const uint8_t* wm = m == 0 ? ex.w_gate : ex.w_up;
                const float* sm = m == 0 ? ex.s_gate : ex.s_up;
                for (int q = 0; q < kUgTileRows / kStageRows && ok; ++q) {
                    d.mat = m;
                    d.row0 = j * kUgTileRows + q * kStageRows;
                    d.first = (m == 0 && q == 0);
                    d.last = (m == 1 && q == kUgTileRows / kStageRows - 1);
                    d.sit = m * (kUgTileRows / kStageRows) + q;
                    const size_t r = static_cast<size_t>(d.e) * p.I + d.row0;
                    // per-row scales travel with the stage; grouped ones are read in place
                    ok = issue(d, wm + r * rb_ug, static_cast<uint32_t>(kStageRows * rb_ug), gs ? nullptr : sm + r,
                               gs ? 0u : kStageRows * 4);
                }
            }
        } else {  // down tile: rows j*dr .. j*dr+dr-1; the helper warp copies its
                  // activation records once the expert's h is complete, so the
                  // weight stages stream meanwhile
            d.type = D_DOWN;
            d.mat = 2;
            if (!mbar_wait(&s.areq_free[aslot], aphase ^ 1u, lim(s, kProducerWait))) {
                ok = false;
                break;
            }
            ActReq& rq = s.areq[aslot];
            rq.src = p.qrec + static_cast<size_t>(d.pair[0]) * p.rec_bytes;
            rq.bytes = static_cast<uint32_t>(d.n_tok) * p.rec_bytes;
            rq.cslot = d.cslot;
            rq.need = nug;
            rq.exit = 0;
            mbar_arrive(&s.areq_full[aslot]);
            d.aslot = aslot;
            // always two stages (one per consumer group), the rows split evenly
            const int c_beg = j * p.dr, n = min(p.H, c_beg + p.dr) - c_beg, h1 = (n + 1) / 2;
            d.nst = kDownStagesPerTile;
            for (int q = 0; q < kDownStagesPerTile && ok; ++q) {
                d.sit = q;
                d.row0 = c_beg + (q == 0 ? 0 : h1);
                d.nrows = q == 0 ? h1 : n - h1;
                d.first = q == 0;
                d.last = q == kDownStagesPerTile - 1;
                const size_t r = static_cast<size_t>(d.e) * p.H + d.row0;
                ok = issue(d, ex.w_down + r * rb_d, static_cast<uint32_t>(d.nrows * rb_d), gs ? nullptr : ex.s_down + r,
                           gs ? 0u : static_cast<uint32_t>(d.nrows * 4));
            }
            if (++aslot == p.nact) {
                aslot = 0;
                aphase ^= 1u;
            }
        }
    }
    if (!ok) record_status(p.status, MOE_EDEVICE_TIMEOUT);
    if (!marked) mark();  // the consumers route before they look for the end
    // tell the helper warp and the consumers to stop
    if (mbar_wait(&s.areq_free[aslot], aphase ^ 1u, lim(s, kProducerWait))) {
        s.areq[aslot].exit = 1;
        mbar_arrive(&s.areq_full[aslot]);
    }
    for (int g = 0; g < kGroups; ++g) {  // one end marker per consumer group
        if (!acquire_stage()) break;
        s.desc[stage].type = D_EXIT;
        mbar_arrive(&s.full[stage]);
        advance();
    }
    // drain: wait until every copy issued into this CTA's shared memory has landed
    for (int st = 0; st < p.nstage; ++st) {
        const long uses = n_issued / p.nstage + (st < n_issued % p.nstage ? 1 : 0);
        if (uses > 0) mbar_wait(&s.full[st], static_cast<uint32_t>((uses - 1) & 1), kProducerWait);
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

// ------------------------------------------------------------------ consumers
// Q8_0 of every token's x (threads idx of nth; TPB threads per 32-block),
// stored permuted for dp4a against qtype QT.  Same arithmetic as q8_0_lane.
// Each thread's permuted words hold only its own elements, so no exchange
// through shared memory is needed: thread `part` of a block owns elements
// [part EPT, part EPT + EPT) and words [part WPT, part WPT + WPT).
template <int QT>
__device__ __forceinline__ void quantize_x(const FusedParams& p, const Smem& s, int idx, int nth) {
    constexpr int TPB = QT == 2 ? 2 : 4, EPT = 32 / TPB, WPT = 8 / TPB;
    const int nbH = p.H / 32, ntask = p.T * nbH * TPB;
    for (int base = 0; base < ntask; base += nth) {
        const int task = base + idx;
        const bool active = task < ntask;
        const int blk = task / TPB, part = task % TPB;
        float v[EPT];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < EPT; ++i) v[i] = 0.0f;
        if (active) {
            const int t = blk / nbH, b = blk % nbH;
            const uint4* src = reinterpret_cast<const uint4*>(s.xs + static_cast<size_t>(t) * p.H + 32 * b + EPT * part);
#pragma unroll
            for (int c = 0; c < EPT / 8; ++c) {
                const uint4 u = src[c];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    v[8 * c + 2 * i] = bf16_bits_to_f32(static_cast<uint16_t>(w[i]));
                    v[8 * c + 2 * i + 1] = bf16_bits_to_f32(static_cast<uint16_t>(w[i] >> 16));
                }
            }
#pragma unroll
            for (int i = 0; i < EPT; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
#pragma unroll
        for (int o = 1; o < TPB; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float d = __fdiv_rn(amax, 127.0f);
        // q = round(v / d) with the correctly rounded quotient.  t = v * RN(1/d)
        // is within 2.5e-5 of RN(v / d) while |v / d| <= 127, so where t lies
        // farther than 1e-4 from a half-integer both round to the same
        // integer; elsewhere (and when 1/d overflows) the division decides.
        const float r = d != 0.0f ? __frcp_rn(d) : 0.0f;
        int q[EPT];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < EPT; ++i) {
            const float t = __fmul_rn(v[i], r), a = fabsf(t);
            float qf;
            if (a <= 128.0f && fabsf(a - floorf(a) - 0.5f) >= 1e-4f) {
                qf = roundf(t);
            } else {
                qf = roundf(__fdiv_rn(v[i], d));
            }
            const int qi = d != 0.0f ? static_cast<int>(fminf(fmaxf(qf, -127.0f), 127.0f)) : 0;
            q[i] = qi;
            sum += qi;
        }
#pragma unroll
        for (int o = 1; o < TPB; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (active) {
            uint32_t o[WPT];
#pragma unroll
            for (int k = 0; k < WPT; ++k) {
                uint32_t word = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) word |= (static_cast<uint32_t>(q[perm_src<QT>(k, i)]) & 0xFFu) << (8 * i);
                o[k] = word;
            }
            if constexpr (TPB == 4) {
                uint32_t* dst = reinterpret_cast<uint32_t*>(part < 2 ? s.q0 + blk : s.q1 + blk) + 2 * (part & 1);
                *reinterpret_cast<uint2*>(dst) = make_uint2(o[0], o[1]);
            } else {
                (part == 0 ? s.q0 : s.q1)[blk] = make_uint4(o[0], o[1], o[2], o[3]);
            }
            if (part == 0) {
                s.qd[blk] = d;
                s.qs[blk] = sum;
            }
        }
    }
}

// x and the bias into shared memory, and this launch's tag (the previous
// launch's number + 1), whose load overlaps those of x.
__device__ void consumer_init(const FusedParams& p, const Smem& s) {
    const int tid = threadIdx.x;
    const int ep = tid == 0 ? ld_relaxed_gpu(reinterpret_cast<const int*>(p.epoch)) : 0;
    const int n16 = p.T * p.H / 8;
    for (int i = tid; i < n16; i += kConsumers)
        reinterpret_cast<uint4*>(s.xs)[i] = reinterpret_cast<const uint4*>(p.x)[i];
    for (int e = tid; e < p.E; e += kConsumers) s.bias[e] = __ldg(p.bias + e);
    if (tid == 0) *s.tag = static_cast<uint32_t>(ep) + 1u;
    consumers_sync();
}

// One router stage: logits of rows e0 .. e0 + nrows - 1 for every token.
template <int NT>
__device__ void consume_router(const FusedParams& p, const Smem& s, int e0, int nrows, const uint8_t* sbuf,
                               int g) {
    const int gtid = threadIdx.x % kGroupThreads, gwarp = gtid >> 5, lane = gtid & 31;
    const int h4 = p.H / 4;
    double* red = s.red + g * (kGroupWarps * kMaxRouterRows * kMaxT);
    double acc[kMaxRouterRows][NT];
#pragma unroll
    for (int q = 0; q < kMaxRouterRows; ++q)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[q][t] = 0.0;
    for (int j = gtid; j < h4; j += kGroupThreads) {
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
                if (lane == 0) red[(gwarp * kMaxRouterRows + q) * kMaxT + t] = v;
            }
        }
    group_sync(g);
    if (gtid < nrows * p.T) {
        // logit rounded once to fp32, sigmoid in fp64 rounded once; published
        // with this launch's tag in the same 64-bit word
        const int q = gtid / p.T, t = gtid % p.T;
        double sum = 0.0;
        for (int w = 0; w < kGroupWarps; ++w) sum += red[(w * kMaxRouterRows + q) * kMaxT + t];
        const double l = static_cast<double>(__double2float_rn(sum));
        const float sc = __double2float_rn(1.0 / (1.0 + exp(-l)));
        st_relaxed_gpu_u64(p.scores + static_cast<size_t>(t) * p.E + e0 + q,
                           (static_cast<unsigned long long>(*s.tag) << 32) | __float_as_uint(sc));
    }
    group_sync(g);  // the reduction buffer is reused by this group's next router stage
}

// Order-preserving map of fp32 values to unsigned keys (+0 and -0 equal; the
// key 0 is below every value and marks an excluded expert).
__device__ __forceinline__ uint32_t order_key(float v) {
    uint32_t b = __float_as_uint(v);
    if ((b << 1) == 0) b = 0;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ uint32_t max_u32(uint32_t a, uint32_t b) { return a > b ? a : b; }
__device__ __forceinline__ uint32_t min_u32(uint32_t a, uint32_t b) { return a < b ? a : b; }

// Merges the (largest, second largest) pair (b1, b2) into (a1, a2); a maximum
// held twice counts twice.
__device__ __forceinline__ void top2_merge(uint32_t& a1, uint32_t& a2, uint32_t b1, uint32_t b2) {
    a2 = max_u32(min_u32(a1, b1), max_u32(a2, b2));
    a1 = max_u32(a1, b1);
}

// noaux_tc routing (DeepSeek-V3 routing, as [HN] "구현된 주요 기능" names it)
// and the batch union, by all consumer threads: each half of them (256
// threads, one expert each) routes one token, two tokens at a time.
//   b = s + bias (fp32); group score = sum of the group's two largest b (a
//   maximum held twice counts twice); the TG best groups kept, ties to the
//   lower group; the top K experts of the kept groups by b fill the slots in
//   order, ties to the lower index; gate weight of slot k = s_k / (s_0 + ...
//   + s_{K-1}) * rsf with the sum taken in slot order.
// The routed weight stream cannot start before routing ends, so the work is
// spread for a short chain per thread: each warp (32 experts) reduces its
// (largest, second) pair by a butterfly, one warp sums and ranks the groups,
// and every candidate of a kept group counts the kept candidates that order
// before it (key, then lower index: one compare of 64-bit words).  The union
// lists the pairs by (expert, token).  Thread 0 then releases the producer
// through route_bar.
// A token with a NaN score is still given K valid experts internally (the
// ticket sequence needs them) but reports index -1 and weight 0 to the caller
// and records MOE_EDEVICE_INDEX; its output row is unspecified.
__device__ void route_block(const FusedParams& p, const Smem& s) {
    const int tid = threadIdx.x, half = tid >> 8, e = tid & 255, lane = tid & 31, hw = e >> 5;
    const int T = p.T, K = p.K, E = p.E, G = p.G, TG = p.TG, gsz = E / G, wpg = gsz >> 5;
    RouteScratch* rs = reinterpret_cast<RouteScratch*>(s.xs);
    RouteHalf& h = rs->h[half];
    const uint32_t tag = *s.tag;
    bool ok = true;
    for (int t0 = 0; t0 < T; t0 += 2) {
        const int t = t0 + half;
        const bool tok = t < T, live = tok && e < E;
        // this token's score of expert e, once it carries this launch's tag
        float sc = 0.0f;
        if (live) {
            for (long it = 0;; ++it) {
                const u64 v = ld_relaxed_gpu_u64(p.scores + static_cast<size_t>(t) * E + e);
                if (static_cast<uint32_t>(v >> 32) == tag) {
                    sc = __uint_as_float(static_cast<uint32_t>(v));
                    break;
                }
                if (it >= lim(s, kConsumerWait)) {
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
        }
        const float b = live ? __fadd_rn(sc, s.bias[e]) : 0.0f;
        const uint32_t key = live ? order_key(b) : 0u;
        h.sc[e] = sc;
        h.cand[e] = (static_cast<u64>(key) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(e));
        uint32_t t1 = key, t2 = 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            top2_merge(t1, t2, __shfl_xor_sync(0xffffffffu, t1, o), __shfl_xor_sync(0xffffffffu, t2, o));
        const bool nan = __any_sync(0xffffffffu, live && b != b);
        if (lane == 0) {
            h.part[hw][0] = t1;
            h.part[hw][1] = t2;
            if (hw == 0) h.nan = 0;
        }
        consumers_sync();
        if (nan && lane == 0) h.nan = 1;
        // group scores and the kept groups, by the first warp of the half
        if (hw == 0 && tok) {
            float gs = 0.0f;
            if (lane < G) {
                uint32_t a1 = 0u, a2 = 0u;
                for (int w = lane * wpg; w < lane * wpg + wpg; ++w) top2_merge(a1, a2, h.part[w][0], h.part[w][1]);
                gs = __fadd_rn(key_value(a1), key_value(a2));
            }
            int r = 0;
            for (int g = 0; g < G; ++g) {
                const float o = __shfl_sync(0xffffffffu, gs, g);
                r += (o > gs) || (o == gs && g < lane);
            }
            const uint32_t kept = __ballot_sync(0xffffffffu, lane < G && r < TG);
            if (lane == 0) h.kept = kept;
        }
        consumers_sync();
        // rank of each kept candidate among the kept candidates
        const uint32_t kept = h.kept;
        if (live && ((kept >> (e / gsz)) & 1u)) {
            const u64 mine = h.cand[e];
            int rank = 0;
            for (uint32_t km = kept; km; km &= km - 1) {
                const ulonglong2* c2 = reinterpret_cast<const ulonglong2*>(h.cand + (__ffs(km) - 1) * gsz);
                // 32 experts a warp: the group's loads all issued before the compares
                for (int i0 = 0; i0 < gsz / 2; i0 += 16) {
                    ulonglong2 v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = c2[i0 + i];
#pragma unroll
                    for (int i = 0; i < 16; ++i) rank += (v[i].x > mine) + (v[i].y > mine);
                }
            }
            if (rank < K) h.slot[rank] = e;
        }
        consumers_sync();
        // slot k of token t: expert and gate weight; with adaptive top-p the
        // kept slots (every thread of the first K finds the same set) move to
        // the front in slot order and the rest become empty (-1, weight 0)
        if (tok && e < K) {
            int ex[kMaxExpertsPerLane];
            float sv[kMaxExpertsPerLane];
#pragma unroll
            for (int k = 0; k < kMaxExpertsPerLane; ++k) {
                ex[k] = k < K ? h.slot[k] : 0;
                sv[k] = k < K ? h.sc[ex[k]] : 0.0f;
            }
            uint32_t keep = (1u << K) - 1u;
            if (p.top_p > 0.0f && p.top_p < 1.0f) {
                double S = 0.0;
#pragma unroll
                for (int k = 0; k < kMaxExpertsPerLane; ++k)
                    if (k < K) S += static_cast<double>(sv[k]);
                const double thr = static_cast<double>(p.top_p) * S;
                double c = 0.0;
                keep = 0u;
                for (int m = 0; m < K; ++m) {
                    int j = -1;  // the largest remaining score, the earlier slot on ties
                    float best = 0.0f;
#pragma unroll
                    for (int k = 0; k < kMaxExpertsPerLane; ++k)
                        if (k < K && !((keep >> k) & 1u) && (j < 0 || sv[k] > best)) {
                            j = k;
                            best = sv[k];
                        }
                    keep |= 1u << j;
                    c += static_cast<double>(best);
                    if (c >= thr) break;
                }
            }
            float den = 0.0f, mys = 0.0f;
#pragma unroll
            for (int k = 0; k < kMaxExpertsPerLane; ++k) {
                if (k < K && ((keep >> k) & 1u)) {
                    den = __fadd_rn(den, sv[k]);
                    if (k == e) mys = sv[k];
                }
            }
            const int nkept = __popc(keep);
            if ((keep >> e) & 1u) {
                const int pos = __popc(keep & ((1u << e) - 1u));
                rs->pe[t * K + pos] = h.slot[e];
                s.rt_w[t * K + pos] = __fmul_rn(__fdiv_rn(mys, den), p.rsf);
            }
            if (e >= nkept) {
                rs->pe[t * K + e] = -1;
                s.rt_w[t * K + e] = 0.0f;
            }
        }
        if (tok && e == 0) rs->bad[t] = h.nan;
        consumers_sync();
    }
    if (!ok) record_status(p.status, MOE_EDEVICE_TIMEOUT);
    if (tid >= 32) return;
    // the batch union, by warp 0
    const unsigned all = 0xffffffffu;
    uint32_t bad_tokens = 0;  // bit t: token t had a NaN score
    for (int t = 0; t < T; ++t) bad_tokens |= rs->bad[t] ? 1u << t : 0u;
    if (bad_tokens && lane == 0) record_status(p.status, MOE_EDEVICE_INDEX);
    const int n = T * K;  // <= 32
    const int pe_raw = lane < n ? rs->pe[lane] : -1;
    const bool act = pe_raw >= 0;  // a pair (empty slots have none)
    const int pe = act ? pe_raw : 0;
    const float pw = lane < n ? s.rt_w[lane] : 0.0f;
    if (lane < n && !act) s.rt_pair_of[lane] = -1;
    if (T == 1) {
        // one token: distinct experts, the kept ones first; a pair's position is its expert's rank
        const uint32_t valid = __ballot_sync(all, act);
        int pos = 0;
#pragma unroll
        for (int k = 0; k < kMaxExpertsPerLane; ++k) pos += k < K && ((valid >> k) & 1u) && rs->pe[k] < pe;
        if (act) {
            s.rt_ptok[pos] = 0;
            s.rt_pair_of[lane] = pos;
            s.rt_uniq[pos] = pe;
            s.rt_off[pos] = pos;
        }
        if (lane == 0) {
            *s.rt_U = __popc(valid);
            s.rt_off[__popc(valid)] = __popc(valid);
        }
    } else {
        // pair position = number of pairs with a smaller (expert, token)
        const int key = act ? (pe << 5) | lane : 0x7fffffff;
        const uint32_t same = __match_any_sync(all, act ? pe : -1 - lane);
        const bool first = act && (__ffs(same) - 1 == lane);
        const uint32_t firsts = __ballot_sync(all, first);
        const uint32_t valid = __ballot_sync(all, act);
        int pos = 0, urank = 0;
        for (int j = 0; j < n; ++j) {
            const int kj = __shfl_sync(all, key, j);
            pos += kj < key;
            urank += ((firsts >> j) & 1u) && (kj >> 5) < pe;
        }
        if (act) {
            s.rt_ptok[pos] = lane / K;
            s.rt_pair_of[lane] = pos;
            if (first) {
                s.rt_uniq[urank] = pe;
                s.rt_off[urank] = pos;
            }
        }
        if (lane == 0) {
            *s.rt_U = __popc(firsts);
            s.rt_off[__popc(firsts)] = __popc(valid);
        }
    }
    if (lane < n && blockIdx.x == 0) {  // the routing the caller can see, written once
        const bool bad = (bad_tokens >> (lane / K)) & 1u;
        p.idx[lane] = bad || !act ? -1 : pe;
        p.w[lane] = bad || !act ? 0.0f : pw;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(s.route_bar);
}

// Activations of one token for the blocks a lane owns (b = lane + 32 j), in registers.
template <int NC>
struct ActRegs {
    uint4 a0[NC];
    uint4 a1[NC];
};

// Grouped weight scales ([MO] "int4 양자화 (Quantization)의 품질 비용") of row
// `rs` of a stage, or null with per-row scales (those travel with the stage).
// Block b's factor is then d_b * s[b / gpb] (one rounding) and the row has no
// separate scale.
template <bool G>
__device__ __forceinline__ const float* grouped_row(const FusedParams& p, const Desc& d, int rs) {
    if constexpr (!G) return nullptr;
    const int gs = p.routed.group_size;
    const moe_experts& ex = d.cslot == 0 ? p.shared : p.routed;  // slot 0: the shared expert
    const size_t row = static_cast<size_t>(d.row0 + rs);
    if (d.mat == 2) return ex.s_down + (static_cast<size_t>(d.e) * p.H + row) * (p.I / gs);
    return (d.mat == 0 ? ex.s_gate : ex.s_up) + (static_cast<size_t>(d.e) * p.I + row) * (p.H / gs);
}

__device__ __forceinline__ float block_factor(float da, const float* sg, int b, int gpb) {
    return sg ? __fmul_rn(da, __ldg(sg + b / gpb)) : da;
}

// up/gate stage, NT = 1: the token's Q8_0(x) words are in registers.
template <int QT, bool G>
__device__ __forceinline__ void consume_ug_reg(const FusedParams& p, const Smem& s, const Desc& d, float* dst,
                                               const uint8_t* sbuf, const ActRegs<kRegChunksUg>& ar, int gw) {
    const int lane = threadIdx.x & 31;
    const int row0 = d.row0, gpb = p.routed.group_size / 32;
    const float* sg0 = grouped_row<G>(p, d, gw);
    const float* sg1 = grouped_row<G>(p, d, gw + kGroupWarps);
    const int nbH = p.H / 32;
    const size_t rb = static_cast<size_t>(p.H) * QT / 8;
    const uint8_t* w0 = sbuf + gw * rb;                  // rows gw and gw + kGroupWarps of the stage
    const uint8_t* w1 = sbuf + (gw + kGroupWarps) * rb;
    float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
    for (int j = 0; j < kRegChunksUg; ++j) {
        const int b = lane + 32 * j;
        if (b < nbH) {
            const WBlock<QT> wb0 = load_wblock_smem<QT>(w0, b);
            const WBlock<QT> wb1 = load_wblock_smem<QT>(w1, b);
            const int qs = s.qs[b];
            const float qd = s.qd[b];
            acc0 = fmaf(static_cast<float>(block_dot<QT>(wb0, ar.a0[j], ar.a1[j], qs)), block_factor(qd, sg0, b, gpb),
                        acc0);
            acc1 = fmaf(static_cast<float>(block_dot<QT>(wb1, ar.a0[j], ar.a1[j], qs)), block_factor(qd, sg1, b, gpb),
                        acc1);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        acc0 += __shfl_xor_sync(0xffffffffu, acc0, o);
        acc1 += __shfl_xor_sync(0xffffffffu, acc1, o);
    }
    if (lane == 0) {
        const float* sc = reinterpret_cast<const float*>(sbuf + p.stage_bytes);
        dst[row0 % kUgTileRows + gw] = sg0 ? acc0 : __fmul_rn(acc0, sc[gw]);
        dst[row0 % kUgTileRows + gw + kGroupWarps] = sg1 ? acc1 : __fmul_rn(acc1, sc[gw + kGroupWarps]);
    }
}

// up/gate stage, NT > 1: activations read from the shared-memory cache.
template <int QT, int NT, bool G>
__device__ __forceinline__ void consume_ug_smem(const FusedParams& p, const Smem& s, const Desc& d, float* dst,
                                                const uint8_t* sbuf, int gw) {
    const int lane = threadIdx.x & 31;
    const int nbH = p.H / 32;
    const size_t rb = static_cast<size_t>(p.H) * QT / 8;
    const int n_tok = d.n_tok;
    int tok[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) tok[t] = t < n_tok ? d.tok[t] : 0;
    const float* sc = reinterpret_cast<const float*>(sbuf + p.stage_bytes);
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {  // rows gw and gw + kGroupWarps of the stage
        const int rs = gw + h * kGroupWarps;
        const uint8_t* wrow = sbuf + rs * rb;
        const float* sg = grouped_row<G>(p, d, rs);
        const int gpb = p.routed.group_size / 32;
        float acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.0f;
#pragma unroll 2
        for (int b = lane; b < nbH; b += 32) {
            const WBlock<QT> wb = load_wblock_smem<QT>(wrow, b);
            const float gsc = sg ? __ldg(sg + b / gpb) : 1.0f;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (t < n_tok) {
                    const int q = tok[t] * nbH + b;
                    const int isum = block_dot<QT>(wb, s.q0[q], s.q1[q], s.qs[q]);
                    acc[t] = fmaf(static_cast<float>(isum), sg ? __fmul_rn(s.qd[q], gsc) : s.qd[q], acc[t]);
                }
            }
        }
        const int r = d.row0 % kUgTileRows + rs;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < n_tok) {
                const float v = warp_sum_f32(acc[t]);
                if (lane == 0) dst[t * kUgTileRows + r] = sg ? v : __fmul_rn(v, sc[rs]);
            }
        }
    }
}

// down stage, NT = 1: the pair's Q8_0(h) words are in registers (loaded per tile).
template <int QT, bool G>
__device__ __forceinline__ void consume_down_reg(const FusedParams& p, const Desc& d, const uint8_t* sbuf,
                                                 const ActRegs<kRegChunksDown>& ar, const float* ad,
                                                 const int32_t* as, int gw) {
    const int lane = threadIdx.x & 31;
    const int row0 = d.row0, nrows = d.nrows, pair = d.pair[0], gpb = p.routed.group_size / 32;
    const int nbI = p.I / 32;
    const size_t rb = static_cast<size_t>(p.I) * QT / 8;
    const float* sc = reinterpret_cast<const float*>(sbuf + p.stage_bytes);
    float acc[kMaxDownRowsPerWarp];
#pragma unroll
    for (int k = 0; k < kMaxDownRowsPerWarp; ++k) {
        acc[k] = 0.0f;
        const int r = gw + kGroupWarps * k;
        if (r < nrows) {
            const uint8_t* wrow = sbuf + r * rb;
            const float* sg = grouped_row<G>(p, d, r);
#pragma unroll
            for (int j = 0; j < kRegChunksDown; ++j) {
                const int b = lane + 32 * j;
                if (b < nbI) {
                    const WBlock<QT> wb = load_wblock_smem<QT>(wrow, b);
                    const int isum = block_dot<QT>(wb, ar.a0[j], ar.a1[j], as[b]);
                    acc[k] = fmaf(static_cast<float>(isum), block_factor(ad[b], sg, b, gpb), acc[k]);
                }
            }
        }
    }
#pragma unroll
    for (int k = 0; k < kMaxDownRowsPerWarp; ++k) {
        const int r = gw + kGroupWarps * k;
        if (r < nrows) {
            const float v = warp_sum_f32(acc[k]);
            if (lane == 0) p.y[static_cast<size_t>(pair) * p.H + row0 + r] = G ? v : __fmul_rn(v, sc[r]);
        }
    }
}

// down stage, NT > 1: activations read from the tile's shared-memory slot.
template <int QT, int NT, bool G>
__device__ __forceinline__ void consume_down_smem(const FusedParams& p, const Smem& s, const Desc& d,
                                                  const uint8_t* sbuf, int gw) {
    const int lane = threadIdx.x & 31;
    const int nbI = p.I / 32;
    const size_t rb = static_cast<size_t>(p.I) * QT / 8;
    const uint8_t* act = act_slot(p, s, d.aslot);
    const float* sc = reinterpret_cast<const float*>(sbuf + p.stage_bytes);
    const int n_tok = d.n_tok, nrows = d.nrows, row0 = d.row0;
    int pair[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) pair[t] = d.pair[t];
    const int gpb = p.routed.group_size / 32;
    for (int r = gw; r < nrows; r += kGroupWarps) {
        const uint8_t* wrow = sbuf + r * rb;
        const float* sg = grouped_row<G>(p, d, r);
        float acc[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[t] = 0.0f;
#pragma unroll 2
        for (int b = lane; b < nbI; b += 32) {
            const WBlock<QT> wb = load_wblock_smem<QT>(wrow, b);
            const float gsc = sg ? __ldg(sg + b / gpb) : 1.0f;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (t < n_tok) {
                    const uint8_t* rec = act + static_cast<size_t>(t) * p.rec_bytes;
                    const uint4 a0 = reinterpret_cast<const uint4*>(rec)[b];
                    const uint4 a1 = reinterpret_cast<const uint4*>(rec + p.I / 2)[b];
                    const float da = reinterpret_cast<const float*>(rec + p.I)[b];
                    const int as = reinterpret_cast<const int32_t*>(rec + p.I + nbI * 4)[b];
                    acc[t] = fmaf(static_cast<float>(block_dot<QT>(wb, a0, a1, as)), sg ? __fmul_rn(da, gsc) : da, acc[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (t < n_tok) {
                const float v = warp_sum_f32(acc[t]);
                if (lane == 0) p.y[static_cast<size_t>(pair[t]) * p.H + row0 + r] = sg ? v : __fmul_rn(v, sc[r]);
            }
        }
    }
}

// Hands a finished tile (or the end) to epilogue warp tb through task slot tb.
// Every consumer warp arrives once per tile; `writer` (one warp) fills the task first.
__device__ __forceinline__ void push_task(const Smem& s, int tb, const Desc* d, int type, bool writer) {
    const int lane = threadIdx.x & 31;
    if (writer && lane == 0) {
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

template <int QT, int NT, bool G>
__device__ void consumer(const FusedParams& p, const Smem& s) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = warp / kGroupWarps, gw = warp % kGroupWarps;
    const size_t slot_bytes = static_cast<size_t>(p.stage_bytes) + kScaleBytes;
    consumer_init(p, s);
    // group g takes ring stages g, g + kGroups, g + 2 kGroups, ...
    int stage = g, aslot = 0, tb = 0;
    uint32_t phase = 0, aphase = 0;
    uint32_t tph[kTaskSlots] = {0, 0};
    // Waits for the current stage; returns its type (D_EXIT on timeout).
    auto next_type = [&]() -> int {
        if (!mbar_wait(&s.full[stage], phase, lim(s, kConsumerWait))) {
            record_status(p.status, MOE_EDEVICE_TIMEOUT);
            return D_EXIT;
        }
        return s.desc[stage].type;
    };
    auto release = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty[stage]);
        stage += kGroups;
        if (stage >= p.nstage) {
            stage -= p.nstage;
            phase ^= 1u;
        }
    };
    // Waits until epilogue warp tb has finished with task slot tb.
    auto task_slot_free = [&]() -> bool {
        if (!mbar_wait(&s.tfree[tb], tph[tb] ^ 1u, lim(s, kConsumerWait))) {
            record_status(p.status, MOE_EDEVICE_TIMEOUT);
            return false;
        }
        return true;
    };
    auto next_task = [&]() {
        tph[tb] ^= 1u;
        tb ^= 1;
    };
    // phase A: the router rows up to the route marker, Q8_0 of x, then the
    // routing.  A CTA's router rows start at its stage 0 (group 0); for one
    // token, when the last group's first stage holds none, that group
    // quantises x meanwhile.
    int type = next_type();
    if (p.T == 1 && g == kGroups - 1 && type != D_ROUTER) {
        quantize_x<QT>(p, s, tid % kGroupThreads, kGroupThreads);
        if (tid % kGroupThreads == 0) s.flag[1] = 1;
    }
    while (type == D_ROUTER) {
        const int e0 = s.desc[stage].e, nrows = s.desc[stage].nrows;
        consume_router<NT>(p, s, e0, nrows, s.ring + stage * slot_bytes, g);
        release();
        type = next_type();
    }
    const bool marker = type == D_MARK;
    if (marker) release();
    consumers_sync();
    if (s.flag[1] == 0) {  // the last group had router rows: everyone quantises x now
        quantize_x<QT>(p, s, tid, kConsumers);
        consumers_sync();
    }
    route_block(p, s);  // the x cache holds the routing scratch from here on
    if (marker) type = next_type();
    // phases B and C: runs of up/gate tiles and of down tiles.  A tile's
    // stages alternate between the groups, so every warp sees every tile:
    // its first stage of a tile (sit < kGroups) claims the task slot or the
    // activation records, its last one (sit + kGroups >= nst) hands the tile on.
    bool ok = true;
    while (ok && (type == D_UG || type == D_DOWN)) {
        if (type == D_UG) {
            // NT = 1: the token's Q8_0 x lives in registers for the run
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
                if (d.sit < kGroups && !task_slot_free()) {
                    ok = false;
                    break;
                }
                float* dst = (d.mat == 0 ? s.gbuf : s.ubuf) + tb * kMaxT * kUgTileRows;
                if constexpr (NT == 1) {
                    consume_ug_reg<QT, G>(p, s, d, dst, sbuf, ar, gw);
                } else {
                    consume_ug_smem<QT, NT, G>(p, s, d, dst, sbuf, gw);
                }
                if (d.sit + kGroups >= d.nst) {
                    push_task(s, tb, &d, D_UG, d.sit == d.nst - 1 && gw == 0);
                    next_task();
                }
                release();
                type = next_type();
            }
        } else {
            ActRegs<kRegChunksDown> ar;
            const float* ad = nullptr;
            const int32_t* as = nullptr;
            while (type == D_DOWN) {
                const Desc& d = s.desc[stage];
                const uint8_t* sbuf = s.ring + stage * slot_bytes;
                if (d.sit < kGroups) {
                    if (!mbar_wait(&s.afull[aslot], aphase, lim(s, kConsumerWait))) {
                        record_status(p.status, MOE_EDEVICE_TIMEOUT);
                        ok = false;
                        break;
                    }
                    if constexpr (NT == 1) {
                        const uint8_t* rec = act_slot(p, s, aslot);
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
                    consume_down_reg<QT, G>(p, d, sbuf, ar, ad, as, gw);
                } else {
                    consume_down_smem<QT, NT, G>(p, s, d, sbuf, gw);
                }
                if (d.sit + kGroups >= d.nst) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.aempty[aslot]);
                    if (++aslot == p.nact) {
                        aslot = 0;
                        aphase ^= 1u;
                    }
                    if (!task_slot_free()) {
                        ok = false;
                        break;
                    }
                    push_task(s, tb, &d, D_DOWN, d.sit == d.nst - 1 && gw == 0);
                    next_task();
                }
                release();
                type = next_type();
            }
        }
    }
    // hand the end to both epilogue warps
    for (int i = 0; i < kTaskSlots; ++i) {
        if (!task_slot_free()) break;
        push_task(s, tb, nullptr, D_EXIT, warp == 0);
        next_task();
    }
}

// ------------------------------------------------------------------ helper warp
// Lane 0 serves the producer's down-tile requests in order: waits until the
// slot's previous records are consumed and the expert's h tiles are all
// complete, then bulk-copies the records.
template <int QT>
__device__ __forceinline__ void helper_warp(const FusedParams& p, const Smem& s) {
    if ((threadIdx.x & 31) != 0) return;
    // the workspace's test limit on bounded waits, off every other warp's start-up path
    // (written by the host before the launch; waits use their defaults until it lands)
    atomicExch(&s.flag[2], ld_relaxed_gpu(&p.sync->wait_limit));
    long n_act = 0;
    int slot = 0;
    uint32_t ph = 0;
    bool ok = true;
    while (true) {
        if (!mbar_wait(&s.areq_full[slot], ph, lim(s, kProducerWait))) {
            ok = false;
            break;
        }
        const ActReq rq = s.areq[slot];
        if (rq.exit) break;
        if (!mbar_wait(&s.aempty[slot], ph ^ 1u, lim(s, kProducerWait)) ||
            !wait_counter_geq(p.ug_done + rq.cslot, rq.need, lim(s, kProducerWait))) {
            ok = false;
            break;
        }
        fence_proxy_async_global();
        mbar_arrive_expect_tx(&s.afull[slot], rq.bytes);
        bulk_g2s(act_slot(p, s, slot), rq.src, rq.bytes, &s.afull[slot]);
        ++n_act;
        mbar_arrive(&s.areq_free[slot]);
        if (++slot == p.nact) {
            slot = 0;
            ph ^= 1u;
        }
    }
    if (!ok) record_status(p.status, MOE_EDEVICE_TIMEOUT);
    // drain: every record copy issued into this CTA's shared memory has landed
    for (int a = 0; a < p.nact; ++a) {
        const long uses = n_act / p.nact + (a < n_act % p.nact ? 1 : 0);
        if (uses > 0) mbar_wait(&s.afull[a], static_cast<uint32_t>((uses - 1) & 1), kProducerWait);
    }
}

// ------------------------------------------------------------------ epilogue warp
template <int QT>
__device__ void epilogue_warp(const FusedParams& p, const Smem& s, int tb) {
    // epilogue warp tb serves task slot tb
    const int lane = threadIdx.x & 31;
    const int nbI = p.I / 32;
    const int P = p.T * p.K;
    uint32_t eph = 0;
    while (true) {
        if (!mbar_wait(&s.tfull[tb], eph, lim(s, kEpilogueWait))) {
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
            // each lane's record words before the bulk copies (async proxy) that
            // read them in other CTAs; the warp's writes before lane 0's release;
            // nothing waits for the count here, so the add does not return
            fence_proxy_async_global();
            __syncwarp();
            if (lane == 0) red_release_add_gpu(p.ug_done + tk.cslot, 1);
        } else {
            // count the down tile for its row block; the CTA completing a block combines it
            const int blk = tk.blk, n_experts = tk.n_experts;
            int last = 0;
            // release: the consumers' y rows of this tile (ordered before this
            // warp by the task barrier); acquire: every other tile's rows, for
            // the CTA that completes the block
            if (lane == 0) last = atom_add_acq_rel_gpu(p.rb_done + blk, 1) == n_experts - 1;
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last) {
                // every load of an element first (they are L2 round trips, at
                // the end of the launch), then the sum in slot order
                const int c0 = blk * p.dr, nr = min(p.dr, p.H - c0), K = p.K;
                for (int t = 0; t < p.T; ++t) {
                    // the token's slots, once: an empty slot (weight 0, no pair) adds nothing
                    float wk[kMaxExpertsPerLane];
                    const float* yk[kMaxExpertsPerLane];
#pragma unroll
                    for (int k = 0; k < kMaxExpertsPerLane; ++k) {
                        wk[k] = k < K ? s.rt_w[t * K + k] : 0.0f;
                        yk[k] = wk[k] != 0.0f ? p.y + static_cast<size_t>(s.rt_pair_of[t * K + k]) * p.H : nullptr;
                    }
                    for (int i = lane; i < nr; i += 32) {
                        const int c = c0 + i;
                        float yv[kMaxExpertsPerLane];
#pragma unroll
                        for (int k = 0; k < kMaxExpertsPerLane; ++k) yv[k] = yk[k] ? __ldcg(yk[k] + c) : 0.0f;
                        float o = p.has_shared ? __ldcg(p.y + static_cast<size_t>(P + t) * p.H + c) : 0.0f;
#pragma unroll
                        for (int k = 0; k < kMaxExpertsPerLane; ++k)
                            if (yk[k]) o = __fadd_rn(o, __fmul_rn(wk[k], yv[k]));
                        if (p.out_bf16) {
                            static_cast<uint16_t*>(p.out)[static_cast<size_t>(t) * p.H + c] = f32_to_bf16_bits(o);
                        } else {
                            static_cast<float*>(p.out)[static_cast<size_t>(t) * p.H + c] = o;
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.tfree[tb]);
        eph ^= 1u;
    }
}

template <int QT, int NT, bool G>
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
            mbar_init(&s.empty[i], kGroupWarps);
        }
        for (int i = 0; i < kMaxActSlots; ++i) {
            mbar_init(&s.afull[i], 1);
            mbar_init(&s.aempty[i], kConsumerWarps);
        }
        for (int i = 0; i < kTaskSlots; ++i) {
            mbar_init(&s.tfull[i], kConsumerWarps);
            mbar_init(&s.tfree[i], 1);
        }
        mbar_init(s.route_bar, 1);
        *s.rt_U = -1;  // until the routing sets it
        s.flag[1] = 0;  // set once x is quantised during the router rows
        s.flag[2] = 0;  // the test limit on waits: the helper warp fetches it (default until then)
        for (int i = 0; i < kMaxActSlots; ++i) {
            mbar_init(&s.areq_full[i], 1);
            mbar_init(&s.areq_free[i], 1);
        }
        fence_mbar_init();
        grid_launch_dependents();
    }
    __syncthreads();
    // everyone but the producer waits for the previous grid here (x, the
    // workspace and its launch counter may come from it)
    if (warp != kProducerWarp) grid_dependency_wait();
    if (warp == kProducerWarp) {
        if (lane == 0) producer<QT, G>(p, s);
    } else if (warp == kHelperWarp) {
        helper_warp<QT>(p, s);
    } else if (warp >= kEpilogueWarp0) {
        epilogue_warp<QT>(p, s, warp - kEpilogueWarp0);
    } else {
        consumer<QT, NT, G>(p, s);
    }
    // Count this CTA out: the add releases the counters its warps advanced
    // (ordered before it by the barrier) and, in the last CTA, acquires every
    // other CTA's.  The last CTA then clears what this launch advanced for the
    // next call on this workspace: completion counters 0 .. U (the shared
    // expert and the U routed ones; all of them if the routing did not finish)
    // and the row-block counters.  Kernel completion makes the stores visible
    // to the next grid.
    __syncthreads();
    if (tid == 0) s.flag[0] = atom_add_acq_rel_gpu(&p.sync->exit_count, 1) == static_cast<int>(gridDim.x) - 1;
    __syncthreads();
    if (s.flag[0]) {
        const int nu = *s.rt_U;
        const int nr = nu >= 0 && nu < p.E ? nu : p.E;
        for (int i = tid; i <= nr; i += kThreadsF) p.ug_done[i] = 0;
        for (int i = tid; i < p.n_dt; i += kThreadsF) p.rb_done[i] = 0;
        if (tid == 0) {
            p.sync->ticket = 0;
            p.sync->exit_count = 0;
            *p.epoch = *s.tag;
        }
    }
}

template <int QT>
const void* fused_kernel(int nt, bool grouped) {
    if (grouped)
        return nt == 1 ? reinterpret_cast<const void*>(k_decode_fused<QT, 1, true>)
                       : reinterpret_cast<const void*>(k_decode_fused<QT, kMaxT, true>);
    return nt == 1 ? reinterpret_cast<const void*>(k_decode_fused<QT, 1, false>)
                   : reinterpret_cast<const void*>(k_decode_fused<QT, kMaxT, false>);
}

}  // namespace

bool fused_geometry(FusedParams& p, int qtype) {
    // one warp routes the batch: experts lane + 32 j in registers (E <= 256),
    // groups of a multiple of 32 experts, the batch's T K pairs in one warp
    if (p.T < 1 || p.T > kMaxT || p.K < 1 || p.K > kMaxExpertsPerLane || p.K * p.T > 32 || p.T * p.E > kFusedMaxSlots)
        return false;
    if (p.E % 32 || p.E > 32 * kMaxExpertsPerLane || p.G < 1 || p.E % p.G || (p.E / p.G) % 32) return false;
    if (p.TG < 1 || p.TG > p.G || p.TG * (p.E / p.G) < p.K) return false;
    const size_t rb_ug = static_cast<size_t>(p.H) * qtype / 8, rb_d = static_cast<size_t>(p.I) * qtype / 8;
    size_t stage = std::max(static_cast<size_t>(4) * p.H, kStageRows * rb_ug);
    stage = (stage + 127) / 128 * 128;
    const int sr = static_cast<int>(stage / (kStageRows * rb_d)) * kStageRows;
    if (sr < kStageRows || sr > kGroupWarps * kMaxDownRowsPerWarp || sr * 4 > kScaleBytes) return false;
    p.stage_bytes = static_cast<int>(stage);
    p.rps = std::min<int>(kMaxRouterRows, static_cast<int>(stage / (4 * static_cast<size_t>(p.H))));
    p.n_rt = (p.E + p.rps - 1) / p.rps;
    p.sr_down = sr;
    p.dr = sr * kDownStagesPerTile;
    p.n_ugt = p.I / kUgTileRows;
    p.n_dt = (p.H + p.dr - 1) / p.dr;
    p.rec_bytes = static_cast<int>(fused_record_bytes(p.I));
    p.act_bytes = static_cast<int>(a16(static_cast<size_t>(p.T) * p.rec_bytes));
    {
        const size_t xs_bytes = a16(std::max(static_cast<size_t>(p.T) * p.H * 2, sizeof(RouteScratch)));
        p.nact = kActSlots + static_cast<int>(std::min<size_t>(kMaxActSlots - kActSlots, xs_bytes / p.act_bytes));
    }
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
        case MOE_Q_INT4: kern = fused_kernel<4>(p.nt, p.routed.group_size != 0); break;
        case MOE_Q_INT8: kern = fused_kernel<8>(p.nt, p.routed.group_size != 0); break;
        case MOE_Q_INT2: kern = fused_kernel<2>(p.nt, p.routed.group_size != 0); break;
        default: return cudaErrorInvalidValue;
    }
    e = ensure_smem(kern, smem);
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: this grid may start while the previous
    // one in the stream drains (it waits for it before touching shared data)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreadsF);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {const_cast<FusedParams*>(&p)};
    e = cudaLaunchKernelExC(&cfg, kern, args);
    if (e != cudaSuccess) return e;
    return counted(cudaGetLastError());
}

}  // namespace moe
