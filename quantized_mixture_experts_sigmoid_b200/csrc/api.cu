// C ABI entry points (declared in include/moe.h): argument checks, workspace
// carving and the launch sequence of each call.  No device memory is
// allocated here; every scratch buffer is carved from the caller's workspace.
#include <algorithm>
#include <cstddef>
#include <atomic>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.cuh"

using namespace moe;

namespace {
// An NVTX range named after the entry point, open for the call's duration
// (visible in profilers; without one attached it costs a few nanoseconds).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace

namespace moe {

cudaError_t ensure_smem(const void* kernel, size_t bytes) {
    static std::mutex mu;
    static std::vector<std::pair<const void*, int>> done;  // (kernel, device) raised to 227 KB
    if (bytes <= 48 * 1024) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    for (const auto& d : done)
        if (d.first == kernel && d.second == dev) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e == cudaSuccess) done.emplace_back(kernel, dev);
    return e;
}

namespace {
std::atomic<long long> g_launches{0};
}

void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int check_cfg(const moe_router_cfg* c) {
    if (!c) return MOE_EINVAL;
    const int E = c->n_expert, G = c->n_group;
    if (E <= 0 || E > 1024 || G <= 0 || G > 32 || E % G != 0 || E / G < 2) return MOE_EINVAL;
    if (c->topk_group <= 0 || c->topk_group > G) return MOE_EINVAL;
    if (c->top_k <= 0 || c->top_k > 32 || c->top_k > c->topk_group * (E / G)) return MOE_EINVAL;
    if (!(c->routed_scaling_factor == c->routed_scaling_factor)) return MOE_EINVAL;
    return MOE_OK;
}

}  // namespace moe

namespace {

// Event pairs recorded around the dominant kernel while profiling is enabled.
struct Profiler {
    bool on = false;
    int used = 0;
    std::vector<cudaEvent_t> ev;  // start, stop, start, stop, ...
    static constexpr int kMax = 65536;
    bool begin(cudaStream_t st) {
        if (!on || used >= kMax) return false;
        while (static_cast<int>(ev.size()) < 2 * (used + 1)) {
            cudaEvent_t e;
            if (cudaEventCreate(&e) != cudaSuccess) return false;
            ev.push_back(e);
        }
        return cudaEventRecord(ev[2 * used], st) == cudaSuccess;
    }
    void end(cudaStream_t st) {
        if (cudaEventRecord(ev[2 * used + 1], st) == cudaSuccess) ++used;
    }
};
Profiler g_prof;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

int check_experts(const moe_experts* ex) {
    if (!ex) return MOE_EINVAL;
    if (ex->qtype != MOE_Q_INT2 && ex->qtype != MOE_Q_INT4 && ex->qtype != MOE_Q_INT8)
        return MOE_EUNSUPPORTED;
    if (ex->n_expert <= 0 || ex->hidden <= 0 || ex->inter <= 0) return MOE_EINVAL;
    if (ex->hidden % 32 || ex->inter % 32) return MOE_EINVAL;
    if (ex->hidden > 16384 || ex->inter > 16384) return MOE_EUNSUPPORTED;
    const int gs = ex->group_size;
    if (gs < 0 || (gs && (gs % 32 || ex->hidden % gs || ex->inter % gs))) return MOE_EINVAL;
    const void* ps[6] = {ex->w_gate, ex->w_up, ex->w_down, ex->s_gate, ex->s_up, ex->s_down};
    for (const void* p : ps)
        if (!p || !aligned16(p)) return MOE_EINVAL;
    return MOE_OK;
}

// The CUDA error behind the most recent MOE_ECUDA returned on this thread.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

int cuda_rc(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    g_last_cuda_error = e;
    return MOE_ECUDA;
}

struct LayerWs {
    int32_t* status;
    float* logits;
    int32_t* idx;
    float* w;
    int32_t* n_unique;
    int32_t* uniq;
    int32_t* offsets;
    int32_t* pair_tok;
    int32_t* pair_slot;
    int8_t* qx;
    float* dx;
    int8_t* qh;
    float* dh;
    int8_t* qhs;
    float* dhs;
    float* y;
    float* ys;
    // tensor-core batch-union path (T > kGeneralMaxTokens, int4)
    __half* xg;    // Q8_0(x) codes as fp16 per up/gate row [(P + T)][H] (union order, shared rows last)
    __half* hc;    // Q8_0(h) codes as fp16 [(P + T)][I]
    float* hs;     // their block scales
    // fused small-batch path only (T <= kFusedMaxTokens)
    int32_t* pair_of;
    uint8_t* qrec;
    float* yf;
    size_t bytes;
};

LayerWs carve_layer(void* ws, int T, const moe_router_cfg& c, const moe_experts& r,
                    const moe_experts* s) {
    Carver cv(ws, 0);
    LayerWs L{};
    L.status = cv.take<int32_t>(kWsHeader / sizeof(int32_t));
    const size_t P = static_cast<size_t>(T) * c.top_k;
    const int H = r.hidden, I = r.inter;
    L.logits = cv.take<float>(static_cast<size_t>(T) * c.n_expert);
    L.idx = cv.take<int32_t>(P);
    L.w = cv.take<float>(P);
    L.n_unique = cv.take<int32_t>(4);
    L.uniq = cv.take<int32_t>(c.n_expert);
    L.offsets = cv.take<int32_t>(c.n_expert + 1);
    L.pair_tok = cv.take<int32_t>(P);
    L.pair_slot = cv.take<int32_t>(P);
    L.qx = cv.take<int8_t>(static_cast<size_t>(T) * H);
    L.dx = cv.take<float>(static_cast<size_t>(T) * H / 32);
    L.qh = cv.take<int8_t>(P * I);
    L.dh = cv.take<float>(P * I / 32);
    if (s) {
        L.qhs = cv.take<int8_t>(static_cast<size_t>(T) * s->inter);
        L.dhs = cv.take<float>(static_cast<size_t>(T) * s->inter / 32);
        L.ys = cv.take<float>(static_cast<size_t>(T) * H);
    }
    L.y = cv.take<float>(P * H);
    if (T > kGeneralMaxTokens && tc_gemm_supported(r, s, c.n_expert)) {
        const size_t rows = P + static_cast<size_t>(T);
        L.xg = cv.take<__half>(rows * H);
        L.hc = cv.take<__half>(rows * I);
        L.hs = cv.take<float>(rows * I / 32);
    }
    if (T <= kFusedMaxTokens) {
        L.pair_of = cv.take<int32_t>(P);
        L.qrec = cv.take<uint8_t>((P + T) * fused_record_bytes(I));
        L.yf = cv.take<float>((P + T) * static_cast<size_t>(H));
    }
    L.bytes = align_up(cv.off, 256);
    return L;
}

// The fused kernel takes small batches whose shared expert (if any) has the
// routed experts' qtype and intermediate size.
bool fused_params(FusedParams& f, const LayerWs& L, void* ws, const uint16_t* x, int T,
                  const float* w_router, const float* bias, const moe_router_cfg& c,
                  const moe_experts& r, const moe_experts* s, void* out, int out_dtype,
                  int32_t* idx, float* w) {
    if (T > kFusedMaxTokens) return false;
    if (s && (s->qtype != r.qtype || s->inter != r.inter || s->hidden != r.hidden || s->group_size != r.group_size))
        return false;
    f = FusedParams{};
    f.x = x;
    f.T = T;
    f.H = r.hidden;
    f.I = r.inter;
    f.E = c.n_expert;
    f.G = c.n_group;
    f.TG = c.topk_group;
    f.K = c.top_k;
    f.rsf = c.routed_scaling_factor;
    f.top_p = c.top_p;
    f.w_router = w_router;
    f.bias = bias;
    f.routed = r;
    if (s) f.shared = *s;
    f.has_shared = s != nullptr;
    f.out = out;
    f.out_bf16 = out_dtype == MOE_OUT_BF16;
    f.idx = idx;
    f.w = w;
    char* base = static_cast<char*>(ws);
    f.status = reinterpret_cast<int32_t*>(base + kWsStatusOff);
    f.sync = reinterpret_cast<FusedSync*>(base + kWsSyncOff);
    f.ug_done = reinterpret_cast<int32_t*>(base + kWsUgDoneOff);
    f.rb_done = reinterpret_cast<int32_t*>(base + kWsRbDoneOff);
    f.epoch = reinterpret_cast<uint32_t*>(base + kWsEpochOff);
    f.scores = reinterpret_cast<unsigned long long*>(base + kWsScoresOff);
    f.n_unique = L.n_unique;
    f.uniq = L.uniq;
    f.offsets = L.offsets;
    f.pair_tok = L.pair_tok;
    f.pair_slot = L.pair_slot;
    f.pair_of = L.pair_of;
    f.qrec = L.qrec;
    f.y = L.yf;
    return fused_geometry(f, r.qtype);
}

struct FfnWs {
    int32_t* status;
    int8_t* qx;
    float* dx;
    int8_t* qh;
    float* dh;
    size_t bytes;
};

FfnWs carve_ffn(void* ws, const moe_experts& ex, int T, int top_k) {
    Carver cv(ws, 0);
    FfnWs F{};
    const size_t P = static_cast<size_t>(T) * top_k;
    F.status = cv.take<int32_t>(kWsHeader / sizeof(int32_t));
    F.qx = cv.take<int8_t>(static_cast<size_t>(T) * ex.hidden);
    F.dx = cv.take<float>(static_cast<size_t>(T) * ex.hidden / 32);
    F.qh = cv.take<int8_t>(P * ex.inter);
    F.dh = cv.take<float>(P * ex.inter / 32);
    F.bytes = align_up(cv.off, 256);
    return F;
}

size_t route_ws_bytes(int T, int E) {
    Carver cv(nullptr, 0);
    cv.take<int32_t>(kWsHeader / sizeof(int32_t));
    cv.take<float>(static_cast<size_t>(T) * E);
    return align_up(cv.off, 256);
}

}  // namespace

extern "C" {

const char* moe_strerror(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_EINVAL: return "invalid argument (size, null or misaligned pointer, or router config)";
        case MOE_EWORKSPACE: return "workspace too small or not 256-byte aligned";
        case MOE_EUNSUPPORTED: return "unsupported qtype or size";
        case MOE_ECUDA: return "CUDA launch or copy failed";
        case MOE_EDEVICE_TIMEOUT: return "a bounded device-side wait gave up";
        case MOE_EDEVICE_INDEX: return "a kernel saw an expert index outside [0, E)";
        case MOE_ETOO_LARGE: return "batch exceeds the fixed scratch capacity of moe_route_noalloc";
        default: return "unknown moe error code";
    }
}

const char* moe_cuda_error_string(void) {
    return g_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(g_last_cuda_error);
}

size_t moe_route_workspace_bytes(int T, const moe_router_cfg* cfg) {
    if (T < 0 || check_cfg(cfg) != MOE_OK) return 0;
    return route_ws_bytes(T, cfg->n_expert);
}

int moe_route(const uint16_t* x, int T, int H, const float* w_router, const float* bias,
              const moe_router_cfg* cfg, int32_t* topk_idx, float* topk_w, void* ws,
              size_t ws_bytes, moe_stream_t stream) {
    NvtxRange nvtx("moe_route");
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (T < 0 || H <= 0 || H % 32) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (!x || !w_router || !bias || !topk_idx || !topk_w || !aligned16(x) || !aligned16(w_router) ||
        !aligned16(bias) || !aligned16(topk_idx) || !aligned16(topk_w))
        return MOE_EINVAL;
    if (!ws || !aligned256(ws) || ws_bytes < route_ws_bytes(T, cfg->n_expert)) return MOE_EWORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float* logits = reinterpret_cast<float*>(static_cast<char*>(ws) + kWsHeader);
    rc = cuda_rc(launch_router_logits(x, T, H, w_router, cfg->n_expert, logits, st));
    if (rc) return rc;
    return cuda_rc(launch_router_select(logits, T, bias, *cfg, topk_idx, topk_w,
                                        static_cast<int32_t*>(ws), st));
}

int moe_union(const int32_t* topk_idx, int T, int top_k, int E, int32_t* n_unique, int32_t* uniq,
              int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot, int32_t* counts,
              int32_t* status, moe_stream_t stream) {
    NvtxRange nvtx("moe_union");
    if (T < 0 || top_k <= 0 || top_k > 32 || E <= 0 || E > 1024) return MOE_EINVAL;
    if (!n_unique || !uniq || !offsets) return MOE_EINVAL;
    if (T > 0 && (!topk_idx || !pair_tok || !pair_slot)) return MOE_EINVAL;
    if (static_cast<long long>(T) * top_k > (1ll << 30)) return MOE_EUNSUPPORTED;
    return cuda_rc(launch_union(topk_idx, T, top_k, E, n_unique, uniq, offsets, pair_tok, pair_slot,
                                counts, status, reinterpret_cast<cudaStream_t>(stream)));
}

int moe_quantize_q8_0(const void* v, int in_dtype, int rows, int n, int8_t* q, float* d,
                      moe_stream_t stream) {
    NvtxRange nvtx("moe_quantize_q8_0");
    if (rows < 0 || n <= 0 || n % 32) return MOE_EINVAL;
    if (in_dtype != MOE_OUT_BF16 && in_dtype != MOE_OUT_F32) return MOE_EINVAL;
    if (rows == 0) return MOE_OK;
    if (!v || !q || !d) return MOE_EINVAL;
    return cuda_rc(launch_q8_0(v, in_dtype == MOE_OUT_BF16, rows, n, q, d,
                               reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_expert_ffn_workspace_bytes(const moe_experts* ex, int T, int top_k) {
    if (!ex || T < 0 || top_k <= 0 || ex->hidden <= 0 || ex->inter <= 0) return 0;
    return carve_ffn(nullptr, *ex, T, top_k).bytes;
}

int moe_expert_ffn_q(const moe_experts* ex, const uint16_t* x, int T, int top_k,
                     const int32_t* n_unique, const int32_t* uniq, const int32_t* offsets,
                     const int32_t* pair_tok, const int32_t* pair_slot, float* y_pairs, void* ws,
                     size_t ws_bytes, moe_stream_t stream) {
    NvtxRange nvtx("moe_expert_ffn_q");
    int rc = check_experts(ex);
    if (rc) return rc;
    if (T < 0 || top_k <= 0 || top_k > 32) return MOE_EINVAL;
    const bool dense = uniq == nullptr;
    if (dense) {
        if (n_unique || offsets || pair_tok || pair_slot || top_k != 1) return MOE_EINVAL;
    } else if (!n_unique || !offsets || !pair_tok || !pair_slot) {
        return MOE_EINVAL;
    }
    if (T == 0) return MOE_OK;
    if (!x || !y_pairs || !aligned16(x) || !aligned16(y_pairs)) return MOE_EINVAL;
    const FfnWs F0 = carve_ffn(nullptr, *ex, T, top_k);
    if (!ws || !aligned256(ws) || ws_bytes < F0.bytes) return MOE_EWORKSPACE;
    const FfnWs F = carve_ffn(ws, *ex, T, top_k);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    UnionView un{n_unique, uniq, offsets, pair_tok, pair_slot,
                 dense ? 1 : static_cast<int>(std::min<long long>(ex->n_expert, static_cast<long long>(T) * top_k))};
    rc = cuda_rc(launch_q8_0(x, true, T, ex->hidden, F.qx, F.dx, st));
    if (rc) return rc;
    const int tpe = tokens_per_expert(un, T, top_k);
    rc = cuda_rc(launch_expert_up_gate(*ex, F.qx, F.dx, T, un, tpe, F.qh, F.dh, SharedUpGate{}, st));
    if (rc) return rc;
    return cuda_rc(launch_expert_down(*ex, F.qh, F.dh, T, top_k, un, tpe, y_pairs, SharedDown{}, st));
}

int moe_combine(const float* y_pairs, const float* topk_w, const float* shared_y, int T, int top_k,
                int H, void* out, int out_dtype, moe_stream_t stream) {
    NvtxRange nvtx("moe_combine");
    if (T < 0 || top_k <= 0 || top_k > 32 || H <= 0 || H % 4) return MOE_EINVAL;
    if (out_dtype != MOE_OUT_BF16 && out_dtype != MOE_OUT_F32) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (!y_pairs || !topk_w || !out || !aligned16(y_pairs) || !aligned16(out) ||
        (shared_y && !aligned16(shared_y)))
        return MOE_EINVAL;
    return cuda_rc(launch_combine(y_pairs, topk_w, shared_y, T, top_k, H, out, out_dtype,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

int moe_usage_accumulate(const int32_t* topk_idx, int T, int top_k, int E, uint32_t* usage,
                         moe_stream_t stream) {
    NvtxRange nvtx("moe_usage_accumulate");
    if (T < 0 || top_k <= 0 || top_k > 32 || E <= 0 || E > 1024) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (!topk_idx || !usage) return MOE_EINVAL;
    return cuda_rc(launch_usage_accumulate(topk_idx, static_cast<long>(T) * top_k, E, usage,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

int moe_usage_rank(const uint32_t* usage, int E, int32_t* order, moe_stream_t stream) {
    NvtxRange nvtx("moe_usage_rank");
    if (E <= 0 || E > 1024 || !usage || !order) return MOE_EINVAL;
    return cuda_rc(launch_usage_rank(usage, E, order, reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_layer_workspace_bytes(int T, const moe_router_cfg* cfg, const moe_experts* routed,
                                 const moe_experts* shared) {
    if (T < 0 || check_cfg(cfg) != MOE_OK || !routed || routed->hidden <= 0 || routed->inter <= 0)
        return 0;
    return carve_layer(nullptr, T, *cfg, *routed, shared).bytes;
}

int moe_layer_forward(const uint16_t* x, int T, const float* w_router, const float* bias,
                      const moe_router_cfg* cfg, const moe_experts* routed,
                      const moe_experts* shared, void* out, int out_dtype, int32_t* topk_idx_out,
                      float* topk_w_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    NvtxRange nvtx("moe_layer_forward");
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if ((rc = check_experts(routed))) return rc;
    if (shared && (rc = check_experts(shared))) return rc;
    if (routed->n_expert != cfg->n_expert) return MOE_EINVAL;
    if (shared && shared->hidden != routed->hidden) return MOE_EINVAL;
    if (out_dtype != MOE_OUT_BF16 && out_dtype != MOE_OUT_F32) return MOE_EINVAL;
    if (T < 0) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (!x || !w_router || !bias || !out || !aligned16(x) || !aligned16(w_router) ||
        !aligned16(bias) || !aligned16(out))
        return MOE_EINVAL;
    if ((topk_idx_out && !aligned16(topk_idx_out)) || (topk_w_out && !aligned16(topk_w_out)))
        return MOE_EINVAL;
    const LayerWs L0 = carve_layer(nullptr, T, *cfg, *routed, shared);
    if (!ws || !aligned256(ws) || ws_bytes < L0.bytes) return MOE_EWORKSPACE;
    const LayerWs L = carve_layer(ws, T, *cfg, *routed, shared);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int H = routed->hidden, K = cfg->top_k, E = cfg->n_expert;
    int32_t* idx = topk_idx_out ? topk_idx_out : L.idx;
    float* w = topk_w_out ? topk_w_out : L.w;

    FusedParams f;
    if (fused_params(f, L, ws, x, T, w_router, bias, *cfg, *routed, shared, out, out_dtype, idx, w)) {
        const bool timed = g_prof.begin(st);
        rc = cuda_rc(launch_decode_fused(f, st));
        if (timed) g_prof.end(st);
        return rc;
    }

    if ((rc = cuda_rc(launch_router_logits(x, T, H, w_router, E, L.logits, st)))) return rc;
    if ((rc = cuda_rc(launch_router_select(L.logits, T, bias, *cfg, idx, w, L.status, st)))) return rc;
    if ((rc = cuda_rc(launch_union(idx, T, K, E, L.n_unique, L.uniq, L.offsets, L.pair_tok,
                                   L.pair_slot, nullptr, L.status, st))))
        return rc;
    if ((rc = cuda_rc(launch_q8_0(x, true, T, H, L.qx, L.dx, st)))) return rc;

    if (L.xg) {  // many tokens per expert: tensor-core batch-union FFN
        const int I = routed->inter, P = T * K;
        if ((rc = cuda_rc(launch_gather_codes(L.qx, H, P, P + (shared ? T : 0), L.pair_tok, L.xg, st)))) return rc;
        GemmParams gp{};
        gp.T = T;
        gp.H = H;
        gp.I = I;
        gp.P = P;
        gp.K = K;
        gp.has_shared = shared != nullptr;
        gp.n_unique = L.n_unique;
        gp.uniq = L.uniq;
        gp.offsets = L.offsets;
        gp.pair_tok = L.pair_tok;
        gp.pair_slot = L.pair_slot;
        gp.status = L.status;
        gp.wait_limit = &reinterpret_cast<const FusedSync*>(reinterpret_cast<const uint8_t*>(L.status) + kWsSyncOff)->wait_limit;
        GemmOperands go{};
        go.n_expert = E;
        // up/gate: Q8_0(h) per pair (union order), shared rows last
        gp.a_codes = L.xg;
        gp.a_scales = L.dx;
        gp.s_a = routed->s_gate;
        gp.s_b = routed->s_up;
        gp.s_a_sh = shared ? shared->s_gate : nullptr;
        gp.s_b_sh = shared ? shared->s_up : nullptr;
        gp.h_codes = L.hc;
        gp.h_scales = L.hs;
        go.w0 = routed->w_gate;
        go.w1 = routed->w_up;
        go.w0s = shared ? shared->w_gate : nullptr;
        go.w1s = shared ? shared->w_up : nullptr;
        // the profiled region covers both GEMM launches (up/gate and down)
        const bool timed = g_prof.begin(st);
        rc = cuda_rc(launch_moe_gemm(kGemmUpGate, gp, go, st));
        if (rc) {
            if (timed) g_prof.end(st);
            return rc;
        }
        // down: fp32 output per (token, slot), shared rows separately
        gp.a_codes = L.hc;
        gp.a_scales = L.hs;
        gp.s_a = routed->s_down;
        gp.s_b = nullptr;
        gp.s_a_sh = shared ? shared->s_down : nullptr;
        gp.s_b_sh = nullptr;
        gp.y = L.y;
        gp.ys = shared ? L.ys : nullptr;
        go.w0 = routed->w_down;
        go.w1 = nullptr;
        go.w0s = shared ? shared->w_down : nullptr;
        go.w1s = nullptr;
        rc = cuda_rc(launch_moe_gemm(kGemmDown, gp, go, st));
        if (timed) g_prof.end(st);
        if (rc) return rc;
        return cuda_rc(launch_combine(L.y, w, shared ? L.ys : nullptr, T, K, H, out, out_dtype, st));
    }

    const UnionView un{L.n_unique, L.uniq, L.offsets, L.pair_tok, L.pair_slot,
                       static_cast<int>(std::min<long long>(E, static_cast<long long>(T) * K))};
    const bool timed = g_prof.begin(st);
    const int tpe = tokens_per_expert(un, T, K);
    // a shared expert of the routed experts' shape rides in the routed launches
    // (grid row 0), so its few CTAs overlap theirs instead of running after them;
    // up to 8 tokens (beyond, its CTAs' passes over all T tokens outlast the
    // routed ones: measured 3% faster at T = 8, 11% for int8 at T = 4, 5% slower at 32)
    const bool ride = shared && T <= 8 && shared->qtype == routed->qtype && shared->hidden == routed->hidden &&
                      shared->inter == routed->inter && shared->group_size == routed->group_size;
    const SharedUpGate sug =
        ride ? SharedUpGate{shared->w_gate, shared->w_up, shared->s_gate, shared->s_up, L.qhs, L.dhs} : SharedUpGate{};
    const SharedDown sdn = ride ? SharedDown{shared->w_down, shared->s_down, L.qhs, L.dhs, L.ys} : SharedDown{};
    rc = cuda_rc(launch_expert_up_gate(*routed, L.qx, L.dx, T, un, tpe, L.qh, L.dh, sug, st));
    if (timed) g_prof.end(st);
    if (rc) return rc;
    const UnionView dense{nullptr, nullptr, nullptr, nullptr, nullptr, 1};
    if (shared && !ride &&
        (rc = cuda_rc(launch_expert_up_gate(*shared, L.qx, L.dx, T, dense, T, L.qhs, L.dhs, SharedUpGate{}, st))))
        return rc;
    if ((rc = cuda_rc(launch_expert_down(*routed, L.qh, L.dh, T, K, un, tpe, L.y, sdn, st)))) return rc;
    if (shared && !ride &&
        (rc = cuda_rc(launch_expert_down(*shared, L.qhs, L.dhs, T, 1, dense, T, L.ys, SharedDown{}, st))))
        return rc;
    return cuda_rc(launch_combine(L.y, w, shared ? L.ys : nullptr, T, K, H, out, out_dtype, st));
}

int moe_layer_path(int T, const moe_router_cfg* cfg, const moe_experts* routed, const moe_experts* shared) {
    if (!cfg || !routed || T <= 0 || check_cfg(cfg) || check_experts(routed) || (shared && check_experts(shared)))
        return MOE_EINVAL;
    const LayerWs L = carve_layer(nullptr, T, *cfg, *routed, shared);
    FusedParams f;
    void* fake = reinterpret_cast<void*>(static_cast<uintptr_t>(4096));  // geometry only: nothing is dereferenced
    const uint16_t* fx = reinterpret_cast<const uint16_t*>(fake);
    if (fused_params(f, L, fake, fx, T, reinterpret_cast<const float*>(fake), reinterpret_cast<const float*>(fake),
                     *cfg, *routed, shared, fake, MOE_OUT_F32, nullptr, nullptr))
        return MOE_PATH_FUSED;
    if (T > kGeneralMaxTokens && tc_gemm_supported(*routed, shared, cfg->n_expert)) return MOE_PATH_TENSOR_CORE;
    return MOE_PATH_GENERAL;
}

int moe_profile_enable(int on) {
    g_prof.on = on != 0;
    g_prof.used = 0;
    return MOE_OK;
}

int moe_profile_read(double* total_ms, int* launches) {
    if (!total_ms || !launches) return MOE_EINVAL;
    double sum = 0.0;
    for (int i = 0; i < g_prof.used; ++i) {
        if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess) return MOE_ECUDA;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess) return MOE_ECUDA;
        sum += ms;
    }
    *total_ms = sum;
    *launches = g_prof.used;
    return MOE_OK;
}

long long moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_workspace_set_wait_limit(void* ws, int polls, moe_stream_t stream) {
    NvtxRange nvtx("moe_workspace_set_wait_limit");
    if (!ws || polls < 0) return MOE_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int32_t v = polls;  // pageable source: copied out before the call returns
    const size_t off = kWsSyncOff + offsetof(FusedSync, wait_limit);
    if (cudaMemcpyAsync(static_cast<uint8_t*>(ws) + off, &v, sizeof(v), cudaMemcpyHostToDevice, st) != cudaSuccess)
        return MOE_ECUDA;
    return MOE_OK;
}

int moe_workspace_status(void* ws, int clear, int* status, moe_stream_t stream) {
    NvtxRange nvtx("moe_workspace_status");
    if (!ws || !status) return MOE_EINVAL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ECUDA;
    // the launch counter at the end of the header survives a clear
    if (clear && cudaMemsetAsync(ws, 0, kWsEpochOff, st) != cudaSuccess) return MOE_ECUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ECUDA;
    *status = h;
    return MOE_OK;
}

}  // extern "C"
