// Launch wrappers of the library's kernels (internal; the C ABI is in moe.h).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace moe {

// Raises a kernel's dynamic shared-memory cap to `bytes` (once per kernel and device).
cudaError_t ensure_smem(const void* kernel, size_t bytes);

// Adds n to the process-wide count of kernels this library launched.
void count_launch(int n = 1);

// MOE_OK or MOE_EINVAL: the router configuration limits of moe.h (every
// entry point that takes a moe_router_cfg checks it with this function).
int check_cfg(const moe_router_cfg* c);

// Returns e after counting one launch when it succeeded.
inline cudaError_t counted(cudaError_t e) {
    if (e == cudaSuccess) count_launch(1);
    return e;
}

cudaError_t launch_router_logits(const uint16_t* x, int T, int H, const float* w, int E,
                                 float* logits, cudaStream_t st);
cudaError_t launch_router_select(const float* logits, int T, const float* bias,
                                 const moe_router_cfg& c, int32_t* idx, float* w, int32_t* status,
                                 cudaStream_t st);

cudaError_t launch_union(const int32_t* idx, int T, int K, int E, int32_t* n_unique, int32_t* uniq,
                         int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot, int32_t* counts,
                         int32_t* status, cudaStream_t st);

cudaError_t launch_q8_0(const void* v, bool bf16, long rows, int n, int8_t* q, float* d,
                        cudaStream_t st);

// Union descriptor of one expert pass.  uniq == nullptr: dense mode (expert 0, pair p = token p).
struct UnionView {
    const int32_t* n_unique;
    const int32_t* uniq;
    const int32_t* offsets;
    const int32_t* pair_tok;
    const int32_t* pair_slot;
    int max_unique;  // grid bound (device value n_unique <= max_unique)
};

// Tokens each expert of a union sees on average (rounded up): it picks the
// general path kernels' CTA geometry.  A dense view (uniq null) is one expert
// seeing all T tokens.
inline int tokens_per_expert(const UnionView& un, int T, int top_k) {
    if (!un.uniq) return T;
    const long long pairs = static_cast<long long>(T) * top_k;
    return static_cast<int>((pairs + un.max_unique - 1) / un.max_unique);
}
// A shared expert of the routed experts' shape computed in the same launch
// (grid row 0, all T tokens): its weights and outputs; w_gate / w_down null
// when there is none.
struct SharedUpGate {
    const uint8_t* w_gate;
    const uint8_t* w_up;
    const float* s_gate;
    const float* s_up;
    int8_t* qh;  // [T][I]
    float* dh;   // [T][I/32]
};
struct SharedDown {
    const uint8_t* w_down;
    const float* s_down;
    const int8_t* qh;  // [T][I]
    const float* dh;   // [T][I/32]
    float* y;          // [T][H]
};
// up/gate + SwiGLU + Q8_0(h) for every pair; qh [P][I], dh [P][I/32] by pair index.
cudaError_t launch_expert_up_gate(const moe_experts& ex, const int8_t* qx, const float* dx, int T,
                                  const UnionView& un, int tok_per_expert, int8_t* qh, float* dh,
                                  const SharedUpGate& sx, cudaStream_t st);
// down rows for every pair, written to y_pairs[tok][slot][:].
cudaError_t launch_expert_down(const moe_experts& ex, const int8_t* qh, const float* dh, int T,
                               int top_k, const UnionView& un, int tok_per_expert, float* y_pairs,
                               const SharedDown& sx, cudaStream_t st);

cudaError_t launch_usage_accumulate(const int32_t* idx, long n, int E, uint32_t* usage, cudaStream_t st);
cudaError_t launch_usage_rank(const uint32_t* usage, int E, int32_t* order, cudaStream_t st);
cudaError_t launch_combine(const float* y, const float* w, const float* shared_y, int T, int K,
                           int H, void* out, int out_dtype, cudaStream_t st);

// ------------------------------------------------------------ fused small-batch layer
constexpr int kFusedMaxTokens = 4;
// Up to this many tokens a call's experts see one or two tokens each: the
// lane-per-row integer-dot kernels beat 128-row tensor-core tiles there
// (GLM-5.2 shape: 0.43 against 1.09 ms per layer at 8 tokens, 1.78 against
// 2.60 ms at 32; at 64 the tensor cores were faster than earlier versions of
// those kernels), so int4 batches take the tensor cores only above it.
constexpr int kGeneralMaxTokens = 32;

// Control block at the start of every workspace (kWsHeader bytes).  The
// counters before kWsScoresOff are zero when idle.  The score slots hold the
// router scores of the last launch, each tagged with its launch number; the
// word at kWsEpochOff counts the fused kernel's launches on this workspace and
// is never cleared, so a slot written by an earlier launch (or zeroed by a
// status clear) never carries the current launch's tag.  Nothing but the
// fused kernel writes the slots.
struct FusedSync {
    int ticket;
    int exit_count;
    int wait_limit;  // test knob: nonzero caps every bounded wait at that many polls
    int pad[13];
};
constexpr size_t kWsStatusOff = 0;
constexpr size_t kWsSyncOff = 64;
constexpr size_t kWsUgDoneOff = 128;                    // int[E + 1], E <= 1024
constexpr size_t kWsRbDoneOff = kWsUgDoneOff + 4 * 1032; // int[n_dt], n_dt <= 16384 / 32 + 1
constexpr size_t kWsScoresOff = 6400;                   // u64[T * E], T * E <= kFusedMaxSlots
constexpr int kFusedMaxSlots = 1024;
constexpr size_t kWsEpochOff = kWsHeader - 64;
static_assert(kWsRbDoneOff + 4 * 520 <= kWsScoresOff, "workspace header too small");
static_assert(kWsScoresOff + 8 * kFusedMaxSlots <= kWsEpochOff, "workspace header too small");

struct FusedParams {
    const uint16_t* x;
    int T, H, I, E, G, TG, K;
    float rsf;
    float top_p;  // adaptive expert top-p (off outside (0, 1))
    const float* w_router;
    const float* bias;
    moe_experts routed;
    moe_experts shared;
    int has_shared;
    void* out;
    int out_bf16;
    int32_t* idx;
    float* w;
    int32_t* status;
    FusedSync* sync;
    int32_t* ug_done;
    int32_t* rb_done;
    uint32_t* epoch;                 // launch counter (workspace header, never cleared)
    unsigned long long* scores;      // [T][E] router scores, low word fp32 bits, high word launch tag
    int32_t* n_unique;
    int32_t* uniq;
    int32_t* offsets;
    int32_t* pair_tok;
    int32_t* pair_slot;
    int32_t* pair_of;
    uint8_t* qrec;  // [(T*K + T)][rec_bytes] permuted Q8_0(h) records
    float* y;       // [(T*K + T)][H] per-pair expert outputs (shared rows last)
    int rec_bytes;
    int nstage, stage_bytes, act_bytes, sr_down, dr, n_ugt, n_dt;
    int nact;  // activation-record slots (2 of their own, the rest in the x cache)
    int rps;   // router rows per stage
    int n_rt;  // router tickets
    int nt;    // token capacity of the kernel instantiation (1 or kFusedMaxTokens)
};

// Bytes of one pair's Q8_0(h) record: two 16-byte planes per block, the block
// scales and block sums, padded so records can be bulk-copied back to back.
inline size_t fused_record_bytes(int I) { return (static_cast<size_t>(I) + I / 4 + 15) & ~size_t(15); }

// ------------------------------------------------------------ tensor-core batch-union FFN
// (prefill and long verify: every unique expert applied to its tokens in 128-row tiles)
constexpr int kGemmUpGate = 0, kGemmDown = 1;

struct GemmParams {
    int T, H, I, P, K, has_shared;
    const int32_t* n_unique;
    const int32_t* uniq;
    const int32_t* offsets;
    const int32_t* pair_tok;
    const int32_t* pair_slot;
    const void* a_codes;     // activation Q8_0 codes as fp16: up/gate x [T][H]; down h [(P + T)][I]
    const float* a_scales;   // their block scales [rows][K / 32]
    const float* s_a;        // row scales: up/gate: gate [E][I]; down: down [E][H]
    const float* s_b;        // up/gate: up [E][I]
    const float* s_a_sh;     // shared expert's
    const float* s_b_sh;
    void* h_codes;           // up/gate out: Q8_0(h) codes as fp16 [(P + T)][I] (union order, shared rows last)
    float* h_scales;         //              block scales [(P + T)][I / 32]
    float* y;                // down out: routed [T][K][H]
    float* ys;               //           shared [T][H]
    int32_t* status;
    const int32_t* wait_limit;  // the workspace header's test limit on pipeline waits
};

struct GemmOperands {
    const void* w0;          // packed routed weights: gate (up/gate) or down
    const void* w1;          // packed routed up weights
    const void* w0s;         // shared expert's
    const void* w1s;
    int n_expert;
};

bool tc_gemm_supported(const moe_experts& r, const moe_experts* s, int E);
cudaError_t launch_gather_codes(const int8_t* q, int H, int P, int rows, const int32_t* pair_tok, __half* out,
                                cudaStream_t st);
cudaError_t launch_moe_gemm(int mode, const GemmParams& p, const GemmOperands& o, cudaStream_t st);

// Fills the geometry fields; false if the fused kernel cannot take this shape.
bool fused_geometry(FusedParams& p, int qtype);
size_t fused_smem_bytes(const FusedParams& p);
cudaError_t launch_decode_fused(const FusedParams& p, cudaStream_t st);

}  // namespace moe
