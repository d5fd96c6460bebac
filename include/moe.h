/*
 * moe.h -- C ABI of the B200 (sm_100a) routed Mixture-of-Experts layer.
 *
 * The layer is the one the colibri engine runs for GLM-5.2 (pages cited per
 * call below):
 *  [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기" (amuse.peoplentools.com)
 *  [MO] "Colibri: 25GB RAM을 탑재한 노트북에서 744B AI 모델 실행하기" (molayo1419.me)
 *  [YO] "Colibri: como corre um modelo de 744B parâmetros em uma laptop de
 *        32GB sem GPU, sem BLAS" (yodev.dev)
 *
 * Conventions for every call:
 *  - Pointers named in the signature are DEVICE pointers unless the comment
 *    says host.  The moe_router_cfg / moe_experts structs themselves live in
 *    host memory and are read during the call only.
 *  - The caller owns every buffer.  The library allocates no device memory:
 *    scratch comes from a caller-provided workspace `ws` of at least the
 *    size returned by the matching *_workspace_bytes query (256-byte aligned).
 *  - All calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and never synchronise the device, except
 *    moe_workspace_status, which says so.
 *  - Return 0 (MOE_OK) on success or a negative MOE_E* code.  On an argument
 *    error nothing is launched.
 *  - Device pointers must be 16-byte aligned; weight matrices are row-major.
 *  - bf16 values are passed as their 16-bit patterns (uint16_t).
 *  - Not thread-safe per workspace: two calls in flight that share a `ws`
 *    race on it.
 *  - The first 16 KiB of every workspace belong to the library: a status
 *    word, and for moe_layer_forward counters, router score slots and a
 *    launch counter that persist from one call to the next.  Zero-fill a
 *    workspace once before its first use and do not write into it afterwards.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* moe_stream_t; /* same type as cudaStream_t */

/* ---------------------------------------------------------------- errors */
#define MOE_OK 0
#define MOE_EINVAL (-1)         /* bad size, null or misaligned pointer, bad config */
#define MOE_EWORKSPACE (-2)     /* workspace too small or misaligned */
#define MOE_EUNSUPPORTED (-3)   /* qtype or size outside what the kernels handle */
#define MOE_ECUDA (-4)          /* a CUDA launch or copy failed */
#define MOE_EDEVICE_TIMEOUT (-5) /* a bounded device-side wait gave up (see moe_workspace_status) */
#define MOE_EDEVICE_INDEX (-6)  /* a kernel saw an out-of-range expert index (see moe_workspace_status) */
#define MOE_ETOO_LARGE (-7)     /* the batch exceeds a fixed capacity (moe_route_noalloc) */

/* Human-readable text of an MOE_* code (static string, never NULL). */
const char* moe_strerror(int code);

/* Text of the CUDA error behind the most recent MOE_ECUDA that a call of this
 * library returned on the calling thread ("no CUDA error" if none; static
 * string, never NULL).  This library's own diagnostic, not a step of the layer. */
const char* moe_cuda_error_string(void);

/* ------------------------------------------------------------ data types */

/* Weight code width.  Layout of one row of n codes (the pages name packed
 * int4 / int2 and int8 with per-row scales, [HN] "구현된 주요 기능"; the bit
 * layout is this library's):
 *   MOE_Q_INT4: n/2 bytes; byte j = (q[2j] + 8) | (q[2j+1] + 8) << 4, q in [-8, 7]
 *   MOE_Q_INT2: n/4 bytes; byte j = sum_m (q[4j+m] + 2) << 2m,        q in [-2, 1]
 *   MOE_Q_INT8: n bytes, two's complement,                            q in [-127, 127]
 * Each row r of a matrix has one fp32 scale s[r]; its dequantised value is
 * s[r] * q. */
typedef enum { MOE_Q_INT2 = 2, MOE_Q_INT4 = 4, MOE_Q_INT8 = 8 } moe_qtype;

typedef enum { MOE_OUT_BF16 = 0, MOE_OUT_F32 = 1 } moe_out_dtype;

/* noaux_tc router configuration ([HN] "구현된 주요 기능", router bullet).
 * n_expert (E) routed experts in n_group contiguous groups of E/n_group
 * (at least 2 per group); topk_group groups kept; top_k experts chosen.
 * Limits: E <= 1024, n_group <= 32, top_k <= 32.
 * top_p: adaptive expert top-p ([HN] options list, "--topp 0.7": fewer
 * experts read per token).  When 0 < top_p < 1, of the top_k slots chosen
 * for a token the shortest set of largest unbiased scores s whose sum (fp64,
 * running in that order, ties to the earlier slot) reaches top_p times the
 * sum of all top_k scores (fp64, slot order) is kept; the kept slots keep
 * their slot order and move to the front, the others become empty slots
 * (index -1, weight 0), and the weights are renormalised over the kept slots.
 * Any other value (0, 1, negative, NaN) leaves the routing unchanged. */
typedef struct {
    int n_expert;
    int n_group;
    int topk_group;
    int top_k;
    float routed_scaling_factor;
    float top_p;  /* adaptive expert top-p; any value outside (0, 1) turns it off (0 is the default) */
} moe_router_cfg;

/* A stack of n_expert experts of one shape and qtype, every array contiguous:
 *   w_gate, w_up: [n_expert][inter][hidden*qtype/8] packed codes
 *   w_down:       [n_expert][hidden][inter*qtype/8]
 *   s_gate, s_up: [n_expert][inter] fp32 row scales;  s_down: [n_expert][hidden]
 * hidden and inter must be multiples of 32 (one Q8_0 block);
 * hidden, inter <= 16384.
 * Grouped weight scales ([MO] "int4 양자화 (Quantization)의 품질 비용": grouped
 * scales recover most of int4's quality loss), group_size = G != 0: one fp32
 * scale per row and group of G consecutive codes along the row instead of one
 * per row; G a multiple of 32 that divides hidden and inter; s_gate, s_up:
 * [n_expert][inter][hidden/G]; s_down: [n_expert][hidden][inter/G].  Block b
 * of a row then takes the factor d_b * s[g(b)] (rounded once to fp32) in the
 * fold of the quantised dot and the row has no separate scale.  Batches above
 * the fused kernel's size take the general path with grouped scales, never the
 * tensor-core path (moe_layer_path reports MOE_PATH_GENERAL for them). */
typedef struct {
    int qtype;
    int n_expert;
    int hidden;
    int inter;
    const uint8_t* w_gate;
    const uint8_t* w_up;
    const uint8_t* w_down;
    const float* s_gate;
    const float* s_up;
    const float* s_down;
    int group_size;  /* 0: per-row scales; else grouped scales of group_size codes (above) */
} moe_experts;

/* ------------------------------------------------------------------ route */

/* Bytes of workspace moe_route needs for T tokens. */
size_t moe_route_workspace_bytes(int T, const moe_router_cfg* cfg);

/*
 * Router: steps (1) and (2) of the layer ([HN] "구현된 주요 기능", router
 * bullet: DeepSeek-V3-style sigmoid router, noaux_tc, routed_scaling_factor).
 *   logit[t][e] = sum_h x[t][h] * w_router[e][h], products and sum in fp64,
 *                 rounded once to fp32 (so indices do not depend on the
 *                 summation order)
 *   s = sigmoid(logit) (fp64, rounded once);  b = s + bias[e]  (choice only)
 *   group score = sum of the two largest b of each group; keep topk_group
 *   groups; among their experts keep the top_k largest b; ties go to the lower
 *   index; slot order is descending b.
 *   topk_w[t][k] = s[idx] / sum_k s[idx] * routed_scaling_factor
 *   then adaptive top-p when cfg->top_p is in (0, 1) (see moe_router_cfg)
 * x: [T][H] bf16; w_router: [E][H] fp32; bias: [E] fp32;
 * topk_idx: [T][top_k] int32 out; topk_w: [T][top_k] fp32 out.
 * A token with a NaN score (NaN in x, w_router or bias) gets index -1 (an
 * empty slot, which moe_union leaves out) and weight 0 in every slot, and
 * MOE_EDEVICE_INDEX is recorded in the workspace status word.
 * T = 0 is a no-op.  Errors: MOE_EINVAL, MOE_EWORKSPACE, MOE_ECUDA.
 */
int moe_route(const uint16_t* x, int T, int H, const float* w_router, const float* bias,
              const moe_router_cfg* cfg, int32_t* topk_idx, float* topk_w, void* ws,
              size_t ws_bytes, moe_stream_t stream);

/* Capacity, in fp32 logits (T * n_expert), of moe_route_noalloc's built-in
 * scratch: 65536 logits = 256 KiB of device memory on every GPU that loads
 * the library, held until the process exits. */
#define MOE_ROUTE_NOALLOC_MAX_LOGITS 65536

/*
 * moe_route without a workspace, for callers that cannot allocate device
 * memory when they route: work recorded into a CUDA graph while a stream is
 * being captured, inference-engine plugins whose enqueue step must not
 * allocate, or latency-critical loops that cannot afford cudaMalloc's implicit
 * device synchronisation.  The pages have no counterpart to this call; it is
 * part of this library's interface only.
 *
 * Same arguments and results as moe_route minus ws / ws_bytes.  The logits
 * scratch is a fixed array inside the library (MOE_ROUTE_NOALLOC_MAX_LOGITS
 * floats); batches with T * n_expert above that return MOE_ETOO_LARGE and
 * launch nothing.  The call allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine).
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before capturing a stream on the device.
 *  - Every call in the process shares the one array per device and leaves its
 *    logits there.  Calls whose kernels may overlap on the same device (on
 *    different streams, or from different threads) race on it: order them.
 *  - Unlike moe_route it records no device-side status word; a token with a
 *    NaN score still gets index -1 and weight 0 in every slot.
 */
int moe_route_noalloc(const uint16_t* x, int T, int H, const float* w_router, const float* bias,
                      const moe_router_cfg* cfg, int32_t* topk_idx, float* topk_w,
                      moe_stream_t stream);

/* ------------------------------------------------------------------ union */

/*
 * Batch union: step (3) ([HN] "구현된 주요 기능", batch-union bullet: each
 * distinct expert of a prefill / MTP-verify batch is read once and applied to
 * all positions routed to it).  From topk_idx [T][top_k] (each row distinct):
 *   *n_unique (device int32)  number U of distinct experts
 *   uniq[0..U)                the distinct experts, ascending            ([E])
 *   offsets[0..U]             exclusive prefix sum of their counts       ([E+1])
 *   pair_tok, pair_slot       [T*top_k] (token, slot) pairs grouped by expert
 *                             ascending, tokens ascending within an expert
 *   counts (optional, NULL)   [E] entries per expert (all E, zeros included)
 * Entries of uniq / offsets past U are left unspecified.  An index of -1 is
 * an empty slot (dropped by top-p, or a token the router could not route)
 * and has no pair; any other index outside [0, E), and any repeat of an
 * expert earlier in the same row, is skipped too and recorded as
 * MOE_EDEVICE_INDEX in `status` (optional device int32, not cleared by this
 * call).  The offsets[U] valid pairs come first in pair_tok / pair_slot;
 * the remaining entries of the T*top_k get token 0 and slot -1.  One CTA; no
 * workspace.
 */
int moe_union(const int32_t* topk_idx, int T, int top_k, int E, int32_t* n_unique,
              int32_t* uniq, int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot,
              int32_t* counts, int32_t* status, moe_stream_t stream);

/* ------------------------------------------------------------------- Q8_0 */

/*
 * Q8_0-style quantisation of `rows` rows of n values (n % 32 == 0)
 * ([HN] "구현된 주요 기능", integer-dot bullet: Q8_0-style int8 activations):
 * per block of 32, d = max|v| / 127 (fp32), q = round(v / d) half away from
 * zero, clamped to [-127, 127]; d = 0 gives q = 0.
 * v: [rows][n] bf16 (in_dtype MOE_OUT_BF16) or fp32 (MOE_OUT_F32);
 * q: [rows][n] int8 out; d: [rows][n/32] fp32 out.
 */
int moe_quantize_q8_0(const void* v, int in_dtype, int rows, int n, int8_t* q, float* d,
                      moe_stream_t stream);

/* ------------------------------------------------------------ expert usage */

/*
 * Expert-usage record ([HN] "Learning cache와 하드웨어별 기대치": the engine
 * records which experts routing picks and pins the most used ones in spare
 * RAM; [YO] names the STATS / PIN switches).  usage: [E] uint32 device counts
 * owned by the caller (zero it once; one record per layer); each call adds,
 * for every (token, slot) of topk_idx [T][top_k], one to usage[idx].  Empty
 * slots (-1) and indices outside [0, E) add nothing.  Counts wrap at 2^32.
 * Errors: MOE_EINVAL (sizes, null pointers), MOE_ECUDA.
 */
int moe_usage_accumulate(const int32_t* topk_idx, int T, int top_k, int E, uint32_t* usage,
                         moe_stream_t stream);

/*
 * The pin order of a usage record: order[r] (device int32 [E]) = the expert of
 * rank r, most used first, ties to the lower index.  With every expert of a
 * B200 resident in HBM, this order is what a caller uses to place the hot
 * experts (the pages' pinning) wherever its memory hierarchy rewards it.
 * E <= 1024.  Errors: MOE_EINVAL, MOE_ECUDA.
 */
int moe_usage_rank(const uint32_t* usage, int E, int32_t* order, moe_stream_t stream);

/* ----------------------------------------------------------------- experts */

/* Bytes of workspace moe_expert_ffn_q needs. */
size_t moe_expert_ffn_workspace_bytes(const moe_experts* ex, int T, int top_k);

/*
 * Quantised SwiGLU experts over a batch union: step (4) ([HN] "구현된 주요
 * 기능": int8/packed int4/packed int2 kernels with per-row scales and
 * dequant-on-use, integer dot against Q8_0 activations; batch-union bullet).
 * For every distinct expert u (uniq[u], pairs offsets[u]..offsets[u+1]):
 *   a = Q8_0(x[t]);  g[r] = s_gate[r] * sum_b d_a[b] * isum_b(q_a, q_gate[r]);
 *   u[r] likewise;   h = silu(g) * u;  a' = Q8_0(h);
 *   y[c] = s_down[c] * sum_b d_a'[b] * isum_b(q_a', q_down[c])
 * where isum_b is the exact integer dot of 32-block b, the sum over b is an
 * fp32 accumulator starting at 0 that takes one fused multiply-add per block
 * in ascending b, then one fp32 multiply by the row scale; silu(g) =
 * g / (1 + e^-g) is evaluated in fp64 and rounded once to fp32, and h is the
 * fp32 product silu(g) * u; y_pairs[t][slot][:] = y for each pair (t, slot)
 * of the expert.  The five union arrays are device memory laid out as
 * moe_union writes them for a topk_idx of the same T and top_k; their entries
 * are not range-checked on the device (a token outside [0, T), a slot outside
 * [0, top_k) or an expert outside [0, n_expert) would be read or written out
 * of bounds), so pass lists that moe_union built.
 * Pass n_unique = uniq = offsets = pair_tok = pair_slot = NULL to apply expert
 * 0 of `ex` to every token (the shared expert); top_k must then be 1.
 * x: [T][H] bf16; y_pairs: [T][top_k][H] fp32 out (entries of pairs that are
 * not listed are left untouched).  Errors: MOE_EINVAL, MOE_EUNSUPPORTED
 * (qtype), MOE_EWORKSPACE, MOE_ECUDA.
 */
int moe_expert_ffn_q(const moe_experts* ex, const uint16_t* x, int T, int top_k,
                     const int32_t* n_unique, const int32_t* uniq, const int32_t* offsets,
                     const int32_t* pair_tok, const int32_t* pair_slot, float* y_pairs,
                     void* ws, size_t ws_bytes, moe_stream_t stream);

/* ----------------------------------------------------------------- combine */

/*
 * Weighted combine with the shared expert: step (5) ([HN] router bullet:
 * shared expert; routed_scaling_factor already inside topk_w).
 *   o[t][c] = shared_y[t][c] + sum_k topk_w[t][k] * y_pairs[t][k][c]
 * accumulated in fp32 in slot order, each product and sum rounded separately;
 * a slot whose weight is 0 (an empty slot) adds nothing and its y_pairs row is
 * not read.  out is fp32 or bf16 (round to nearest even).  shared_y may be NULL.
 */
int moe_combine(const float* y_pairs, const float* topk_w, const float* shared_y, int T,
                int top_k, int H, void* out, int out_dtype, moe_stream_t stream);

/* ------------------------------------------------------------------ layer */

/* Bytes of workspace moe_layer_forward needs (a multiple of 256); 0 for a bad
 * router configuration or T < 0.  Only the shape fields of the expert structs
 * are read (not their pointers), so the size can be queried before the
 * weights exist; moe_layer_forward checks the rest. */
size_t moe_layer_workspace_bytes(int T, const moe_router_cfg* cfg, const moe_experts* routed,
                                 const moe_experts* shared);

/*
 * The whole routed-MoE layer, steps (1)-(5): route, union, routed experts,
 * shared expert (weight 1; may be NULL), combine.  x: [T][H] bf16;
 * out: [T][H] bf16 or fp32.  topk_idx_out / topk_w_out (optional, NULL) receive
 * the routing.  routed->n_expert must equal cfg->n_expert; shared (if given)
 * must have the same hidden size and qtype-independent shape rules.
 * Device-side failures (a bounded wait that gave up, a bad index) are recorded
 * in the workspace and read with moe_workspace_status.
 */
int moe_layer_forward(const uint16_t* x, int T, const float* w_router, const float* bias,
                      const moe_router_cfg* cfg, const moe_experts* routed,
                      const moe_experts* shared, void* out, int out_dtype, int32_t* topk_idx_out,
                      float* topk_w_out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Which kernels moe_layer_forward runs for these shapes (host-only query, no
 * launch; this library's own introspection, not a step of the pages' layer):
 *   MOE_PATH_FUSED        one persistent launch for the whole layer (T <= 4,
 *                         T*top_k <= 32, n_expert <= 256 and a multiple of 32,
 *                         groups of a multiple of 32 experts, fits shared memory);
 *   MOE_PATH_TENSOR_CORE  batch-union FFN on tcgen05 tensor cores (T > 32, int4
 *                         with per-row scales, hidden and inter multiples of 64,
 *                         shared expert shaped like the routed ones);
 *   MOE_PATH_GENERAL      router, union, Q8_0, integer-dot expert kernels, combine.
 * Returns one of those or MOE_EINVAL.
 */
#define MOE_PATH_FUSED 1
#define MOE_PATH_TENSOR_CORE 2
#define MOE_PATH_GENERAL 3
int moe_layer_path(int T, const moe_router_cfg* cfg, const moe_experts* routed, const moe_experts* shared);

/*
 * Read (and clear when `clear` != 0) the device status word that kernels of
 * moe_layer_forward / moe_expert_ffn_q record in `ws`.  Synchronises `stream`.
 * *status receives MOE_OK or the first device-side MOE_E* code.  A clear also
 * zeroes the layer's counters (needed after a device-side timeout, which can
 * leave them mid-count); the launch counter is kept.
 */
int moe_workspace_status(void* ws, int clear, int* status, moe_stream_t stream);

/*
 * Test and diagnosis only.  From the next call on `ws` (in stream order), every
 * bounded device-side wait of moe_layer_forward's kernels gives up after at
 * most `polls` polls (0 restores the defaults: about a second for each wait)
 * and records MOE_EDEVICE_TIMEOUT; the kernels then stop issuing work, let
 * the copies already in flight land (those last waits keep their defaults),
 * release what they hold and exit, leaving the output unspecified.  A status
 * clear (moe_workspace_status with `clear` != 0) also restores the defaults.
 * Writes one word of the library-owned header of `ws` on `stream`; returns
 * MOE_OK, MOE_EINVAL (null ws, polls < 0) or MOE_ECUDA.
 */
int moe_workspace_set_wait_limit(void* ws, int polls, moe_stream_t stream);

/* ------------------------------------------------------------ measurement */

/*
 * Kernel timing for benchmarks (no counterpart on the pages).  While enabled,
 * moe_layer_forward records a CUDA event pair on its stream around the
 * layer's dominant work: the fused kernel (small batches), the two
 * tensor-core expert GEMMs taken together (MOE_PATH_TENSOR_CORE), or the
 * up/gate expert kernel (general path); moe_profile_read waits for the
 * recorded events and returns the summed milliseconds and the number of
 * timed regions since the last enable.
 * At most 65536 launches are timed per enable.  moe_launch_count returns the
 * number of kernels this library has launched in the process so far.
 * Host-side state; not thread-safe.
 */
int moe_profile_enable(int on);
int moe_profile_read(double* total_ms, int* launches);
long long moe_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
