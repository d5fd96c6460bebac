/*
 * CPU oracle for the routed-MoE layer -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct C99 restatement of what the layer
 * computes.  Only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg may load it; the GPU library never does, and the two share
 * no code, header, table or helper.
 *
 * Sources (web pages about the colibri engine for GLM-5.2):
 *  [HN]  "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기" (amuse.peoplentools.com)
 *  [MO]  "Colibri: 25GB RAM을 탑재한 노트북에서 744B AI 모델 실행하기" (molayo1419.me)
 *  [YO]  "Colibri: como corre um modelo de 744B parâmetros em uma laptop de
 *         32GB sem GPU, sem BLAS" (yodev.dev)
 * The pages name the steps (DeepSeek-V3-style sigmoid router with noaux_tc,
 * routed_scaling_factor, shared expert, batch-union MoE, int8/int4/int2
 * per-row-scaled weights with dequant-on-use, Q8_0-style int8 activations)
 * but print no formula; each function states the reading it implements.
 *
 * Parity pins: every function here is pinned by a CPU test against an
 * independent fact (hand-worked cases, brute force, exact-integer cases,
 * closed forms, invariants).  One item stays "parity unpinned" by the pages:
 * the GLM-5.2 constants themselves (H=6144, I=2048, 8 groups, topk_group 4,
 * scaling factor 2.5) are a workload choice, not something the pages fix.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Expert set on the host: per-expert pointer tables so that a caller can
 * supply only the experts it needs (NULL elsewhere).
 * w_gate[e], w_up[e]: [I][H*qtype/8] packed codes; w_down[e]: [H][I*qtype/8];
 * s_gate[e], s_up[e]: [I] fp32 row scales; s_down[e]: [H].
 * group != 0 (grouped scales): one scale per row and group of `group`
 * consecutive codes along the row instead: s_gate[e], s_up[e]: [I][H/group],
 * s_down[e]: [H][I/group]. */
typedef struct {
    int qtype; /* 2, 4 or 8 bits per weight */
    int n_expert;
    int H;
    int I;
    const uint8_t* const* w_gate;
    const uint8_t* const* w_up;
    const uint8_t* const* w_down;
    const float* const* s_gate;
    const float* const* s_up;
    const float* const* s_down;
    int group; /* 0: per-row scales; else codes per scale group (a multiple of 32) */
} oracle_experts;

float oracle_bf16_to_f32(uint16_t v);
uint16_t oracle_f32_to_bf16(float f);

/* Router logits, fp64 accumulation rounded once to fp32. */
void oracle_router_logits(const uint16_t* x, int T, int H, const float* w_router, int E,
                          float* logits);

/* noaux_tc selection + renormalised, scaled gate weights from logits. */
int oracle_select(const float* logits, int T, const float* bias, int E, int n_group,
                  int topk_group, int top_k, float rsf, int32_t* topk_idx, float* topk_w,
                  float* gap_expert, float* gap_group);

int oracle_route(const uint16_t* x, int T, int H, const float* w_router, const float* bias,
                 int E, int n_group, int topk_group, int top_k, float rsf, int32_t* topk_idx,
                 float* topk_w, float* gap_expert, float* gap_group);

/* The same with adaptive expert top-p (0 < top_p < 1; any other value: as above). */
int oracle_select_topp(const float* logits, int T, const float* bias, int E, int n_group,
                       int topk_group, int top_k, float rsf, float top_p, int32_t* topk_idx,
                       float* topk_w, float* gap_expert, float* gap_group);

int oracle_route_topp(const uint16_t* x, int T, int H, const float* w_router, const float* bias,
                      int E, int n_group, int topk_group, int top_k, float rsf, float top_p,
                      int32_t* topk_idx, float* topk_w, float* gap_expert, float* gap_group);

int oracle_union(const int32_t* topk_idx, int T, int top_k, int E, int32_t* n_unique,
                 int32_t* uniq, int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot,
                 int32_t* counts);

void oracle_q8_0(const float* v, int n, int8_t* q, float* d);

int oracle_unpack(const uint8_t* packed, int qtype, int n, int8_t* codes);

float oracle_qdot(const int8_t* wcodes, float w_scale, const int8_t* qa, const float* da, int n);

float oracle_qdot_grouped(const int8_t* wcodes, const float* w_scales, int group, const int8_t* qa,
                          const float* da, int n);

int oracle_expert_token(const oracle_experts* ex, int e, const float* x, float* y, float* h_out);

int oracle_expert_ffn(const oracle_experts* ex, const uint16_t* x, int T, int top_k,
                      int n_unique, const int32_t* uniq, const int32_t* offsets,
                      const int32_t* pair_tok, const int32_t* pair_slot, float* y_pairs);

int oracle_expert_ffn_per_token(const oracle_experts* ex, const uint16_t* x, int T, int top_k,
                                const int32_t* topk_idx, float* y_pairs);

void oracle_combine(const float* y_pairs, const float* topk_w, const float* shared_y, int T,
                    int top_k, int H, float* out_f32, uint16_t* out_bf16);

int oracle_layer_forward(const uint16_t* x, int T, const float* w_router, const float* bias,
                         int E, int n_group, int topk_group, int top_k, float rsf,
                         const oracle_experts* routed, const oracle_experts* shared,
                         float* out_f32, uint16_t* out_bf16, int32_t* topk_idx, float* topk_w);

int oracle_layer_forward_topp(const uint16_t* x, int T, const float* w_router, const float* bias,
                              int E, int n_group, int topk_group, int top_k, float rsf, float top_p,
                              const oracle_experts* routed, const oracle_experts* shared,
                              float* out_f32, uint16_t* out_bf16, int32_t* topk_idx, float* topk_w);

#ifdef __cplusplus
}
#endif
#endif
