/*
 * CPU oracle for the routed-MoE layer -- TEST INFRASTRUCTURE ONLY.
 * See moe_oracle.h for the sources and for who may call this code.
 *
 * Build: gcc -O2 -std=c99 -ffp-contract=off -fopenmp (no fused multiply-add,
 * so every "a * b + c" below is two IEEE roundings, exactly as written).
 *
 * Two compile-time switches build VARIANTS of the oracle, used only to
 * measure how much the layer output depends on roundings the pages leave
 * open (oracle/variant_report.py); the default build defines neither:
 *   ORACLE_SILU_F32    silu(g) = g / (1 + expf(-g)) in fp32 instead of fp64
 *   ORACLE_FOLD_MULADD the block fold acc = acc + isum * d (two roundings)
 *                      instead of one fused multiply-add
 * OpenMP only splits independent output rows / logits across threads; the
 * arithmetic of each row is the single-threaded loop as written.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_EINVAL (-1)
#define ORACLE_ENOMEM (-2)

/* ------------------------------------------------------------------ bf16 */

/* bf16 is the top half of an IEEE binary32; widening is exact. */
float oracle_bf16_to_f32(uint16_t v) {
    uint32_t u = (uint32_t)v << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round-to-nearest-even narrowing of a finite fp32 to bf16. */
uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7F800000u) == 0x7F800000u) /* inf / nan: truncate, keep nan quiet */
        return (uint16_t)((u >> 16) | ((u & 0x007FFFFFu) ? 0x40u : 0u));
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ---------------------------------------------------------------- router */

/*
 * Router logits  l[t][e] = sum_h x[t][h] * W[e][h].
 * [HN] section "구현된 주요 기능", router bullet: a DeepSeek-V3-style sigmoid
 * router.  The pages give no precision; this oracle forms every product in
 * fp64 (a bf16 x fp32 product has at most 8 + 24 significant bits, so it is
 * exact), sums in fp64 in ascending h, and rounds once to fp32.
 */
void oracle_router_logits(const uint16_t* x, int T, int H, const float* w_router, int E,
                          float* logits) {
    long n = (long)T * E;
#pragma omp parallel for schedule(static)
    for (long te = 0; te < n; ++te) {
        const int t = (int)(te / E), e = (int)(te % E);
        const uint16_t* xt = x + (size_t)t * H;
        const float* we = w_router + (size_t)e * H;
        double acc = 0.0;
        for (int h = 0; h < H; ++h) acc += (double)oracle_bf16_to_f32(xt[h]) * (double)we[h];
        logits[te] = (float)acc;
    }
}

/* sigma(l) = 1 / (1 + e^-l), evaluated in fp64 and rounded once to fp32. */
static float sigmoid_f32(float l) { return (float)(1.0 / (1.0 + exp(-(double)l))); }

/*
 * noaux_tc selection and gate weights for each token.
 * [HN] "구현된 주요 기능" (router bullet: noaux_tc, routed_scaling_factor);
 * [YO] "O que está implementado" (same list).  Reading of noaux_tc (the
 * published DeepSeek-V3 routing, which the pages name but do not spell out):
 *   s[e]  = sigmoid(l[e])                       (unbiased affinity)
 *   b[e]  = s[e] + bias[e]                      (bias used for choosing only)
 *   groups: G contiguous blocks of E/G experts; group score = sum of the two
 *           largest b in the group
 *   keep the topk_group best groups (ties: lower group index);
 *   among experts of kept groups only, keep the top_k largest b
 *           (ties: lower expert index); slots in that order
 *   w[k]  = (s[idx[k]] / sum_j s[idx[j]]) * rsf  (sum in slot order)
 * gap_expert[t] (optional) = b of the last chosen expert minus the best b left
 * among kept groups' experts; gap_group[t] = score of the last kept group
 * minus the best score of a dropped group (INFINITY where nothing is left).
 *
 * Adaptive expert top-p ([HN] options list, "--topp 0.7": adaptive expert
 * top-p with 30-40% less expert traffic; the pages name it and give no
 * definition).  Reading, applied when 0 < top_p < 1 (any other value leaves
 * the routing as above): order the K slots by s, largest first (ties: the
 * earlier slot); keep the shortest such prefix whose running sum of s reaches
 * top_p times the sum of all K scores, both sums in fp64 (S in slot order,
 * the running sum in that order); the kept slots stay in slot order at the
 * front, the others become empty (index -1, weight 0); the gate weights are
 * renormalised over the kept slots as above (fp32 sum in slot order).
 */
int oracle_select_topp(const float* logits, int T, const float* bias, int E, int n_group,
                       int topk_group, int top_k, float rsf, float top_p, int32_t* topk_idx,
                       float* topk_w, float* gap_expert, float* gap_group) {
    if (T < 0 || E <= 0 || n_group <= 0 || E % n_group != 0 || E / n_group < 2 ||
        topk_group <= 0 || topk_group > n_group || top_k <= 0 || top_k > 32 ||
        top_k > topk_group * (E / n_group))
        return ORACLE_EINVAL;
    const int gsz = E / n_group;
    float* s = (float*)malloc(sizeof(float) * (size_t)E);
    float* b = (float*)malloc(sizeof(float) * (size_t)E);
    float* gs = (float*)malloc(sizeof(float) * (size_t)n_group);
    char* gkeep = (char*)malloc((size_t)n_group);
    char* taken = (char*)malloc((size_t)E);
    if (!s || !b || !gs || !gkeep || !taken) {
        free(s); free(b); free(gs); free(gkeep); free(taken);
        return ORACLE_ENOMEM;
    }
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        for (int e = 0; e < E; ++e) {
            s[e] = sigmoid_f32(l[e]);
            b[e] = s[e] + bias[e];
        }
        /* group score: two largest b (first = max with lowest index, second =
         * max over the rest) */
        for (int g = 0; g < n_group; ++g) {
            int i1 = g * gsz;
            for (int e = g * gsz + 1; e < (g + 1) * gsz; ++e)
                if (b[e] > b[i1]) i1 = e;
            int i2 = -1;
            for (int e = g * gsz; e < (g + 1) * gsz; ++e) {
                if (e == i1) continue;
                if (i2 < 0 || b[e] > b[i2]) i2 = e;
            }
            gs[g] = b[i1] + b[i2];
        }
        /* keep topk_group groups by repeated arg-max (ties -> lower index) */
        memset(gkeep, 0, (size_t)n_group);
        float last_g = 0.0f;
        for (int j = 0; j < topk_group; ++j) {
            int best = -1;
            for (int g = 0; g < n_group; ++g)
                if (!gkeep[g] && (best < 0 || gs[g] > gs[best])) best = g;
            gkeep[best] = 1;
            last_g = gs[best];
        }
        if (gap_group) {
            float rest = -INFINITY;
            int any = 0;
            for (int g = 0; g < n_group; ++g)
                if (!gkeep[g] && (!any || gs[g] > rest)) { rest = gs[g]; any = 1; }
            gap_group[t] = any ? last_g - rest : INFINITY;
        }
        /* top_k experts among kept groups by repeated arg-max */
        memset(taken, 0, (size_t)E);
        int32_t* idx = topk_idx + (size_t)t * top_k;
        for (int k = 0; k < top_k; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (!gkeep[e / gsz] || taken[e]) continue;
                if (best < 0 || b[e] > b[best]) best = e;
            }
            taken[best] = 1;
            idx[k] = best;
        }
        if (gap_expert) {
            float rest = -INFINITY;
            int any = 0;
            for (int e = 0; e < E; ++e)
                if (gkeep[e / gsz] && !taken[e] && (!any || b[e] > rest)) { rest = b[e]; any = 1; }
            gap_expert[t] = any ? b[idx[top_k - 1]] - rest : INFINITY;
        }
        /* adaptive top-p: drop the lowest-s slots past the mass top_p */
        int kept = top_k;
        if (top_p > 0.0f && top_p < 1.0f) {
            int ord[32];
            for (int k = 0; k < top_k; ++k) {  /* stable insertion sort by s, largest first */
                int m = k;
                while (m > 0 && s[idx[ord[m - 1]]] < s[idx[k]]) { ord[m] = ord[m - 1]; --m; }
                ord[m] = k;
            }
            double S = 0.0;
            for (int k = 0; k < top_k; ++k) S += (double)s[idx[k]];
            const double thr = (double)top_p * S;
            double c = 0.0;
            for (int m = 0; m < top_k; ++m) {
                c += (double)s[idx[ord[m]]];
                if (c >= thr) { kept = m + 1; break; }
            }
            char keep[32] = {0};
            for (int m = 0; m < kept; ++m) keep[ord[m]] = 1;
            int j = 0;
            for (int k = 0; k < top_k; ++k)
                if (keep[k]) idx[j++] = idx[k];
            for (; j < top_k; ++j) idx[j] = -1;
        }
        /* renormalised, scaled gate weights from the unbiased s */
        float den = 0.0f;
        for (int k = 0; k < kept; ++k) den += s[idx[k]];
        float* w = topk_w + (size_t)t * top_k;
        for (int k = 0; k < top_k; ++k) {
            if (k >= kept) { w[k] = 0.0f; continue; }
            float r = s[idx[k]] / den;
            w[k] = r * rsf;
        }
    }
    free(s); free(b); free(gs); free(gkeep); free(taken);
    return 0;
}

int oracle_select(const float* logits, int T, const float* bias, int E, int n_group,
                  int topk_group, int top_k, float rsf, int32_t* topk_idx, float* topk_w,
                  float* gap_expert, float* gap_group) {
    return oracle_select_topp(logits, T, bias, E, n_group, topk_group, top_k, rsf, 0.0f, topk_idx,
                              topk_w, gap_expert, gap_group);
}

int oracle_route_topp(const uint16_t* x, int T, int H, const float* w_router, const float* bias,
                      int E, int n_group, int topk_group, int top_k, float rsf, float top_p,
                      int32_t* topk_idx, float* topk_w, float* gap_expert, float* gap_group) {
    if (T < 0 || H <= 0 || E <= 0) return ORACLE_EINVAL;
    float* logits = (float*)malloc(sizeof(float) * ((size_t)T * E + 1));
    if (!logits) return ORACLE_ENOMEM;
    oracle_router_logits(x, T, H, w_router, E, logits);
    int rc = oracle_select_topp(logits, T, bias, E, n_group, topk_group, top_k, rsf, top_p, topk_idx,
                                topk_w, gap_expert, gap_group);
    free(logits);
    return rc;
}

int oracle_route(const uint16_t* x, int T, int H, const float* w_router, const float* bias,
                 int E, int n_group, int topk_group, int top_k, float rsf, int32_t* topk_idx,
                 float* topk_w, float* gap_expert, float* gap_group) {
    return oracle_route_topp(x, T, H, w_router, bias, E, n_group, topk_group, top_k, rsf, 0.0f,
                             topk_idx, topk_w, gap_expert, gap_group);
}

/* ----------------------------------------------------------------- union */

/*
 * Batch union.  [HN] "구현된 주요 기능", batch-union bullet: in prefill and MTP
 * verification each distinct expert of the batch is read once and applied to
 * every position routed to it.  Lists:
 *   counts[e]   number of (token, slot) entries choosing e   (optional)
 *   uniq[u]     the distinct experts, ascending; *n_unique of them
 *   offsets[u]  exclusive prefix sum of their counts (n_unique + 1 entries)
 *   pairs       (token, slot) entries grouped by expert ascending, tokens
 *               ascending within an expert; slot = the k with idx[t][k] = e
 * An index of -1 is an empty slot (dropped by adaptive top-p, or a token the
 * router could not route) and is left out; any other value outside [0, E)
 * is an error.
 */
int oracle_union(const int32_t* topk_idx, int T, int top_k, int E, int32_t* n_unique,
                 int32_t* uniq, int32_t* offsets, int32_t* pair_tok, int32_t* pair_slot,
                 int32_t* counts) {
    if (T < 0 || top_k <= 0 || E <= 0) return ORACLE_EINVAL;
    int32_t* c = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    if (!c) return ORACLE_ENOMEM;
    for (long i = 0; i < (long)T * top_k; ++i) {
        const int e = topk_idx[i];
        if (e == -1) continue;
        if (e < 0 || e >= E) { free(c); return ORACLE_EINVAL; }
        c[e]++;
    }
    int u = 0, off = 0;
    for (int e = 0; e < E; ++e) {
        if (counts) counts[e] = c[e];
        if (c[e] == 0) continue;
        uniq[u] = e;
        offsets[u] = off;
        off += c[e];
        ++u;
    }
    offsets[u] = off;
    *n_unique = u;
    int p = 0;
    for (int j = 0; j < u; ++j) {
        const int e = uniq[j];
        for (int t = 0; t < T; ++t)
            for (int k = 0; k < top_k; ++k)
                if (topk_idx[(size_t)t * top_k + k] == e) {
                    pair_tok[p] = t;
                    pair_slot[p] = k;
                    ++p;
                }
    }
    free(c);
    return 0;
}

/* ------------------------------------------------------------------ Q8_0 */

/*
 * Q8_0-style activation quantisation.  [HN] "구현된 주요 기능", integer-dot
 * bullet: int8 activations in the Q8_0 style.  Reading: blocks of 32 values,
 * one fp32 scale per block, d = max|v| / 127, q = round(v / d) (IEEE division,
 * round half away from zero), clamped to [-127, 127]; d = 0 gives q = 0.
 */
void oracle_q8_0(const float* v, int n, int8_t* q, float* d) {
    for (int b = 0; b < n / 32; ++b) {
        const float* vb = v + 32 * b;
        float amax = 0.0f;
        for (int i = 0; i < 32; ++i) {
            const float a = fabsf(vb[i]);
            if (a > amax) amax = a;
        }
        const float db = amax / 127.0f;
        d[b] = db;
        for (int i = 0; i < 32; ++i) {
            int8_t qi = 0;
            if (db != 0.0f) {
                float r = roundf(vb[i] / db);
                if (r > 127.0f) r = 127.0f;
                if (r < -127.0f) r = -127.0f;
                qi = (int8_t)r;
            }
            q[32 * b + i] = qi;
        }
    }
}

/* --------------------------------------------------------------- weights */

/*
 * Packed weight codes.  [HN] "구현된 주요 기능", quantisation-kernel bullet
 * (int8, packed int4, packed int2, per-row scales, dequant-on-use).  The pages
 * give no bit layout; the layout read here (row-major, one row per output
 * feature):
 *   int4: byte j holds element 2j in its low nibble and 2j+1 in its high
 *         nibble, offset binary (stored u = q + 8, q in [-8, 7]);
 *   int2: byte j holds element 4j+m in bits 2m..2m+1, stored u = q + 2,
 *         q in [-2, 1];
 *   int8: two's complement, q in [-127, 127].
 */
int oracle_unpack(const uint8_t* packed, int qtype, int n, int8_t* codes) {
    if (qtype == 4) {
        for (int j = 0; j < n / 2; ++j) {
            codes[2 * j] = (int8_t)((packed[j] & 0x0F) - 8);
            codes[2 * j + 1] = (int8_t)((packed[j] >> 4) - 8);
        }
    } else if (qtype == 2) {
        for (int j = 0; j < n / 4; ++j)
            for (int m = 0; m < 4; ++m) codes[4 * j + m] = (int8_t)(((packed[j] >> (2 * m)) & 3) - 2);
    } else if (qtype == 8) {
        for (int j = 0; j < n; ++j) codes[j] = (int8_t)packed[j];
    } else {
        return ORACLE_EINVAL;
    }
    return 0;
}

/*
 * One quantised row dot product: integer dot per 32-block, promoted with the
 * activation block's scale and accumulated in fp32 over blocks in ascending
 * order with one fused multiply-add per block (one rounding), then times the
 * row scale.  [HN] "구현된 주요 기능" (integer-dot kernel with
 * Q8_0 activations; per-row scales, dequant on use).
 */
float oracle_qdot(const int8_t* wcodes, float w_scale, const int8_t* qa, const float* da, int n) {
    float acc = 0.0f;
    for (int b = 0; b < n / 32; ++b) {
        int32_t isum = 0;
        for (int i = 32 * b; i < 32 * b + 32; ++i) isum += (int32_t)qa[i] * (int32_t)wcodes[i];
#ifdef ORACLE_FOLD_MULADD
        acc = acc + (float)isum * da[b];  /* variant: two roundings per block */
#else
        acc = fmaf((float)isum, da[b], acc);  /* one rounding per block */
#endif
    }
    return acc * w_scale;
}

/*
 * The same dot with grouped weight scales: one scale per `group` consecutive
 * codes of the row ([MO] "int4 양자화 (Quantization)의 품질 비용": grouped
 * scales recover most of int4's quality loss; the page gives no layout).
 * Reading: block b's integer dot is scaled by the product of its activation
 * scale and its group's weight scale, d_b * s_w[g(b)] rounded once to fp32,
 * and folded like the per-row dot: one fused multiply-add per block in
 * ascending order; there is no separate row scale.
 */
float oracle_qdot_grouped(const int8_t* wcodes, const float* w_scales, int group, const int8_t* qa,
                          const float* da, int n) {
    float acc = 0.0f;
    for (int b = 0; b < n / 32; ++b) {
        int32_t isum = 0;
        for (int i = 32 * b; i < 32 * b + 32; ++i) isum += (int32_t)qa[i] * (int32_t)wcodes[i];
        const float f = da[b] * w_scales[(32 * b) / group];
#ifdef ORACLE_FOLD_MULADD
        acc = acc + (float)isum * f;
#else
        acc = fmaf((float)isum, f, acc);
#endif
    }
    return acc;
}

/* ---------------------------------------------------------------- expert */

static int row_bytes(int qtype, int n) { return n * qtype / 8; }

/*
 * One expert on one token: Q8_0(x) -> gate and up rows -> SwiGLU ->
 * Q8_0(h) -> down rows.  The SwiGLU is h = silu(g) * u with
 * silu(g) = g / (1 + e^-g), as in GLM-5.2's expert MLP, evaluated in fp64 and
 * rounded once to fp32 (the router's sigmoid is evaluated the same way), then
 * multiplied by u in fp32; h is
 * re-quantised to Q8_0 because the integer-dot kernel runs against Q8_0
 * activations ([HN] "구현된 주요 기능").  The shared expert uses the same
 * function ([HN] router bullet lists the shared expert; [MO] "3단계 메모리
 * 전략" places it with the dense part).
 */
int oracle_expert_token(const oracle_experts* ex, int e, const float* x, float* y, float* h_out) {
    const int H = ex->H, I = ex->I, q = ex->qtype, gs = ex->group;
    if (e < 0 || e >= ex->n_expert || H % 32 || I % 32) return ORACLE_EINVAL;
    if (gs < 0 || (gs && (gs % 32 || H % gs || I % gs))) return ORACLE_EINVAL;
    if (!ex->w_gate[e] || !ex->w_up[e] || !ex->w_down[e] || !ex->s_gate[e] || !ex->s_up[e] ||
        !ex->s_down[e])
        return ORACLE_EINVAL;
    int8_t* qa = (int8_t*)malloc((size_t)H);
    float* da = (float*)malloc(sizeof(float) * (size_t)(H / 32));
    float* h = (float*)malloc(sizeof(float) * (size_t)I);
    int8_t* qh = (int8_t*)malloc((size_t)I);
    float* dh = (float*)malloc(sizeof(float) * (size_t)(I / 32));
    if (!qa || !da || !h || !qh || !dh) {
        free(qa); free(da); free(h); free(qh); free(dh);
        return ORACLE_ENOMEM;
    }
    oracle_q8_0(x, H, qa, da);
    const int rb_in = row_bytes(q, H), rb_out = row_bytes(q, I);
#pragma omp parallel
    {
        int8_t* codes = (int8_t*)malloc((size_t)(H > I ? H : I));
#pragma omp for schedule(static)
        for (int r = 0; r < I; ++r) {
            oracle_unpack(ex->w_gate[e] + (size_t)r * rb_in, q, H, codes);
            const float g = gs ? oracle_qdot_grouped(codes, ex->s_gate[e] + (size_t)r * (H / gs), gs, qa, da, H)
                               : oracle_qdot(codes, ex->s_gate[e][r], qa, da, H);
            oracle_unpack(ex->w_up[e] + (size_t)r * rb_in, q, H, codes);
            const float u = gs ? oracle_qdot_grouped(codes, ex->s_up[e] + (size_t)r * (H / gs), gs, qa, da, H)
                               : oracle_qdot(codes, ex->s_up[e][r], qa, da, H);
#ifdef ORACLE_SILU_F32
            const float silu = g / (1.0f + expf(-g));  /* variant: fp32 throughout */
#else
            const float silu = (float)((double)g / (1.0 + exp(-(double)g)));
#endif
            h[r] = silu * u;
        }
#pragma omp single
        oracle_q8_0(h, I, qh, dh);
#pragma omp for schedule(static)
        for (int c = 0; c < H; ++c) {
            oracle_unpack(ex->w_down[e] + (size_t)c * rb_out, q, I, codes);
            y[c] = gs ? oracle_qdot_grouped(codes, ex->s_down[e] + (size_t)c * (I / gs), gs, qh, dh, I)
                      : oracle_qdot(codes, ex->s_down[e][c], qh, dh, I);
        }
        free(codes);
    }
    if (h_out) memcpy(h_out, h, sizeof(float) * (size_t)I);
    free(qa); free(da); free(h); free(qh); free(dh);
    return 0;
}

static void token_f32(const uint16_t* x, int H, int t, float* out) {
    for (int h = 0; h < H; ++h) out[h] = oracle_bf16_to_f32(x[(size_t)t * H + h]);
}

/*
 * Batch-union expert pass: walk the distinct experts, and for each the
 * (token, slot) pairs routed to it; y_pairs[t][slot][:] = expert(x_t).
 * [HN] "구현된 주요 기능", batch-union bullet.
 */
int oracle_expert_ffn(const oracle_experts* ex, const uint16_t* x, int T, int top_k,
                      int n_unique, const int32_t* uniq, const int32_t* offsets,
                      const int32_t* pair_tok, const int32_t* pair_slot, float* y_pairs) {
    const int H = ex->H;
    float* xt = (float*)malloc(sizeof(float) * (size_t)H);
    if (!xt) return ORACLE_ENOMEM;
    for (int u = 0; u < n_unique; ++u) {
        for (int p = offsets[u]; p < offsets[u + 1]; ++p) {
            const int t = pair_tok[p], k = pair_slot[p];
            if (t < 0 || t >= T || k < 0 || k >= top_k) { free(xt); return ORACLE_EINVAL; }
            token_f32(x, H, t, xt);
            int rc = oracle_expert_token(ex, uniq[u], xt, y_pairs + ((size_t)t * top_k + k) * H, NULL);
            if (rc) { free(xt); return rc; }
        }
    }
    free(xt);
    return 0;
}

/* Per-token expert pass (each token, each of its slots, no union). */
int oracle_expert_ffn_per_token(const oracle_experts* ex, const uint16_t* x, int T, int top_k,
                                const int32_t* topk_idx, float* y_pairs) {
    const int H = ex->H;
    float* xt = (float*)malloc(sizeof(float) * (size_t)H);
    if (!xt) return ORACLE_ENOMEM;
    for (int t = 0; t < T; ++t) {
        token_f32(x, H, t, xt);
        for (int k = 0; k < top_k; ++k) {
            if (topk_idx[(size_t)t * top_k + k] == -1) continue;  /* empty slot */
            int rc = oracle_expert_token(ex, topk_idx[(size_t)t * top_k + k], xt,
                                         y_pairs + ((size_t)t * top_k + k) * H, NULL);
            if (rc) { free(xt); return rc; }
        }
    }
    free(xt);
    return 0;
}

/* ---------------------------------------------------------------- combine */

/*
 * Weighted combine with the shared expert.  [HN] router bullet (shared
 * expert) and the scaling factor: out[t] = shared(x_t) + sum_k w[t][k] * y_k,
 * the shared expert added with weight 1, accumulated in fp32 in slot order
 * starting from the shared output, then narrowed to bf16 (round to nearest
 * even).  shared_y may be NULL (no shared expert).  A slot of weight 0 (an
 * empty slot) adds nothing: its y is not read.
 */
void oracle_combine(const float* y_pairs, const float* topk_w, const float* shared_y, int T,
                    int top_k, int H, float* out_f32, uint16_t* out_bf16) {
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < H; ++c) {
            float o = shared_y ? shared_y[(size_t)t * H + c] : 0.0f;
            for (int k = 0; k < top_k; ++k) {
                const float wk = topk_w[(size_t)t * top_k + k];
                if (wk == 0.0f) continue;
                const float p = wk * y_pairs[((size_t)t * top_k + k) * H + c];
                o = o + p;
            }
            if (out_f32) out_f32[(size_t)t * H + c] = o;
            if (out_bf16) out_bf16[(size_t)t * H + c] = oracle_f32_to_bf16(o);
        }
}

/* ------------------------------------------------------------------ layer */

/* The whole layer: route, union, routed experts, shared expert, combine. */
int oracle_layer_forward_topp(const uint16_t* x, int T, const float* w_router, const float* bias,
                              int E, int n_group, int topk_group, int top_k, float rsf, float top_p,
                              const oracle_experts* routed, const oracle_experts* shared,
                              float* out_f32, uint16_t* out_bf16, int32_t* topk_idx, float* topk_w) {
    const int H = routed->H;
    if (T < 0 || routed->n_expert != E || (shared && (shared->H != H || shared->n_expert < 1)))
        return ORACLE_EINVAL;
    int rc = oracle_route_topp(x, T, H, w_router, bias, E, n_group, topk_group, top_k, rsf, top_p,
                               topk_idx, topk_w, NULL, NULL);
    if (rc) return rc;
    const size_t P = (size_t)T * top_k;
    int32_t* uniq = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int32_t* offsets = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t* ptok = (int32_t*)malloc(sizeof(int32_t) * (P + 1));
    int32_t* pslot = (int32_t*)malloc(sizeof(int32_t) * (P + 1));
    float* y = (float*)malloc(sizeof(float) * (P * H + 1));
    float* ys = shared ? (float*)malloc(sizeof(float) * ((size_t)T * H + 1)) : NULL;
    float* xt = (float*)malloc(sizeof(float) * (size_t)H);
    int32_t nu = 0;
    if (!uniq || !offsets || !ptok || !pslot || !y || (shared && !ys) || !xt) {
        rc = ORACLE_ENOMEM;
        goto done;
    }
    rc = oracle_union(topk_idx, T, top_k, E, &nu, uniq, offsets, ptok, pslot, NULL);
    if (rc) goto done;
    rc = oracle_expert_ffn(routed, x, T, top_k, nu, uniq, offsets, ptok, pslot, y);
    if (rc) goto done;
    if (shared) {
        for (int t = 0; t < T; ++t) {
            token_f32(x, H, t, xt);
            rc = oracle_expert_token(shared, 0, xt, ys + (size_t)t * H, NULL);
            if (rc) goto done;
        }
    }
    oracle_combine(y, topk_w, ys, T, top_k, H, out_f32, out_bf16);
done:
    free(uniq); free(offsets); free(ptok); free(pslot); free(y); free(ys); free(xt);
    return rc;
}

int oracle_layer_forward(const uint16_t* x, int T, const float* w_router, const float* bias,
                         int E, int n_group, int topk_group, int top_k, float rsf,
                         const oracle_experts* routed, const oracle_experts* shared,
                         float* out_f32, uint16_t* out_bf16, int32_t* topk_idx, float* topk_w) {
    return oracle_layer_forward_topp(x, T, w_router, bias, E, n_group, topk_group, top_k, rsf, 0.0f,
                                     routed, shared, out_f32, out_bf16, topk_idx, topk_w);
}
