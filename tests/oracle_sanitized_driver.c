/*
 * Runs every entry point of the CPU oracle (oracle/moe_oracle.c) on small
 * seeded inputs.  tests/test_oracle_sanitized.py compiles it together with the
 * oracle under AddressSanitizer and UndefinedBehaviorSanitizer, so an
 * out-of-bounds access, a use after free, a leak or undefined behaviour in the
 * oracle ends the run with an error.  Every buffer is allocated at exactly the
 * size its function documents, so an overrun by one element is caught.
 *
 * So that the run does real work, it also checks two of the oracle's own
 * identities: the batch-union expert pass equals the per-token pass bit for
 * bit, and the layer equals route + union + experts + combine done step by
 * step.  Test infrastructure only.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static unsigned long long g_state = 0x243F6A8885A308D3ull;

/* xorshift64* (Vigna): input values only, no arithmetic of the layer */
static unsigned long long next64(void) {
    g_state ^= g_state >> 12;
    g_state ^= g_state << 25;
    g_state ^= g_state >> 27;
    return g_state * 0x2545F4914F6CDD1Dull;
}

static float uniform(float a, float b) { return a + (b - a) * (float)((next64() >> 40) / 16777216.0); }

static void* xmalloc(size_t n) {
    void* p = malloc(n ? n : 1);
    if (!p) {
        fprintf(stderr, "out of memory\n");
        exit(2);
    }
    return p;
}

static int g_fail = 0;

static void check(int ok, const char* what) {
    if (!ok) {
        fprintf(stderr, "FAILED: %s\n", what);
        g_fail = 1;
    }
}

/* A stack of n experts, each matrix in its own exactly-sized allocation. */
typedef struct {
    oracle_experts ex;
    uint8_t** w[3];
    float** s[3];
} host_experts;

static void make_experts(host_experts* he, int qtype, int n, int H, int I, int group) {
    const int rows[3] = {I, I, H}, cols[3] = {H, H, I};
    for (int m = 0; m < 3; ++m) {
        he->w[m] = (uint8_t**)xmalloc(sizeof(uint8_t*) * (size_t)n);
        he->s[m] = (float**)xmalloc(sizeof(float*) * (size_t)n);
        for (int e = 0; e < n; ++e) {
            const size_t nb = (size_t)rows[m] * cols[m] * qtype / 8;
            const size_t ns = (size_t)rows[m] * (group ? cols[m] / group : 1);
            he->w[m][e] = (uint8_t*)xmalloc(nb);
            he->s[m][e] = (float*)xmalloc(sizeof(float) * ns);
            for (size_t i = 0; i < nb; ++i) {
                uint8_t v = (uint8_t)(next64() >> 56);
                if (qtype == 8 && v == 0x80) v = 0x81; /* int8 codes stay in [-127, 127] */
                he->w[m][e][i] = v;
            }
            for (size_t i = 0; i < ns; ++i) he->s[m][e][i] = uniform(0.01f, 0.05f);
        }
    }
    he->ex.qtype = qtype;
    he->ex.n_expert = n;
    he->ex.H = H;
    he->ex.I = I;
    he->ex.w_gate = (const uint8_t* const*)he->w[0];
    he->ex.w_up = (const uint8_t* const*)he->w[1];
    he->ex.w_down = (const uint8_t* const*)he->w[2];
    he->ex.s_gate = (const float* const*)he->s[0];
    he->ex.s_up = (const float* const*)he->s[1];
    he->ex.s_down = (const float* const*)he->s[2];
    he->ex.group = group;
}

static void free_experts(host_experts* he) {
    for (int m = 0; m < 3; ++m) {
        for (int e = 0; e < he->ex.n_expert; ++e) {
            free(he->w[m][e]);
            free(he->s[m][e]);
        }
        free(he->w[m]);
        free(he->s[m]);
    }
}

static void run_config(int qtype, int group, float top_p) {
    const int T = 5, H = 64, I = 96, E = 16, G = 4, TG = 2, K = 4;
    const float rsf = 2.5f;
    const size_t P = (size_t)T * K;
    uint16_t* x = (uint16_t*)xmalloc(sizeof(uint16_t) * (size_t)T * H);
    float* W = (float*)xmalloc(sizeof(float) * (size_t)E * H);
    float* bias = (float*)xmalloc(sizeof(float) * (size_t)E);
    for (int i = 0; i < T * H; ++i) x[i] = oracle_f32_to_bf16(uniform(-2.0f, 2.0f));
    for (int i = 0; i < E * H; ++i) W[i] = uniform(-0.1f, 0.1f);
    for (int i = 0; i < E; ++i) bias[i] = uniform(-0.1f, 0.1f);
    host_experts routed, shared;
    make_experts(&routed, qtype, E, H, I, group);
    make_experts(&shared, qtype, 1, H, I, group);

    /* router, both ways */
    float* logits = (float*)xmalloc(sizeof(float) * (size_t)T * E);
    int32_t* idx = (int32_t*)xmalloc(sizeof(int32_t) * P);
    float* w = (float*)xmalloc(sizeof(float) * P);
    float* gap_e = (float*)xmalloc(sizeof(float) * (size_t)T);
    float* gap_g = (float*)xmalloc(sizeof(float) * (size_t)T);
    int32_t* idx2 = (int32_t*)xmalloc(sizeof(int32_t) * P);
    float* w2 = (float*)xmalloc(sizeof(float) * P);
    oracle_router_logits(x, T, H, W, E, logits);
    check(oracle_select_topp(logits, T, bias, E, G, TG, K, rsf, top_p, idx, w, gap_e, gap_g) == 0, "select");
    check(oracle_route_topp(x, T, H, W, bias, E, G, TG, K, rsf, top_p, idx2, w2, NULL, NULL) == 0, "route");
    check(memcmp(idx, idx2, sizeof(int32_t) * P) == 0 && memcmp(w, w2, sizeof(float) * P) == 0,
          "route equals logits + select");
    check(oracle_select(logits, T, bias, E, G, TG, K, rsf, idx2, w2, NULL, NULL) == 0, "select, p = 1");
    check(oracle_route(x, T, H, W, bias, E, G, TG, K, rsf, idx2, w2, gap_e, gap_g) == 0, "route, p = 1");

    /* union, experts both ways */
    int32_t nu = -1;
    int32_t* uniq = (int32_t*)xmalloc(sizeof(int32_t) * (size_t)E);
    int32_t* offsets = (int32_t*)xmalloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t* ptok = (int32_t*)xmalloc(sizeof(int32_t) * P);
    int32_t* pslot = (int32_t*)xmalloc(sizeof(int32_t) * P);
    int32_t* counts = (int32_t*)xmalloc(sizeof(int32_t) * (size_t)E);
    check(oracle_union(idx, T, K, E, &nu, uniq, offsets, ptok, pslot, counts) == 0, "union");
    float* y = (float*)calloc(P * H, sizeof(float));
    float* y2 = (float*)calloc(P * H, sizeof(float));
    if (!y || !y2) exit(2);
    check(oracle_expert_ffn(&routed.ex, x, T, K, nu, uniq, offsets, ptok, pslot, y) == 0, "expert ffn");
    check(oracle_expert_ffn_per_token(&routed.ex, x, T, K, idx, y2) == 0, "expert ffn per token");
    check(memcmp(y, y2, sizeof(float) * P * H) == 0, "union pass equals per-token pass");

    /* shared expert, combine, and the layer in one call */
    float* ys = (float*)xmalloc(sizeof(float) * (size_t)T * H);
    float* xt = (float*)xmalloc(sizeof(float) * (size_t)H);
    float* hbuf = (float*)xmalloc(sizeof(float) * (size_t)I);
    for (int t = 0; t < T; ++t) {
        for (int c = 0; c < H; ++c) xt[c] = oracle_bf16_to_f32(x[(size_t)t * H + c]);
        check(oracle_expert_token(&shared.ex, 0, xt, ys + (size_t)t * H, hbuf) == 0, "shared expert");
    }
    float* of = (float*)xmalloc(sizeof(float) * (size_t)T * H);
    uint16_t* ob = (uint16_t*)xmalloc(sizeof(uint16_t) * (size_t)T * H);
    float* of2 = (float*)xmalloc(sizeof(float) * (size_t)T * H);
    uint16_t* ob2 = (uint16_t*)xmalloc(sizeof(uint16_t) * (size_t)T * H);
    oracle_combine(y, w, ys, T, K, H, of, ob);
    check(oracle_layer_forward_topp(x, T, W, bias, E, G, TG, K, rsf, top_p, &routed.ex, &shared.ex, of2, ob2,
                                    idx2, w2) == 0, "layer");
    check(memcmp(of, of2, sizeof(float) * (size_t)T * H) == 0 && memcmp(ob, ob2, sizeof(uint16_t) * (size_t)T * H) == 0,
          "layer equals its steps");
    oracle_combine(y, w, NULL, T, K, H, of, NULL);
    check(oracle_layer_forward_topp(x, T, W, bias, E, G, TG, K, rsf, top_p, &routed.ex, NULL, of2, NULL, idx2,
                                    w2) == 0 && memcmp(of, of2, sizeof(float) * (size_t)T * H) == 0,
          "layer without a shared expert");
    check(oracle_layer_forward(x, 0, W, bias, E, G, TG, K, rsf, &routed.ex, &shared.ex, NULL, NULL, NULL, NULL) == 0,
          "empty batch");

    /* the building blocks on their own */
    int8_t* q = (int8_t*)xmalloc((size_t)I);
    float* d = (float*)xmalloc(sizeof(float) * (size_t)(I / 32));
    int8_t* codes = (int8_t*)xmalloc((size_t)I);
    float* ws = (float*)xmalloc(sizeof(float) * (size_t)(I / 32));
    for (int i = 0; i < I / 32; ++i) ws[i] = uniform(0.01f, 0.05f);
    oracle_q8_0(hbuf, I, q, d);
    check(oracle_unpack(routed.w[2][0], qtype, I, codes) == 0, "unpack");
    const float r1 = oracle_qdot(codes, 0.02f, q, d, I);
    const float r2 = oracle_qdot_grouped(codes, ws, 32, q, d, I);
    check(isfinite(r1) && isfinite(r2), "dots");

    free(q); free(d); free(codes); free(ws);
    free(of); free(ob); free(of2); free(ob2); free(ys); free(xt); free(hbuf);
    free(y); free(y2); free(uniq); free(offsets); free(ptok); free(pslot); free(counts);
    free(logits); free(idx); free(w); free(gap_e); free(gap_g); free(idx2); free(w2);
    free_experts(&routed);
    free_experts(&shared);
    free(x); free(W); free(bias);
}

int main(void) {
    const int qtypes[3] = {2, 4, 8};
    for (int i = 0; i < 3; ++i)
        for (int group = 0; group <= 32; group += 32)
            for (int p = 0; p < 2; ++p) run_config(qtypes[i], group, p ? 0.7f : 1.0f);
    if (g_fail) return 1;
    printf("oracle ran clean\n");
    return 0;
}
