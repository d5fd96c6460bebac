// noaux_tc selection of one token by one warp (internal).
//
// [HN] "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", section "구현된 주요 기능",
// router bullet (DeepSeek-V3-style sigmoid router, noaux_tc,
// routed_scaling_factor).  Reading: s = sigmoid(logit) in fp64 rounded once;
// b = s + bias (for choosing only); group score = sum of the two largest b of
// each contiguous group; keep topk_group groups; choose top_k experts by b
// among kept groups; ties to the lower index; w = s / sum(s) * rsf with the
// sum in slot order.  Adaptive expert top-p (same page, options list:
// "--topp 0.7"), when 0 < top_p < 1: the slots ranked by s (largest first,
// ties to the earlier slot), the shortest prefix whose fp64 running sum
// reaches top_p times the fp64 sum of all K scores is kept, in slot order at
// the front; the other slots become empty (index -1, weight 0) and the
// weights are renormalised over the kept ones.
#pragma once

#include "common.cuh"

namespace moe {

// s, b: this warp's shared-memory scratch of E floats each.  logit(e) returns
// the fp32 logit of expert e.  Lane 0 writes idx[k], w[k] (k < K); chosen
// (shared, >= K ints) receives the indices for every lane.
template <typename LogitFn>
__device__ __forceinline__ void select_token_warp(LogitFn logit, const float* __restrict__ bias,
                                                  int E, int G, int TG, int K, float rsf, float top_p,
                                                  float* s, float* b, int* chosen,
                                                  int32_t* idx, float* w, int32_t* status) {
    const int lane = threadIdx.x & 31;
    bool nan = false;
    for (int e = lane; e < E; e += 32) {
        const double l = static_cast<double>(logit(e));
        const float sv = __double2float_rn(1.0 / (1.0 + exp(-l)));
        s[e] = sv;
        b[e] = __fadd_rn(sv, __ldg(bias + e));
        nan |= b[e] != b[e];
    }
    __syncwarp();
    if (__any_sync(0xffffffffu, nan)) {
        // a NaN score leaves no expert choosable: every slot gets index -1
        // (an empty slot) and weight 0, and the status records it
        record_status(status, MOE_EDEVICE_INDEX);
        for (int k = lane; k < K; k += 32) {
            idx[k] = -1;
            w[k] = 0.0f;
        }
        __syncwarp();
        return;
    }
    const int gsz = E / G;
    float gs = -INFINITY;
    if (lane < G) {
        float v1 = -INFINITY, v2 = -INFINITY;
        for (int e = lane * gsz; e < (lane + 1) * gsz; ++e) {
            const float v = b[e];
            if (v > v1) {
                v2 = v1;
                v1 = v;
            } else if (v > v2) {
                v2 = v;
            }
        }
        gs = __fadd_rn(v1, v2);
    }
    uint32_t keep = 0;
    for (int j = 0; j < TG; ++j) {
        const bool ok = lane < G && !((keep >> lane) & 1u);
        float v = ok ? gs : -INFINITY;
        int i = ok ? lane : 0x7fffffff;
        warp_argmax(v, i);
        if (i >= G) {  // only reachable with NaN scores: no group is kept for this round
            record_status(status, MOE_EDEVICE_INDEX);
            continue;
        }
        keep |= 1u << i;
    }
    for (int k = 0; k < K; ++k) {
        float best = -INFINITY;
        int bi = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            if (!((keep >> (e / gsz)) & 1u)) continue;
            const float v = b[e];
            if (v > best) {  // ascending e within a lane: first of equals wins
                best = v;
                bi = e;
            }
        }
        warp_argmax(best, bi);
        if (bi >= E) {  // only reachable with NaN scores: no expert for this slot
            record_status(status, MOE_EDEVICE_INDEX);
            bi = -1;
        }
        if (lane == 0) {
            chosen[k] = bi;
            if (bi >= 0) b[bi] = -INFINITY;
        }
        __syncwarp();
    }
    if (lane == 0) {
        // adaptive top-p: keep the largest scores until their mass reaches top_p
        uint32_t kept = K >= 32 ? 0xffffffffu : (1u << K) - 1u;
        if (top_p > 0.0f && top_p < 1.0f) {
            double S = 0.0;
            for (int k = 0; k < K; ++k)
                if (chosen[k] >= 0) S += static_cast<double>(s[chosen[k]]);
            const double thr = static_cast<double>(top_p) * S;
            double c = 0.0;
            kept = 0u;
            for (int m = 0; m < K; ++m) {
                int j = -1;  // the largest remaining score, the earlier slot on ties
                for (int k = 0; k < K; ++k)
                    if (!((kept >> k) & 1u) && chosen[k] >= 0 && (j < 0 || s[chosen[k]] > s[chosen[j]])) j = k;
                if (j < 0) break;
                kept |= 1u << j;
                c += static_cast<double>(s[chosen[j]]);
                if (c >= thr) break;
            }
        }
        // a slot left without an expert (NaN scores) or dropped by top-p gets
        // index -1 (an empty slot) and weight 0; kept slots move to the front
        float den = 0.0f;
        for (int k = 0; k < K; ++k)
            if (((kept >> k) & 1u) && chosen[k] >= 0) den = __fadd_rn(den, s[chosen[k]]);
        int j = 0;
        for (int k = 0; k < K; ++k) {
            const int e = chosen[k];
            if (!((kept >> k) & 1u) || e < 0) continue;
            idx[j] = e;
            w[j] = __fmul_rn(__fdiv_rn(s[e], den), rsf);
            ++j;
        }
        for (; j < K; ++j) {
            idx[j] = -1;
            w[j] = 0.0f;
        }
    }
    __syncwarp();
}

}  // namespace moe
