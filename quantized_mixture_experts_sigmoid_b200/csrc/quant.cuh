// Packed-weight block loads and the integer block dot product (internal).
//
// A "block" is 32 consecutive codes of one weight row: one Q8_0 activation
// block.  Its packed bytes are 4*QT long (int2: 8 B, int4: 16 B, int8: 32 B).
// Weight layout (moe.h): int4 byte j = (q[2j]+8) | (q[2j+1]+8) << 4;
// int2 byte j = sum_m (q[4j+m]+2) << 2m; int8 two's complement.
//
// The dot product uses dp4a on the raw offset-binary fields (a nibble 0..15
// or a 2-bit field 0..3 is the same value as a signed byte), so the
// activations are pre-permuted to the order in which a mask-and-shift of a
// weight word presents its fields, and the offset is removed with the block's
// activation sum:  sum q_w * q_a = sum u * q_a - off * sum q_a.
#pragma once

#include "common.cuh"

namespace moe {

template <int QT>
struct WBlock {
    uint32_t w[QT];
};

// Block b of a weight row through the L1 cache (lane-per-row kernels: a lane
// reads its row's consecutive blocks, so the rest of each 32-byte sector is
// reused).
template <int QT>
__device__ __forceinline__ WBlock<QT> load_wblock_l1(const uint8_t* row, int b) {
    WBlock<QT> r;
    if constexpr (QT == 2) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(row + 8 * b));
        r.w[0] = v.x;
        r.w[1] = v.y;
    } else if constexpr (QT == 4) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + 16 * b));
        r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
    } else {
        const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(row + 32 * b));
        const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(row + 32 * b + 16));
        r.w[0] = v0.x; r.w[1] = v0.y; r.w[2] = v0.z; r.w[3] = v0.w;
        r.w[4] = v1.x; r.w[5] = v1.y; r.w[6] = v1.z; r.w[7] = v1.w;
    }
    return r;
}

// Permute 32 activation bytes (natural order, a[i] = byte i of the 8 words)
// into the order matching the weight fields of qtype QT.
template <int QT>
__device__ __forceinline__ void permute_act(const uint32_t a[8], uint32_t o[8]) {
    if constexpr (QT == 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = a[i];
    } else if constexpr (QT == 4) {
        // weight word j holds codes 8j..8j+7; low nibbles give the even codes
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            o[2 * j] = __byte_perm(a[2 * j], a[2 * j + 1], 0x6420);
            o[2 * j + 1] = __byte_perm(a[2 * j], a[2 * j + 1], 0x7531);
        }
    } else {
        // weight word j holds codes 16j..16j+15; field m of byte i is code 16j+4i+m
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint32_t sel = static_cast<uint32_t>(m | ((4 + m) << 4));
                const uint32_t lo = __byte_perm(a[4 * j], a[4 * j + 1], sel);
                const uint32_t hi = __byte_perm(a[4 * j + 2], a[4 * j + 3], sel);
                o[4 * j + m] = __byte_perm(lo, hi, 0x5410);
            }
        }
    }
}

// Exact int32 dot of one block: permuted activation words a[0..7] (as two
// uint4), activation block sum asum.
template <int QT>
__device__ __forceinline__ int block_dot(const WBlock<QT>& w, const uint4& a0, const uint4& a1, int asum) {
    const int a[8] = {static_cast<int>(a0.x), static_cast<int>(a0.y), static_cast<int>(a0.z),
                      static_cast<int>(a0.w), static_cast<int>(a1.x), static_cast<int>(a1.y),
                      static_cast<int>(a1.z), static_cast<int>(a1.w)};
    int acc = 0;
    if constexpr (QT == 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            acc = __dp4a(static_cast<int>(w.w[j] & 0x0F0F0F0Fu), a[2 * j], acc);
            acc = __dp4a(static_cast<int>((w.w[j] >> 4) & 0x0F0F0F0Fu), a[2 * j + 1], acc);
        }
        acc -= 8 * asum;
    } else if constexpr (QT == 2) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
            for (int m = 0; m < 4; ++m)
                acc = __dp4a(static_cast<int>((w.w[j] >> (2 * m)) & 0x03030303u), a[4 * j + m], acc);
        }
        acc -= 2 * asum;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc = __dp4a(static_cast<int>(w.w[i]), a[i], acc);
    }
    return acc;
}

// Stage one Q8_0 row (n = 32*nb codes, natural order) into shared memory:
// planes p0/p1 hold the first/second 16 bytes of each permuted block, sd the
// block scales and ss the block sums.
template <int QT>
__device__ __forceinline__ void stage_act_row(const int8_t* __restrict__ q, const float* __restrict__ d,
                                              int nb, uint4* p0, uint4* p1, float* sd, int32_t* ss,
                                              int tid, int nth) {
    for (int b = tid; b < nb; b += nth) {
        const uint4 lo = *reinterpret_cast<const uint4*>(q + 32 * b);
        const uint4 hi = *reinterpret_cast<const uint4*>(q + 32 * b + 16);
        const uint32_t a[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        uint32_t o[8];
        permute_act<QT>(a, o);
        int s = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) s = __dp4a(static_cast<int>(a[i]), 0x01010101, s);
        p0[b] = make_uint4(o[0], o[1], o[2], o[3]);
        p1[b] = make_uint4(o[4], o[5], o[6], o[7]);
        sd[b] = d[b];
        ss[b] = s;
    }
}

}  // namespace moe
