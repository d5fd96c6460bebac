// Shared device helpers of the B200 MoE library (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <cstddef>

#include "moe.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace moe {

constexpr int kWarp = 32;
constexpr int kQBlock = 32;  // Q8_0 block length

// Every workspace starts with a control header owned by the library: the
// device status word at offset 0, then the fused kernel's self-resetting
// counters, its router score slots and its launch counter.
constexpr size_t kWsHeader = 16384;

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_sum_f32(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max_f32(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// (value desc, index asc) arg-max across a warp; returns the winner to every lane.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (ov > v || (ov == v && oi < i)) {
            v = ov;
            i = oi;
        }
    }
}

// Q8_0 of one 32-block held one value per lane: returns this lane's code and
// writes the block scale to *d (every lane gets it).  d = amax / 127 and
// q = round(v / d) half away from zero, each a single IEEE operation.
__device__ __forceinline__ int8_t q8_0_lane(float v, float* d_out) {
    const float amax = warp_max_f32(fabsf(v));
    const float d = __fdiv_rn(amax, 127.0f);
    *d_out = d;
    if (d == 0.0f) return 0;
    float r = roundf(__fdiv_rn(v, d));
    r = fminf(fmaxf(r, -127.0f), 127.0f);
    return static_cast<int8_t>(r);
}

// silu(g) * u: silu(g) = g / (1 + e^-g) evaluated in fp64 and rounded once to
// fp32 (as the router's sigmoid), then times u in fp32.
__device__ __forceinline__ float swiglu(float g, float u) {
    const double dg = static_cast<double>(g);
    const float silu = __double2float_rn(__ddiv_rn(dg, __dadd_rn(1.0, exp(-dg))));
    return __fmul_rn(silu, u);
}

__device__ __forceinline__ void record_status(int32_t* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

__host__ __device__ constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---------------------------------------------------------------- workspace carving
struct Carver {
    char* base;
    size_t off;
    size_t cap;
    __host__ explicit Carver(void* b, size_t c) : base(static_cast<char*>(b)), off(0), cap(c) {}
    template <typename T>
    __host__ T* take(size_t n) {
        off = align_up(off, 256);
        T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
        off += n * sizeof(T);
        return p;
    }
    __host__ bool fits() const { return off <= cap; }
};

}  // namespace moe
