// Seeded synthetic-input generator, device twin of synth_host.c.
//
// Test-input infrastructure only: it fills large resident weight sets on the
// GPU (tens of GB) with the same bytes, codes and scales that synth_host.c
// produces on the host, so the CPU oracle can regenerate any expert it needs.
// Holds none of the MoE layer's arithmetic.  The word generator is Vigna's
// splitmix64 mixer used as a counter-based hash; see synth_host.c for the
// definition.  Equality with the host generator is checked by a GPU test.
#include <cstdint>
#include <cstddef>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint64_t mix(uint64_t z) {
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

uint64_t host_mix(uint64_t z) {
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

uint64_t host_key(uint64_t seed, uint64_t stream) { return host_mix(host_mix(seed) ^ stream); }

// Bytes [start, start+n): each thread writes 16 bytes (two words) when the
// range is word-aligned; a generic per-byte path handles the rest.
__global__ void k_bytes_aligned(uint64_t key, uint64_t first_word, size_t n_words, uint64_t* out) {
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (; i < n_words; i += stride) out[i] = mix(key + first_word + i);
}

__global__ void k_bytes_generic(uint64_t key, uint64_t start_byte, size_t n, uint8_t* out) {
    size_t j = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (; j < n; j += stride) {
        const uint64_t b = start_byte + j;
        out[j] = (uint8_t)(mix(key + (b >> 3)) >> (8u * (unsigned)(b & 7u)));
    }
}

__global__ void k_codes_i8(uint64_t key, uint64_t start_code, size_t n, int8_t* out) {
    size_t j = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (; j < n; j += stride) {
        const uint64_t c = start_code + j;
        const uint64_t r = (mix(key + (c >> 1)) >> (32u * (unsigned)(c & 1u))) & 0xFFFFFFFFull;
        out[j] = (int8_t)((int)((r * 255ull) >> 32) - 127);
    }
}

__global__ void k_scales(uint64_t key, uint64_t start, size_t n, float lo, float span, float* out) {
    size_t j = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (; j < n; j += stride) {
        const uint32_t u = (uint32_t)(mix(key + start + j) >> 40);
        const float a = __fmul_rn((float)u, 5.9604644775390625e-08f);
        const float b = __fmul_rn(a, span);
        out[j] = __fadd_rn(b, lo);
    }
}

int grid_for(size_t n) {
    size_t g = (n + 255) / 256;
    if (g > 148 * 32) g = 148 * 32;
    if (g < 1) g = 1;
    return (int)g;
}

}  // namespace

extern "C" {

// All functions: device output pointer, asynchronous on `stream`
// (a cudaStream_t), return cudaError_t of the launch as int.
int synth_gpu_bytes(uint64_t seed, uint64_t stream_id, uint64_t start_byte, size_t n, void* out,
                    void* stream) {
    if (n == 0) return 0;
    const uint64_t key = host_key(seed, stream_id);
    cudaStream_t s = (cudaStream_t)stream;
    if ((start_byte & 7u) == 0 && (n & 7u) == 0 && (((uintptr_t)out) & 7u) == 0) {
        const size_t nw = n >> 3;
        k_bytes_aligned<<<grid_for(nw), 256, 0, s>>>(key, start_byte >> 3, nw, (uint64_t*)out);
    } else {
        k_bytes_generic<<<grid_for(n), 256, 0, s>>>(key, start_byte, n, (uint8_t*)out);
    }
    return (int)cudaGetLastError();
}

int synth_gpu_codes_i8(uint64_t seed, uint64_t stream_id, uint64_t start_code, size_t n, void* out,
                       void* stream) {
    if (n == 0) return 0;
    k_codes_i8<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(host_key(seed, stream_id), start_code,
                                                               n, (int8_t*)out);
    return (int)cudaGetLastError();
}

int synth_gpu_scales(uint64_t seed, uint64_t stream_id, uint64_t start, size_t n, float lo,
                     float span, void* out, void* stream) {
    if (n == 0) return 0;
    k_scales<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(host_key(seed, stream_id), start, n, lo,
                                                             span, (float*)out);
    return (int)cudaGetLastError();
}

}  // extern "C"
