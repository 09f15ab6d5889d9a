// Shared device helpers for the DSA kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

constexpr int kWarp = 32;

// ---------------------------------------------------------------- element IO

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float *p, size_t i) { return p[i]; }
    static __device__ __forceinline__ void store(float *p, size_t i, float v) { p[i] = v; }
};
template <> struct Elem<__nv_fp8_e4m3> {  // indexer inputs only: loads
    static __device__ __forceinline__ float load(const __nv_fp8_e4m3 *p, size_t i) {
        return static_cast<float>(p[i]);
    }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p, size_t i) {
        return __bfloat162float(p[i]);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, size_t i, float v) {
        p[i] = __float2bfloat16_rn(v);
    }
};

// Eight bf16 values packed in a 16-byte vector, widened to fp32.
__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float *f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// ---------------------------------------------------------------- warp helpers

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ int warp_inclusive_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// 2^x with the hardware approximation (ex2.approx.ftz: relative error below
// 2^-22, 2^-inf = 0). The softmax loops use it instead of exp2f, whose extra
// range handling measured several times slower in those loops.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------- error words
//
// Each kernel family keeps a device-side error word (a __device__ variable of
// its translation unit) that dsa_device_error reads and clears. Bits:
constexpr unsigned int kErrTimeout = 1u;   // a bounded wait gave up: the launch's outputs are invalid
constexpr unsigned int kErrBadIndex = 2u;  // a selected position outside [0, L) other than -1 was skipped

// Attention kernels: a selected position s that is neither -1 (padding) nor
// inside the cache [0, L) is skipped like padding and reported here.
__device__ __forceinline__ void note_bad_index(unsigned int *word, int s, int L) {
    if (s < -1 || s >= L) atomicOr(word, kErrBadIndex);
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ size_t align_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

}  // namespace dsa
