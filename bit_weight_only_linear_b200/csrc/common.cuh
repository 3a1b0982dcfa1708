// Shared device helpers of the AWQ W4A16 library (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "awq.h"

namespace awq {

// Bits of the device error word: a bounded wait ran out; a dequantised weight of the
// fp16 GEMM path would not be finite in fp16 ((q - zero) * scale16 >= 65520 in magnitude).
constexpr unsigned kErrTimeout = 1u;
constexpr unsigned kErrRange = 2u;

// One error word per device that loads the library.  Kernels OR flags into it;
// awq_device_error() reads and clears it.
__device__ unsigned int g_error_word;

__device__ __forceinline__ void raise_error(unsigned flag) { atomicOr(&g_error_word, flag); }

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Workspace carving: sizes rounded up to 256 bytes.
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Wait limit for every spin in this library: 2 s of wall time.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// ---------------------------------------------------------------------------
// fp16 helpers (bit patterns in, bit patterns out)
// ---------------------------------------------------------------------------

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Largest / smallest of three floats, one instruction each on sm_100 (the three-operand
// forms of max.f32 / min.f32; a NaN operand is ignored as in fmaxf / fminf).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ uint16_t f2h_rn(float f) { return __half_as_ushort(__float2half_rn(f)); }

// Correctly rounded double -> binary16 (one rounding, nearest-even), by the
// PTX conversion instruction.
__device__ __forceinline__ uint16_t d2h_rn(double d) {
    uint16_t h;
    asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(d));
    return h;
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace awq
