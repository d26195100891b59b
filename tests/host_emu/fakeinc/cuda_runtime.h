// Host stand-in for the CUDA runtime header: just enough for kernel source to
// compile as C++ and run one CUDA thread per std::thread (see emu_rt.cpp).
#pragma once
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cstring>
#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)
#define __shared__
#define __grid_constant__
#define __align__(n) __attribute__((aligned(n)))
typedef int cudaError_t;
typedef void *cudaStream_t;
enum { cudaSuccess = 0 };
struct uint3 { unsigned x, y, z; };
struct dim3 {
    unsigned x, y, z;
    dim3(unsigned a = 1, unsigned b = 1, unsigned c = 1) : x(a), y(b), z(c) {}
};
extern thread_local uint3 threadIdx, blockIdx;
extern thread_local dim3 blockDim, gridDim;
void __syncthreads();
int __syncthreads_or(int pred);
void __syncwarp(unsigned mask = 0xffffffffu);
float __shfl_xor_sync(unsigned mask, float v, int off);
inline float atomicAdd(float *a, float v) { return std::atomic_ref<float>(*a).fetch_add(v); }
inline float rsqrtf(float x) { return 1.0f / std::sqrt(x); }
inline float __expf(float x) { return std::exp(x); }
inline float __fdividef(float a, float b) { return a / b; }
using std::max;
using std::min;
struct float4 { float x, y, z, w; };
inline float4 make_float4(float x, float y, float z, float w) { return float4{x, y, z, w}; }
inline float4 __ldcs(const float4 *p) { return *p; }
inline void __stcs(float4 *p, float4 v) { *p = v; }
struct uint2 { unsigned x, y; };
inline uint2 make_uint2(unsigned x, unsigned y) { return uint2{x, y}; }
inline float __uint_as_float(unsigned u) { float f; std::memcpy(&f, &u, 4); return f; }
struct uint4 { unsigned x, y, z, w; };
inline uint4 make_uint4(unsigned x, unsigned y, unsigned z, unsigned w) { return uint4{x, y, z, w}; }
struct float2 { float x, y; };
inline float2 make_float2(float x, float y) { return float2{x, y}; }
inline float2 __ffma2_rn(float2 a, float2 b, float2 c) {
    return float2{std::fma(a.x, b.x, c.x), std::fma(a.y, b.y, c.y)};
}
inline float2 __fadd2_rn(float2 a, float2 b) { return float2{a.x + b.x, a.y + b.y}; }
inline float2 __fmul2_rn(float2 a, float2 b) { return float2{a.x * b.x, a.y * b.y}; }
inline unsigned __float_as_uint(float f) { unsigned u; std::memcpy(&u, &f, 4); return u; }
inline unsigned atomicOr(unsigned *a, unsigned v) { return std::atomic_ref<unsigned>(*a).fetch_or(v); }
#include <chrono>
inline long long clock64() {   // a tenth of a nanosecond per "cycle": generous bounds under emulation
    return (long long)std::chrono::steady_clock::now().time_since_epoch().count() / 10;
}
