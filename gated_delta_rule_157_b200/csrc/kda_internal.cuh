// Internal declarations shared by the CUDA translation units of the library.
// Nothing here is part of the C ABI (include/kda.h is).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <cstring>

#include "../../include/kda.h"

namespace kda {

// Element loads/stores for the two activation dtypes.
__device__ __forceinline__ float ld_act(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float ld_act(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st_act(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st_act(__nv_bfloat16 *p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

// 2^x on the special-function unit (PTX ex2.approx, relative error of a few ulp;
// results below the normal range flush to 0); the plain library call on the host.
constexpr float kLog2E = 1.4426950408889634f;
__device__ __forceinline__ float ex2f_(float x) {
#ifdef __CUDA_ARCH__
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
#else
    return exp2f(x);
#endif
}

// Bounded log-decay g = g_min * sigmoid(exp(A_log) * (z + dt_bias)); `ea` is exp(A_log).
__device__ __forceinline__ float bounded_gate(float z, float bias, float ea, float g_min) {
    return g_min * sigmoidf_(ea * (z + bias));
}

// log(1 + e^x) without overflow for large |x|.
__device__ __forceinline__ float softplusf_(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }

// The in-kernel gate, by mode: 1 = bounded (above), 2 = softplus,
// g = -exp(A_log) * softplus(z + dt_bias) (unbounded below).
__device__ __forceinline__ float kda_gate(int mode, float z, float bias, float ea, float g_min) {
    return mode == 2 ? -ea * softplusf_(z + bias) : bounded_gate(z, bias, ea, g_min);
}

// Element offset of the gate input of (token row tok, value head hv, key
// channel c), and of its dt_bias entry: one value per key channel, or one per
// value head shared by the channels (g_per_head).
__device__ __forceinline__ size_t gate_index(int per_head, size_t tok, int HV, int hv, int Dk, int c) {
    return per_head ? tok * HV + hv : (tok * HV + hv) * Dk + c;
}
__device__ __forceinline__ size_t bias_index(int per_head, int hv, int Dk, int c) {
    return per_head ? (size_t)hv : (size_t)hv * Dk + c;
}

// Asynchronous 16-byte global -> shared copy (both addresses 16-byte aligned),
// its commit, and the wait for every committed copy of this thread.
__device__ __forceinline__ void cp_async16(void *dst_smem, const void *src) {
#ifdef __CUDA_ARCH__
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst_smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
#else
    std::memcpy(dst_smem, src, 16);
#endif
}
__device__ __forceinline__ void cp_async_commit() {
#ifdef __CUDA_ARCH__
    asm volatile("cp.async.commit_group;" ::: "memory");
#endif
}
__device__ __forceinline__ void cp_async_wait_all() {
#ifdef __CUDA_ARCH__
    asm volatile("cp.async.wait_all;" ::: "memory");
#endif
}

// Hint: bring the 128-byte line holding p into L2 (no register, no wait).
__device__ __forceinline__ void prefetch_l2(const void *p) {
#ifdef __CUDA_ARCH__
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
#else
    (void)p;
#endif
}

// Validated arguments of a chunked forward, as the kernels see them.
struct ChunkParams {
    int B, T, H, HV, Dk, Dv, C;
    int group;                       // HV / H
    float g_min, scale, l2_eps;
    int l2norm, beta_sigmoid, gate_in;   // gate_in: 0 none, 1 bounded, 2 softplus
    int g_per_head;                      // g / z [B, T, HV], dt_bias [HV]
    const void *q, *k, *v, *g, *beta;
    const float *A_log, *dt_bias, *S0;
    void *o;
    float *S_T, *M_T;
    float *S_chunks;                 // [B, HV, NC, Dk, Dv]: state entering every chunk, or NULL
    int withhold_ready;              // test hook: the tensor-core kernel's prep warps never hand a chunk over
};

// Validated arguments of a chunked backward.
struct BwdParams {
    int B, T, H, HV, Dk, Dv, C;
    int group;                       // HV / H
    float g_min, scale, l2_eps;
    int l2norm, beta_sigmoid, gate_in;
    int g_per_head;
    const void *q, *k, *v, *g, *beta;
    const float *A_log, *dt_bias, *S_chunks;
    const void *dout;
    const float *dS_T;
    float *dq, *dk, *dv, *dg, *dbeta, *dS0, *dA_log, *ddt_bias;
};

struct StepParams {
    int B, H, HV, Dk, Dv, group;
    float g_min, scale, l2_eps;
    int l2norm, beta_sigmoid, gate_in;
    int g_per_head;
    const void *q, *k, *v, *g, *beta;
    const float *A_log, *dt_bias;
    float *S;
    void *o;
};

struct ConvParams {
    int B, T, C, K, head_dim, silu;
    float l2_eps;
    const void *x;
    const float *w, *bias;
    const void *state_in;
    void *y, *state_out;
};

struct GateParams {
    int N, HV, D;
    float eps;
    const void *o, *gate;
    const float *weight;
    void *y;
};

// Launchers (host).  They assume validated arguments and return the launch status.
cudaError_t launch_chunk_simt(const ChunkParams &p, bool bf16, cudaStream_t s);
cudaError_t launch_chunk_tc(const ChunkParams &p, cudaStream_t s);
bool chunk_tc_supported(const ChunkParams &p, bool bf16);
cudaError_t launch_chunk_empty(const ChunkParams &p, cudaStream_t s);   // T == 0
cudaError_t launch_chunk_bwd(const BwdParams &p, bool bf16, cudaStream_t s);
size_t bwd_smem_bytes(int C, int Dk, bool anchored);
cudaError_t launch_step(const StepParams &p, bool bf16, cudaStream_t s);
cudaError_t launch_short_conv(const ConvParams &p, cudaStream_t s);
cudaError_t launch_output_gate(const GateParams &p, cudaStream_t s);
cudaError_t launch_compose(int n_seg, int BH, int Dk, int Dv, const float *M,
                           const float *S_seg, const float *S_init, float *S_in,
                           cudaStream_t s);
// Device error word (set by bounded waits that gave up).  Reads and clears it.
cudaError_t read_and_clear_device_error(cudaStream_t s, unsigned int *out);
// The decode kernels' error word (after the stream has been synchronised).
cudaError_t read_and_clear_step_error(unsigned int *out);
// Layer prologue: bit 0 = a stage wait of the tiled short convolution gave up.
cudaError_t read_and_clear_conv_error(unsigned int *out);

}  // namespace kda
