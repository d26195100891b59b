// KCP segment prefix combine (page "KDA 模块交互式演示" section 1.6; page
// "Implémenter KDA", "Test 3 - le balayage préfixe"):
//
//   S_in[0] = S_init (or 0),  S_in[s+1] = M[s] S_in[s] + S_seg[s]
//
// One CTA per (bh, 32-column slice); the segments are walked in order inside
// the CTA with the running slice in shared memory and M[s] staged through
// shared memory.  FP32 FMA, summation over the inner index in increasing order.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kVT = 32;

__global__ void __launch_bounds__(kThreads)
compose_kernel(int n_seg, int BH, int Dk, int Dv, const float *__restrict__ M,
               const float *__restrict__ S_seg, const float *__restrict__ S_init,
               float *__restrict__ S_in) {
    extern __shared__ float smem[];
    float *prev = smem;                 // [Dk][kVT]
    float *Ms = prev + Dk * kVT;        // [Dk][Dk]
    const int bh = blockIdx.x, col0 = blockIdx.y * kVT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int col = col0 + lane;
    const size_t st = (size_t)Dk * Dv, mt = (size_t)Dk * Dk;

    for (int c = warp; c < Dk; c += kThreads / 32) {
        float x = 0.f;
        if (col < Dv && S_init) x = S_init[bh * st + (size_t)c * Dv + col];
        prev[c * kVT + lane] = x;
        if (col < Dv) S_in[bh * st + (size_t)c * Dv + col] = x;
    }
    for (int s = 0; s < n_seg; ++s) {
        const float *Mg = M + ((size_t)s * BH + bh) * mt;
        __syncthreads();
        for (int i = tid; i < Dk * Dk; i += kThreads) Ms[i] = Mg[i];
        __syncthreads();
        const float *Sg = S_seg + ((size_t)s * BH + bh) * st;
        float *out = S_in + ((size_t)(s + 1) * BH + bh) * st;
        float acc[(128 + kThreads / 32 - 1) / (kThreads / 32)];
        int n = 0;
        for (int c = warp; c < Dk; c += kThreads / 32, ++n) {
            float a = (col < Dv) ? Sg[(size_t)c * Dv + col] : 0.f;
            const float *mr = Ms + c * Dk;
            for (int m = 0; m < Dk; ++m) a = fmaf(mr[m], prev[m * kVT + lane], a);
            acc[n] = a;
        }
        __syncthreads();
        n = 0;
        for (int c = warp; c < Dk; c += kThreads / 32, ++n) {
            prev[c * kVT + lane] = acc[n];
            if (col < Dv) out[(size_t)c * Dv + col] = acc[n];
        }
    }
}

}  // namespace

cudaError_t launch_compose(int n_seg, int BH, int Dk, int Dv, const float *M, const float *S_seg,
                           const float *S_init, float *S_in, cudaStream_t s) {
    dim3 grid(BH, (Dv + kVT - 1) / kVT);
    size_t smem = ((size_t)Dk * kVT + (size_t)Dk * Dk) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(compose_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    compose_kernel<<<grid, kThreads, smem, s>>>(n_seg, BH, Dk, Dv, M, S_seg, S_init, S_in);
    return cudaGetLastError();
}

}  // namespace kda
