// KCP segment prefix combine (page "KDA 模块交互式演示" section 1.6; page
// "Implémenter KDA", "Test 3 - le balayage préfixe"):
//
//   S_in[0] = S_init (or 0),  S_in[s+1] = M[s] S_in[s] + S_seg[s]
//
// The columns of the state are independent, the segments are not: one CTA per
// (bh, 8-column slice) walks the segments in order with its slice of the
// running state in shared memory.  Thread (row c, column quad h) computes
// S_in[s+1][c][4h..4h+3] = S_seg[s][c][..] + sum_m M[s][c][m] S_in[s][m][..]:
// its row of M[s] streams from global memory (L2: the CTAs of one bh share
// it), the running slice is read as broadcast float4s.  FP32 FMA, summation
// over the inner index in increasing order.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kVT = 8;                      // state columns per CTA

template <bool kVec>
__global__ void __launch_bounds__(kThreads)
compose_kernel(int n_seg, int BH, int Dk, int Dv, const float *__restrict__ M,
               const float *__restrict__ S_seg, const float *__restrict__ S_init,
               float *__restrict__ S_in) {
    __shared__ __align__(16) float prev[128 * kVT];      // [Dk][kVT]
    const int bh = blockIdx.x, col0 = blockIdx.y * kVT;
    const int tid = threadIdx.x, c = tid >> 1, h = tid & 1;
    const int cb = col0 + 4 * h;                         // first column of this thread
    const bool row = c < Dk;
    const size_t st = (size_t)Dk * Dv, mt = (size_t)Dk * Dk;

    auto ld4 = [&](const float *base) {                  // columns cb .. cb+3 of a row
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (kVec) {
            if (cb < Dv) v = *reinterpret_cast<const float4 *>(base + cb);
        } else {
            if (cb + 0 < Dv) v.x = base[cb + 0];
            if (cb + 1 < Dv) v.y = base[cb + 1];
            if (cb + 2 < Dv) v.z = base[cb + 2];
            if (cb + 3 < Dv) v.w = base[cb + 3];
        }
        return v;
    };
    auto st4 = [&](float *base, float4 v) {
        if (kVec) {
            if (cb < Dv) *reinterpret_cast<float4 *>(base + cb) = v;
        } else {
            if (cb + 0 < Dv) base[cb + 0] = v.x;
            if (cb + 1 < Dv) base[cb + 1] = v.y;
            if (cb + 2 < Dv) base[cb + 2] = v.z;
            if (cb + 3 < Dv) base[cb + 3] = v.w;
        }
    };

    if (row) {
        float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (S_init) x0 = ld4(S_init + bh * st + (size_t)c * Dv);
        *reinterpret_cast<float4 *>(prev + c * kVT + 4 * h) = x0;
        st4(S_in + bh * st + (size_t)c * Dv, x0);
    }
    for (int s = 0; s < n_seg; ++s) {
        __syncthreads();
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row) {
            acc = ld4(S_seg + ((size_t)s * BH + bh) * st + (size_t)c * Dv);
            const float *mr = M + ((size_t)s * BH + bh) * mt + (size_t)c * Dk;
            int m = 0;
            if (kVec) {
                for (; m + 4 <= Dk; m += 4) {
                    const float4 mv = *reinterpret_cast<const float4 *>(mr + m);
                    const float mm[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float4 pv = *reinterpret_cast<const float4 *>(prev + (m + u) * kVT + 4 * h);
                        acc.x = fmaf(mm[u], pv.x, acc.x);
                        acc.y = fmaf(mm[u], pv.y, acc.y);
                        acc.z = fmaf(mm[u], pv.z, acc.z);
                        acc.w = fmaf(mm[u], pv.w, acc.w);
                    }
                }
            }
            for (; m < Dk; ++m) {
                const float mv = mr[m];
                const float4 pv = *reinterpret_cast<const float4 *>(prev + m * kVT + 4 * h);
                acc.x = fmaf(mv, pv.x, acc.x);
                acc.y = fmaf(mv, pv.y, acc.y);
                acc.z = fmaf(mv, pv.z, acc.z);
                acc.w = fmaf(mv, pv.w, acc.w);
            }
        }
        __syncthreads();
        if (row) {
            *reinterpret_cast<float4 *>(prev + c * kVT + 4 * h) = acc;
            st4(S_in + ((size_t)(s + 1) * BH + bh) * st + (size_t)c * Dv, acc);
        }
    }
}

}  // namespace

cudaError_t launch_compose(int n_seg, int BH, int Dk, int Dv, const float *M, const float *S_seg,
                           const float *S_init, float *S_in, cudaStream_t s) {
    const dim3 grid(BH, (Dv + kVT - 1) / kVT);
    // float4 rows need Dk, Dv multiples of 4 and 16-byte aligned buffers
    const bool vec = Dk % 4 == 0 && Dv % 4 == 0 && ((uintptr_t)M | (uintptr_t)S_seg | (uintptr_t)S_init |
                                                    (uintptr_t)S_in) % 16 == 0;
    if (vec) compose_kernel<true><<<grid, kThreads, 0, s>>>(n_seg, BH, Dk, Dv, M, S_seg, S_init, S_in);
    else compose_kernel<false><<<grid, kThreads, 0, s>>>(n_seg, BH, Dk, Dv, M, S_seg, S_init, S_in);
    return cudaGetLastError();
}

}  // namespace kda
