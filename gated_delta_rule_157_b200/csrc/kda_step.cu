// Single-token KDA decode against a resident fp32 state, updated in place.
//
// Per chain (b, hv), with S the Dk x Dv state (page "Implémenter KDA", "La forme
// récurrente de référence"; decay before erase, read after update):
//
//   S' = Diag(alpha) S,  a = S'^T k,  e = v - a,  S'' = S' + beta k e^T,
//   o  = S''^T q = S'^T q + beta (k . q) e
//
// so the state is read once and written once.  The kernel is HBM-bound: one CTA
// per chain, each thread keeps RPT float4 pieces of the state in registers
// between the two reductions (S'^T k and S'^T q) and the write-back, loads and
// stores are 16-byte, coalesced along the value axis, and streaming (.cs) so
// the state does not displace other data in L2.
//
// Thread layout (256 threads): lane l owns value columns 4l..4l+3, warp w owns
// key rows w, w+8, w+16, ...  Cross-warp sums go through shared memory.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float4 f4_fma(float a, float4 x, float4 y) {
    return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}
__device__ __forceinline__ float4 f4_scale(float a, float4 x) {
    return make_float4(a * x.x, a * x.y, a * x.z, a * x.w);
}
__device__ __forceinline__ float4 f4_add(float4 x, float4 y) {
    return make_float4(x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w);
}

template <int RPT, typename Tin>
__global__ void __launch_bounds__(kThreads, 2)
step_kernel(StepParams p) {
    __shared__ float qn[128], kn[128], al[128];
    __shared__ float4 red_a[kWarps][32], red_q[kWarps][32];
    __shared__ float part[kWarps][3];
    __shared__ float scal[4];   // beta, q.k (normalised)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int chain = blockIdx.x;
    const int b = chain / p.HV, hv = chain % p.HV, h = hv / p.group;
    const int Dk = p.Dk, Dv = p.Dv;
    const bool col_ok = 4 * lane < Dv;
    float4 *S4 = reinterpret_cast<float4 *>(p.S + (size_t)chain * Dk * Dv);
    const int dv4 = Dv / 4;

    // Issue the state loads first so their latency overlaps the preprocessing.
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        int c = warp + kWarps * i;
        s[i] = (c < Dk && col_ok) ? __ldcs(S4 + (size_t)c * dv4 + lane) : make_float4(0, 0, 0, 0);
    }

    const Tin *q = static_cast<const Tin *>(p.q);
    const Tin *k = static_cast<const Tin *>(p.k);
    const Tin *g = static_cast<const Tin *>(p.g);
    const Tin *v = static_cast<const Tin *>(p.v);
    const Tin *bt = static_cast<const Tin *>(p.beta);

    // Preprocess q, k, gate: thread c < Dk owns channel c.
    float qc = 0.f, kc = 0.f;
    if (tid < Dk) {
        qc = ld_act(q, ((size_t)b * p.H + h) * Dk + tid);
        kc = ld_act(k, ((size_t)b * p.H + h) * Dk + tid);
        float gz = ld_act(g, gate_index(p.g_per_head, (size_t)b, p.HV, hv, Dk, tid));
        if (p.gate_in) {
            float bias = p.dt_bias ? p.dt_bias[bias_index(p.g_per_head, hv, Dk, tid)] : 0.f;
            gz = kda_gate(p.gate_in, gz, bias, expf(p.A_log[hv]), p.g_min);
        }
        al[tid] = expf(gz);
    }
    float sq = qc * qc, sk = kc * kc, sqk = qc * kc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
        sk += __shfl_xor_sync(0xffffffffu, sk, off);
        sqk += __shfl_xor_sync(0xffffffffu, sqk, off);
    }
    if (lane == 0) {
        part[warp][0] = sq;
        part[warp][1] = sk;
        part[warp][2] = sqk;
    }
    __syncthreads();
    if (tid == 0) {
        float tq = 0.f, tk = 0.f, tqk = 0.f;
        for (int w = 0; w < kWarps; ++w) {
            tq += part[w][0];
            tk += part[w][1];
            tqk += part[w][2];
        }
        float rq = p.l2norm ? rsqrtf(tq + p.l2_eps) : 1.f;
        float rk = p.l2norm ? rsqrtf(tk + p.l2_eps) : 1.f;
        float bb = ld_act(bt, (size_t)b * p.HV + hv);
        scal[0] = p.beta_sigmoid ? sigmoidf_(bb) : bb;
        scal[1] = tqk * rq * rk;
        scal[2] = rq;
        scal[3] = rk;
    }
    __syncthreads();
    if (tid < Dk) {
        qn[tid] = qc * scal[2];
        kn[tid] = kc * scal[3];
    }
    __syncthreads();

    // S' = Diag(alpha) S; partial S'^T k and S'^T q over this thread's rows.
    float4 pa = make_float4(0, 0, 0, 0), pq = make_float4(0, 0, 0, 0);
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        int c = warp + kWarps * i;
        if (c < Dk) {
            s[i] = f4_scale(al[c], s[i]);
            pa = f4_fma(kn[c], s[i], pa);
            pq = f4_fma(qn[c], s[i], pq);
        }
    }
    red_a[warp][lane] = pa;
    red_q[warp][lane] = pq;
    __syncthreads();
    float4 a = red_a[0][lane], pr = red_q[0][lane];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
        a = f4_add(a, red_a[w][lane]);
        pr = f4_add(pr, red_q[w][lane]);
    }
    const float beta = scal[0];
    float4 e = make_float4(0, 0, 0, 0);
    if (col_ok) {
        size_t vo = ((size_t)b * p.HV + hv) * Dv + 4 * lane;
        e = make_float4(ld_act(v, vo) - a.x, ld_act(v, vo + 1) - a.y, ld_act(v, vo + 2) - a.z,
                        ld_act(v, vo + 3) - a.w);
    }
    // S'' = S' + beta k e^T, written back in place.
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        int c = warp + kWarps * i;
        if (c < Dk && col_ok) __stcs(S4 + (size_t)c * dv4 + lane, f4_fma(beta * kn[c], e, s[i]));
    }
    if (warp == 0 && col_ok) {
        float bq = beta * scal[1];
        Tin *o = static_cast<Tin *>(p.o);
        size_t oo = ((size_t)b * p.HV + hv) * Dv + 4 * lane;
        st_act(o, oo + 0, p.scale * fmaf(bq, e.x, pr.x));
        st_act(o, oo + 1, p.scale * fmaf(bq, e.y, pr.y));
        st_act(o, oo + 2, p.scale * fmaf(bq, e.z, pr.z));
        st_act(o, oo + 3, p.scale * fmaf(bq, e.w, pr.w));
    }
}

template <int RPT>
cudaError_t launch_rpt(const StepParams &p, bool bf16, cudaStream_t s) {
    dim3 grid(p.B * p.HV);
    if (bf16)
        step_kernel<RPT, __nv_bfloat16><<<grid, kThreads, 0, s>>>(p);
    else
        step_kernel<RPT, float><<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(const StepParams &p, bool bf16, cudaStream_t s) {
    int rpt = (p.Dk + kWarps - 1) / kWarps;
    if (rpt <= 1) return launch_rpt<1>(p, bf16, s);
    if (rpt <= 2) return launch_rpt<2>(p, bf16, s);
    if (rpt <= 4) return launch_rpt<4>(p, bf16, s);
    if (rpt <= 8) return launch_rpt<8>(p, bf16, s);
    return launch_rpt<16>(p, bf16, s);
}

}  // namespace kda
