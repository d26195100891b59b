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
//
// For the Kimi K3 head size (Dk = Dv = 128) a persistent variant, step_bulk_kernel,
// moves each chain's state (64 KB, contiguous) with one bulk copy into a
// three-stage shared-memory ring and back with one bulk store, so that the
// reads of the next chains and the writes of the previous ones are in flight
// while a chain is updated in place in shared memory.
#include "kda_internal.cuh"
#include "tc_ptx.cuh"

namespace kda {

// Error word of the decode kernels (a bounded wait on a bulk copy that gave up).
__device__ unsigned int g_step_error = 0;

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

// ---------------------------------------------------------------------------
// Dk = Dv = 128: persistent CTAs, chains blockIdx.x, blockIdx.x + gridDim.x, ...
// Thread (warp w, lane l) owns value columns 4l..4l+3 of key rows w, w+8, ...
// of the chain in the current stage; q, k, gate, v and beta of the next chain
// are loaded into registers while the current one is computed.
constexpr int kStages = 3;
constexpr uint32_t kStateBytes = 128 * 128 * 4;
// shared memory: the stages, then q, k, alpha [128] each and the partial sums
// (2 KB), the cross-warp sums (2 x [8][32] float4), the mbarriers and the abort flag
constexpr uint32_t BULK_VEC = kStages * kStateBytes;
constexpr uint32_t BULK_RED = BULK_VEC + 2048;
constexpr uint32_t BULK_BAR = BULK_RED + 2 * kWarps * 32 * 16;
constexpr uint32_t BULK_SMEM = BULK_BAR + 64;
constexpr long long kBulkWaitCycles = 4000000000LL;   // about two seconds of SM clock

template <typename Tin>
__global__ void __launch_bounds__(kThreads, 1)
step_bulk_kernel(StepParams p) {
    extern __shared__ __align__(1024) float smem[];
    uint8_t *smem_b = reinterpret_cast<uint8_t *>(smem);
    float *stage0 = smem;
    float *qn = reinterpret_cast<float *>(smem_b + BULK_VEC);                   // [128]
    float *kn = qn + 128, *al = kn + 128;                                       // [128] each
    float *part = al + 128;                                                     // [4][3]
    float4 *red_a = reinterpret_cast<float4 *>(smem_b + BULK_RED);              // [8][32]
    float4 *red_q = red_a + kWarps * 32;                                        // [8][32]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_b + BULK_BAR);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + kStages);
    int last_load[kStages] = {-1, -1, -1};       // iteration of the last state load per stage (thread 0)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nchains = p.B * p.HV;
    const Tin *q = static_cast<const Tin *>(p.q);
    const Tin *k = static_cast<const Tin *>(p.k);
    const Tin *g = static_cast<const Tin *>(p.g);
    const Tin *v = static_cast<const Tin *>(p.v);
    const Tin *bt = static_cast<const Tin *>(p.beta);
    Tin *o = static_cast<Tin *>(p.o);
    const uint32_t sbase = tc::smem_addr(smem_b);
    auto bar = [&](int st) { return tc::smem_addr(bars + st); };
    auto state_of = [&](int chain) { return p.S + (size_t)chain * 128 * 128; };

    if (tid == 0) {
        for (int st = 0; st < kStages; ++st) tc::mbar_init(bar(st), 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    // The first two chains' states.
    if (tid == 0) {
        for (int it = 0; it < 2; ++it) {
            const int chain = blockIdx.x + it * gridDim.x;
            if (chain < nchains) {
                tc::mbar_arrive_expect_tx(bar(it), kStateBytes);
                tc::bulk_load(sbase + it * kStateBytes, state_of(chain), kStateBytes, bar(it));
                last_load[it] = it;
            }
        }
    }
    // Inputs of a chain: thread c < 128 its key channel of q, k and the gate;
    // every thread its value columns and beta.
    float qc = 0.f, kc = 0.f, gz = 0.f, bb = 0.f, vv[4] = {0.f, 0.f, 0.f, 0.f};
    auto load_inputs = [&](int chain) {
        if (chain >= nchains) return;
        const int b = chain / p.HV, hv = chain % p.HV, h = hv / p.group;
        if (tid < 128) {
            qc = ld_act(q, ((size_t)b * p.H + h) * 128 + tid);
            kc = ld_act(k, ((size_t)b * p.H + h) * 128 + tid);
            gz = ld_act(g, gate_index(p.g_per_head, (size_t)b, p.HV, hv, 128, tid));
        }
        const size_t vo = ((size_t)b * p.HV + hv) * 128 + 4 * lane;
#pragma unroll
        for (int u = 0; u < 4; ++u) vv[u] = ld_act(v, vo + u);
        bb = ld_act(bt, (size_t)b * p.HV + hv);
    };
    load_inputs(blockIdx.x);

    int it = 0;
    for (int chain = blockIdx.x; chain < nchains; chain += gridDim.x, ++it) {
        const int st = it % kStages;
        float *S = stage0 + (size_t)st * (kStateBytes / 4);
        const int b = chain / p.HV, hv = chain % p.HV;

        // ---- q, k norms, gate, beta --------------------------------------
        if (tid < 128) {
            float gg = gz;
            if (p.gate_in) {
                const float bias = p.dt_bias ? p.dt_bias[bias_index(p.g_per_head, hv, 128, tid)] : 0.f;
                gg = kda_gate(p.gate_in, gg, bias, expf(p.A_log[hv]), p.g_min);
            }
            al[tid] = expf(gg);
            float sq = qc * qc, sk = kc * kc, sqk = qc * kc;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
                sqk += __shfl_xor_sync(0xffffffffu, sqk, off);
            }
            if (lane == 0) {
                part[3 * warp + 0] = sq;
                part[3 * warp + 1] = sk;
                part[3 * warp + 2] = sqk;
            }
        }
        const float qcur = qc, kcur = kc, bcur = bb;
        const float vcur[4] = {vv[0], vv[1], vv[2], vv[3]};
        __syncthreads();
        float tq = 0.f, tk = 0.f, tqk = 0.f;
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
            tq += part[3 * w4 + 0];
            tk += part[3 * w4 + 1];
            tqk += part[3 * w4 + 2];
        }
        const float rq = p.l2norm ? rsqrtf(tq + p.l2_eps) : 1.f;
        const float rk = p.l2norm ? rsqrtf(tk + p.l2_eps) : 1.f;
        const float beta = p.beta_sigmoid ? sigmoidf_(bcur) : bcur;
        if (tid < 128) {
            qn[tid] = qcur * rq;
            kn[tid] = kcur * rk;
        }
        // the next chain's inputs are in flight while this one is computed
        load_inputs(chain + gridDim.x);

        // ---- this chain's state has landed --------------------------------
        bool ok = tc::mbar_try_wait(bar(st), (uint32_t)((it / kStages) & 1));
        if (!ok) {
            const long long t0 = clock64();
            while (!(ok = tc::mbar_try_wait(bar(st), (uint32_t)((it / kStages) & 1)))) {
                if (*abort_flag || clock64() - t0 > kBulkWaitCycles) break;
            }
        }
        if (!ok) *abort_flag = 1;
        __syncthreads();                        // qn, kn, al visible; abort decided
        if (*abort_flag) break;

        // ---- S' = Diag(alpha) S; partial S'^T k and S'^T q ------------------
        float4 sreg[16];
        float4 pa = make_float4(0, 0, 0, 0), pq = make_float4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int c = warp + kWarps * i;
            sreg[i] = f4_scale(al[c], *reinterpret_cast<const float4 *>(S + c * 128 + 4 * lane));
            pa = f4_fma(kn[c], sreg[i], pa);
            pq = f4_fma(qn[c], sreg[i], pq);
        }
        red_a[warp * 32 + lane] = pa;
        red_q[warp * 32 + lane] = pq;
        __syncthreads();
        float4 a = red_a[lane], pr = red_q[lane];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) {
            a = f4_add(a, red_a[w * 32 + lane]);
            pr = f4_add(pr, red_q[w * 32 + lane]);
        }
        const float4 e = make_float4(vcur[0] - a.x, vcur[1] - a.y, vcur[2] - a.z, vcur[3] - a.w);
        // ---- S'' = S' + beta k e^T, in place; then back to HBM ------------
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int c = warp + kWarps * i;
            *reinterpret_cast<float4 *>(S + c * 128 + 4 * lane) = f4_fma(beta * kn[c], e, sreg[i]);
        }
        if (warp == 0) {
            const float bq = beta * tqk * rq * rk;
            const size_t oo = ((size_t)b * p.HV + hv) * 128 + 4 * lane;
            st_act(o, oo + 0, p.scale * fmaf(bq, e.x, pr.x));
            st_act(o, oo + 1, p.scale * fmaf(bq, e.y, pr.y));
            st_act(o, oo + 2, p.scale * fmaf(bq, e.z, pr.z));
            st_act(o, oo + 3, p.scale * fmaf(bq, e.w, pr.w));
        }
        tc::fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc::bulk_store(state_of(chain), sbase + st * kStateBytes, kStateBytes);
            tc::bulk_commit();
            // the stage of the chain after next: its previous store (one
            // iteration ago) must have left shared memory
            const int nxt = chain + 2 * gridDim.x;
            if (nxt < nchains) {
                tc::bulk_wait_read<1>();
                const int st2 = (it + 2) % kStages;
                tc::mbar_arrive_expect_tx(bar(st2), kStateBytes);
                tc::bulk_load(sbase + st2 * kStateBytes, state_of(nxt), kStateBytes, bar(st2));
                last_load[st2] = it + 2;
            }
        }
    }
    // The bulk stores must finish before the CTA (and its shared memory) is
    // gone; after an abort, so must the loads in flight (bounded).
    if (tid == 0) {
        tc::bulk_wait<0>();
        if (*abort_flag) {
            atomicOr(&g_step_error, 1u);
            for (int st = 0; st < kStages; ++st) {
                if (last_load[st] < 0) continue;
                const uint32_t par = (uint32_t)((last_load[st] / kStages) & 1);
                for (uint32_t i = 0; i < 4000; ++i)
                    if (tc::mbar_try_wait_suspend(bar(st), par, 500000u)) break;
            }
        }
    }
    __syncthreads();
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

static cudaError_t launch_bulk(const StepParams &p, bool bf16, cudaStream_t s) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int nchains = p.B * p.HV;
    const int grid = nchains < sms ? nchains : sms;
    if (bf16) {
        e = cudaFuncSetAttribute(step_bulk_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)BULK_SMEM);
        if (e != cudaSuccess) return e;
        step_bulk_kernel<__nv_bfloat16><<<grid, kThreads, BULK_SMEM, s>>>(p);
    } else {
        e = cudaFuncSetAttribute(step_bulk_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)BULK_SMEM);
        if (e != cudaSuccess) return e;
        step_bulk_kernel<float><<<grid, kThreads, BULK_SMEM, s>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_step(const StepParams &p, bool bf16, cudaStream_t s) {
    // Dk = Dv = 128 (the state rows are 512-byte aligned once S is 16-byte aligned)
    if (p.Dk == 128 && p.Dv == 128 && (reinterpret_cast<uintptr_t>(p.S) & 15) == 0) return launch_bulk(p, bf16, s);
    int rpt = (p.Dk + kWarps - 1) / kWarps;
    if (rpt <= 1) return launch_rpt<1>(p, bf16, s);
    if (rpt <= 2) return launch_rpt<2>(p, bf16, s);
    if (rpt <= 4) return launch_rpt<4>(p, bf16, s);
    if (rpt <= 8) return launch_rpt<8>(p, bf16, s);
    return launch_rpt<16>(p, bf16, s);
}

cudaError_t read_and_clear_step_error(unsigned int *out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_step_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_step_error, &zero, sizeof(unsigned int));
}

}  // namespace kda
