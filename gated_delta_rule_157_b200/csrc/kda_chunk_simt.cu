// FP32 SIMT chunk-parallel KDA forward (CUDA cores only, exact FP32 FMA).
//
// Chunk form of page "KDA 模块交互式演示" section 1.5 (Eqs. 3-4) with the
// decay-weighted UT transform, per chunk of C tokens and per key channel c,
// with G the in-chunk cumulative sum of the log-decay g:
//
//   A_kk[r,i] = beta_r sum_c k_rc k_ic exp(G_rc - G_ic)   (i <  r)
//   A_qk[r,i] =        sum_c q_rc k_ic exp(G_rc - G_ic)   (i <= r)
//   X         = V - (K*exp(G)) S                          (S = state at chunk start)
//   U         = (I + A_kk)^-1 Diag(beta) X                 (forward substitution)
//   O         = (Q*exp(G)) S + A_qk U
//   S        <- Diag(exp(G_last)) S + (K*exp(G_last - G))^T U
//
// U = Ut - W S of page "Implémenter KDA" ("La forme par blocs") is evaluated
// as T Diag(beta)(V - (K*Gamma) S), which is the same product regrouped.
// Every exponential is taken of a difference G_r - G_i <= 0 (or of G <= 0), so
// nothing overflows for any chunk length.
//
// Parallelisation: one CTA per (b, hv, 32-column slice of the state).  The state
// columns evolve independently, so slices need no communication; the k/q-side
// work (A_kk, A_qk) is repeated per slice.  When M_T is requested the state is
// widened by Dk columns that start from the identity and receive v = 0, which
// carries the cumulative transition (S0' = [S0 | I], V' = [V | 0]).
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kVT = 32;            // state columns per CTA

template <typename Tin>
__global__ void __launch_bounds__(kThreads)
chunk_simt_kernel(ChunkParams p) {
    extern __shared__ float smem[];
    const int C = p.C, Dk = p.Dk, Dv = p.Dv;
    const int L = Dk | 1;                  // padded row stride of the [C][Dk] tiles
    float *Qs = smem;                      // [C][L]  q, then q*exp(G)
    float *Ks = Qs + C * L;                // [C][L]  k, then k*exp(G)
    float *Gs = Ks + C * L;                // [C][L]  g -> G -> k*exp(G_last - G)
    float *Vs = Gs + C * L;                // [C][kVT] v -> X -> U
    float *Akk = Vs + C * kVT;             // [C][C]
    float *Aqk = Akk + C * C;              // [C][C]
    float *Ss = Aqk + C * C;               // [Dk][kVT] state slice
    float *bet = Ss + Dk * kVT;            // [C]
    float *Glast = bet + C;                // [Dk]
    float *red = Glast + Dk;               // [2 * kThreads / 32]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int chain = blockIdx.x;
    const int b = chain / p.HV, hv = chain % p.HV, h = hv / p.group;
    const int col0 = blockIdx.y * kVT;     // first state column of this CTA
    const int ncol_state = Dv;             // columns [0, Dv) are the state, [Dv, Dv+Dk) carry M
    const int ncol = Dv + (p.M_T ? Dk : 0);  // columns that exist in this launch
    const Tin *q = static_cast<const Tin *>(p.q);
    const Tin *k = static_cast<const Tin *>(p.k);
    const Tin *v = static_cast<const Tin *>(p.v);
    const Tin *g = static_cast<const Tin *>(p.g);
    const Tin *bt = static_cast<const Tin *>(p.beta);
    Tin *o = static_cast<Tin *>(p.o);
    const float ea = p.gate_in ? expf(p.A_log[hv]) : 0.f;

    // Initial state slice.
    for (int idx = tid; idx < Dk * kVT; idx += kThreads) {
        int c = idx / kVT, jj = idx % kVT, col = col0 + jj;
        float s = 0.f;
        if (col < ncol_state) {
            if (p.S0) s = p.S0[((size_t)chain * Dk + c) * Dv + col];
        } else if (col < ncol) {
            s = (c == col - ncol_state) ? 1.f : 0.f;
        }
        Ss[idx] = s;
    }

    for (int t0 = 0; t0 < p.T; t0 += C) {
        const int Cc = min(C, p.T - t0);
        __syncthreads();
        if (p.S_chunks) {
            // state entering this chunk (state columns only), for the backward
            const size_t base = ((size_t)chain * ((p.T + C - 1) / C) + t0 / C) * Dk;
            for (int idx = tid; idx < Dk * kVT; idx += kThreads) {
                const int c = idx / kVT, col = col0 + idx % kVT;
                if (col < ncol_state) p.S_chunks[(base + c) * Dv + col] = Ss[idx];
            }
        }
        // ---- load and preprocess the chunk --------------------------------
        for (int idx = tid; idx < Cc * Dk; idx += kThreads) {
            int r = idx / Dk, c = idx % Dk;
            size_t tok = (size_t)b * p.T + t0 + r;
            Qs[r * L + c] = ld_act(q, (tok * p.H + h) * Dk + c);
            Ks[r * L + c] = ld_act(k, (tok * p.H + h) * Dk + c);
            float gz = ld_act(g, gate_index(p.g_per_head, tok, p.HV, hv, Dk, c));
            if (p.gate_in) {
                float bias = p.dt_bias ? p.dt_bias[bias_index(p.g_per_head, hv, Dk, c)] : 0.f;
                gz = kda_gate(p.gate_in, gz, bias, ea, p.g_min);
            }
            Gs[r * L + c] = gz;
        }
        for (int idx = tid; idx < Cc * kVT; idx += kThreads) {
            int r = idx / kVT, jj = idx % kVT, col = col0 + jj;
            size_t tok = (size_t)b * p.T + t0 + r;
            Vs[idx] = (col < ncol_state) ? ld_act(v, (tok * p.HV + hv) * Dv + col) : 0.f;
        }
        for (int r = tid; r < Cc; r += kThreads) {
            float x = ld_act(bt, ((size_t)b * p.T + t0 + r) * p.HV + hv);
            bet[r] = p.beta_sigmoid ? sigmoidf_(x) : x;
        }
        __syncthreads();
        if (p.l2norm) {
            for (int r = warp; r < Cc; r += kThreads / 32) {
                float sq = 0.f, sk = 0.f;
                for (int c = lane; c < Dk; c += 32) {
                    float a = Qs[r * L + c], bb = Ks[r * L + c];
                    sq = fmaf(a, a, sq);
                    sk = fmaf(bb, bb, sk);
                }
                for (int off = 16; off > 0; off >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                }
                float rq = rsqrtf(sq + p.l2_eps), rk = rsqrtf(sk + p.l2_eps);
                for (int c = lane; c < Dk; c += 32) {
                    Qs[r * L + c] *= rq;
                    Ks[r * L + c] *= rk;
                }
            }
        }
        // In-chunk cumulative sum of g per key channel.
        for (int c = tid; c < Dk; c += kThreads) {
            float run = 0.f;
            for (int r = 0; r < Cc; ++r) {
                run += Gs[r * L + c];
                Gs[r * L + c] = run;
            }
            Glast[c] = run;
        }
        __syncthreads();
        // ---- intra-chunk matrices ------------------------------------------
        for (int pidx = tid; pidx < Cc * Cc; pidx += kThreads) {
            int r = pidx / Cc, i = pidx % Cc;
            float akk = 0.f, aqk = 0.f;
            if (i <= r) {
                const float *kr = Ks + r * L, *ki = Ks + i * L, *qr = Qs + r * L;
                const float *gr = Gs + r * L, *gi = Gs + i * L;
                for (int c = 0; c < Dk; ++c) {
                    float e = expf(gr[c] - gi[c]);
                    float kie = ki[c] * e;
                    akk = fmaf(kr[c], kie, akk);
                    aqk = fmaf(qr[c], kie, aqk);
                }
                akk = (i < r) ? bet[r] * akk : 0.f;
            }
            Akk[r * C + i] = akk;
            Aqk[r * C + i] = aqk;
        }
        __syncthreads();
        // ---- decay-weighted operands (in place) ----------------------------
        for (int idx = tid; idx < Cc * Dk; idx += kThreads) {
            int r = idx / Dk, c = idx % Dk, a = r * L + c;
            float G = Gs[a];
            float e = expf(G);
            float kd = Ks[a] * expf(Glast[c] - G);
            Qs[a] *= e;
            Ks[a] *= e;
            Gs[a] = kd;
        }
        __syncthreads();
        // ---- X = V - (K*exp(G)) S ------------------------------------------
        for (int idx = tid; idx < Cc * kVT; idx += kThreads) {
            int r = idx / kVT, jj = idx % kVT;
            float acc = Vs[idx];
            const float *kr = Ks + r * L;
            for (int c = 0; c < Dk; ++c) acc = fmaf(-kr[c], Ss[c * kVT + jj], acc);
            Vs[idx] = acc;
        }
        __syncthreads();
        // ---- U = (I + A_kk)^-1 Diag(beta) X, forward substitution (warp 0) ---
        if (warp == 0) {
            for (int r = 0; r < Cc; ++r) {
                float acc = bet[r] * Vs[r * kVT + lane];
                for (int i = 0; i < r; ++i) acc = fmaf(-Akk[r * C + i], Vs[i * kVT + lane], acc);
                Vs[r * kVT + lane] = acc;
                __syncwarp();
            }
        }
        __syncthreads();
        // ---- O = (Q*exp(G)) S + A_qk U (unless o is not asked for) ---------
        if (o && col0 < ncol_state) {
            for (int idx = tid; idx < Cc * kVT; idx += kThreads) {
                int r = idx / kVT, jj = idx % kVT, col = col0 + jj;
                if (col >= ncol_state) continue;
                float acc = 0.f;
                const float *qr = Qs + r * L;
                for (int c = 0; c < Dk; ++c) acc = fmaf(qr[c], Ss[c * kVT + jj], acc);
                const float *ar = Aqk + r * C;
                for (int i = 0; i <= r; ++i) acc = fmaf(ar[i], Vs[i * kVT + jj], acc);
                size_t tok = (size_t)b * p.T + t0 + r;
                st_act(o, (tok * p.HV + hv) * Dv + col, p.scale * acc);
            }
        }
        __syncthreads();
        // ---- S <- Diag(exp(G_last)) S + (K*exp(G_last - G))^T U --------------
        for (int idx = tid; idx < Dk * kVT; idx += kThreads) {
            int c = idx / kVT, jj = idx % kVT;
            float acc = expf(Glast[c]) * Ss[idx];
            for (int r = 0; r < Cc; ++r) acc = fmaf(Gs[r * L + c], Vs[r * kVT + jj], acc);
            Ss[idx] = acc;
        }
    }
    __syncthreads();
    (void)red;
    for (int idx = tid; idx < Dk * kVT; idx += kThreads) {
        int c = idx / kVT, jj = idx % kVT, col = col0 + jj;
        if (col < ncol_state) {
            if (p.S_T) p.S_T[((size_t)chain * Dk + c) * Dv + col] = Ss[idx];
        } else if (col < ncol) {
            p.M_T[((size_t)chain * Dk + c) * Dk + (col - ncol_state)] = Ss[idx];
        }
    }
}

size_t simt_smem_bytes(int C, int Dk) {
    size_t f = (size_t)3 * C * (Dk | 1) + (size_t)C * kVT + (size_t)2 * C * C + (size_t)Dk * kVT + C +
               Dk + 2 * kThreads / 32;
    return f * sizeof(float);
}

// T == 0: S_T = S0 (or 0), M_T = I.
__global__ void chunk_empty_kernel(ChunkParams p) {
    const size_t n_s = (size_t)p.B * p.HV * p.Dk * p.Dv;
    const size_t n_m = (size_t)p.B * p.HV * p.Dk * p.Dk;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_s + n_m;
         i += (size_t)gridDim.x * blockDim.x) {
        if (i < n_s) {
            if (p.S_T) p.S_T[i] = p.S0 ? p.S0[i] : 0.f;
        } else if (p.M_T) {
            size_t j = i - n_s;
            int c = (int)((j / p.Dk) % p.Dk), m = (int)(j % p.Dk);
            p.M_T[j] = (c == m) ? 1.f : 0.f;
        }
    }
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkParams &p, bool bf16, cudaStream_t s) {
    const int ncol = p.Dv + (p.M_T ? p.Dk : 0);
    dim3 grid(p.B * p.HV, (ncol + kVT - 1) / kVT);
    size_t smem = simt_smem_bytes(p.C, p.Dk);
    cudaError_t e;
    if (bf16) {
        e = cudaFuncSetAttribute(chunk_simt_kernel<__nv_bfloat16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        chunk_simt_kernel<__nv_bfloat16><<<grid, kThreads, smem, s>>>(p);
    } else {
        e = cudaFuncSetAttribute(chunk_simt_kernel<float>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        chunk_simt_kernel<float><<<grid, kThreads, smem, s>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_chunk_empty(const ChunkParams &p, cudaStream_t s) {
    if (!p.S_T && !p.M_T) return cudaSuccess;
    chunk_empty_kernel<<<148 * 4, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace kda
