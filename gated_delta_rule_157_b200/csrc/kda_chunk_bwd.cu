// FP32 SIMT chunk-parallel KDA backward (CUDA cores only).
//
// The gradient of <dO, O> + <dS_T, S_T> through the chunk form of the forward
// (page "KDA 模块交互式演示" section 1.5, with the decay-weighted UT transform;
// page "Implémenter KDA", "La forme par blocs"), chunk by chunk in reverse.
// The pages print no backward; every line below is the derivative of one line
// of the forward.  Per chunk, with S the state entering it (written by the
// forward), G the in-chunk cumulative sum of the log-decay and
// E_c(r, i) = exp(G_rc - G_ic) (r >= i, so every exponential is of a value <= 0):
//
//   forward (recomputed)
//     A[r,i] = sum_c q_rc k_ic E_c(r,i)  (i <= r)    P[r,i] = sum_c k_rc k_ic E_c(r,i)  (i < r)
//     X = V - (K*exp(G)) S,   U = (I + Diag(beta) P)^-1 Diag(beta) X
//     O = scale ((Q*exp(G)) S + A U),   S' = Diag(exp(G_last)) S + (K*exp(G_last - G))^T U
//   reverse, given dO (scaled) and dS' (gradient of the state leaving the chunk)
//     dU  = A^T dO + (K*exp(G_last - G)) dS'
//     dZ  = (I + Diag(beta) P)^-T dU                 (back substitution)
//     dX  = Diag(beta) dZ = dV
//     dA  = tril(dO U^T),  dP = Diag(beta) tril(-dZ U^T, -1)
//     dbeta_r = sum_j dZ_rj X_rj + sum_i (-dZ U^T)[r,i] P[r,i]
//     dS  = (Q*exp(G))^T dO + Diag(exp(G_last)) dS' - (K*exp(G))^T dX
//   and, per (r, c), the q/k/G gradients of the pairwise sums A and P and of the
//   elementwise factors exp(G), exp(G_last - G), exp(G_last); dg is the reverse
//   in-chunk cumulative sum of dG.
//
// Parallelisation as the SIMT forward: one CTA per (b, hv, 32-column slice of
// the value channels).  dV, dS are per column; the q/k/g/beta gradients sum over
// the columns (and over the value heads of a q/k head), so each CTA adds its
// share with atomics into zeroed fp32 outputs (with one decay per head, dg also
// sums over the key channels).  A second pair of kernels takes them through
// the in-kernel L2 norm, beta sigmoid and gate (bounded or softplus).
#include "kda_internal.cuh"
#include "tc_ptx.cuh"

namespace kda {
namespace {

constexpr int kThreads = 512;                 // chunk_bwd_kernel: 16 warps, one CTA per SM
constexpr int kRowThreads = 256;              // bwd_l2norm_kernel
constexpr int kVT = 32;                       // value columns per CTA
static_assert(kVT == 32, "the row loops map one lane to one value column");
static_assert(kThreads == 4 * 128, "the dS step maps a thread to (key channel, eight value columns)");
constexpr int kElemsPerThread = 64 * 128 / kThreads;   // (r, c) elements of a chunk per thread
constexpr int kLoadBatch = 8;                 // global loads in flight per thread in the chunk load

// fp32 product on the tensor cores at fp32-level accuracy: each operand split
// into a tf32 head and a tf32 tail (x = hi + lo, both exact in tf32 up to the
// tail's rounding), and D += A_lo B_hi + A_hi B_lo + A_hi B_hi (the lo x lo
// term is below fp32 resolution).
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    hi = tc::to_tf32(x);
    lo = tc::to_tf32(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma3_tf32(float d[4], const uint32_t ah[4], const uint32_t al[4], const uint32_t bh[2],
                                          const uint32_t bl[2]) {
    tc::mma_tf32_16x8x8(d, al, bh);
    tc::mma_tf32_16x8x8(d, ah, bl);
    tc::mma_tf32_16x8x8(d, ah, bh);
}

// kAnchored (Dk = 128, C = 64, the bounded gate with |g_min| <= 5): the
// pairwise sums A and P (step 3) and their gradients (step 8) use the
// forward's 16-token tile anchors, so every factor 2^(G_r - G_i) is a product
// of one per-row and one per-column power, each in [2^-116, 2^116] (16 tokens
// x 5 x log2 e); otherwise every pair takes its own power of a non-positive
// difference (any gate).
template <typename Tin, bool kAnchored>
__global__ void __launch_bounds__(kThreads)
chunk_bwd_kernel(BwdParams p) {
    extern __shared__ float smem[];
    // the anchored shape is fixed (C = 64, Dk = 128): every tile offset and
    // stride below is then a compile-time constant
    const int C = kAnchored ? 64 : p.C, Dk = kAnchored ? 128 : p.Dk, Dv = p.Dv;
    const int L = Dk | 1;                  // padded row stride of the [C][Dk] tiles
    // every array starts on a 16-byte boundary (packed float2 / float4 loads)
    const int CL = (C * L + 3) & ~3, CC = (C * C + 3) & ~3;
    float *Qs = smem;                      // [C][L]  q (normalised)
    float *Ks = Qs + CL;                   // [C][L]  k (normalised)
    float *Gs = Ks + CL;                   // [C][L]  G, then dG
    float *Aqk = Gs + CL;                  // [C][C]  A, then dA
    float *Pkk = Aqk + CC;                 // [C][C]  P, then dP
    float *Xs = Pkk + CC;                  // [C][kVT] X
    float *Us = Xs + C * kVT;              // [C][kVT] U
    float *dOs = Us + C * kVT;             // [C][kVT] scale * dO
    float *dUs = dOs + C * kVT;            // [C][kVT] dU, then dZ
    // the state and its gradient transposed, [kVT][SL]: value column j major,
    // key channels contiguous (SL = 4 mod 32: lane = j reads four channels
    // as one conflict-free float4; lane = c reads one row without conflicts)
    const int C4 = (C + 3) & ~3, Dk4 = (Dk + 3) & ~3, SL = Dk4 + 4;
    float *Ss = dUs + C * kVT;             // [kVT][SL] state entering the chunk (transposed)
    float *dSs = Ss + kVT * SL;            // [kVT][SL] dS of the state leaving, then entering, the chunk
    float *bet = dSs + kVT * SL;           // [C]
    float *dbet = bet + C4;                // [C]
    float *Glast = dbet + C4;              // [Dk]
    float *dlast = Glast + Dk4;            // [Dk]  dG terms of the chunk's last row
    // per-warp row of factors, computed once per row and read by all 32 lanes
    // (one lane per value column): [warp][2 * 128]
    float *wb = dlast + Dk4 + (threadIdx.x >> 5) * 256;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int chain = blockIdx.x;
    const int b = chain / p.HV, hv = chain % p.HV, h = hv / p.group;
    const int col0 = blockIdx.y * kVT;
    const int NC = (p.T + C - 1) / C;
    const Tin *q = static_cast<const Tin *>(p.q);
    const Tin *k = static_cast<const Tin *>(p.k);
    const Tin *v = static_cast<const Tin *>(p.v);
    const Tin *g = static_cast<const Tin *>(p.g);
    const Tin *bt = static_cast<const Tin *>(p.beta);
    const Tin *dout = static_cast<const Tin *>(p.dout);
    const float ea = p.gate_in ? expf(p.A_log[hv]) : 0.f;

    for (int idx = tid; idx < Dk * kVT; idx += kThreads) {
        const int c = idx / kVT, col = col0 + idx % kVT;
        dSs[(idx % kVT) * SL + c] = (p.dS_T && col < Dv) ? p.dS_T[((size_t)chain * Dk + c) * Dv + col] : 0.f;
    }

    // Anchored shape with bf16 inputs, one decay per key channel and 16-byte
    // aligned rows: the raw q, k, g rows of chunk ch - 1 are copied into the A,
    // P, X and U tiles (free after step 8 of chunk ch) by asynchronous copies
    // that run during steps 9 and 10.
    const bool can_stage = kAnchored && sizeof(Tin) == 2 && !p.g_per_head &&
                           ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                             reinterpret_cast<uintptr_t>(g)) & 15) == 0;
    const __nv_bfloat16 *raw = reinterpret_cast<const __nv_bfloat16 *>(Aqk);   // [3][C][Dk] q, k, g

    for (int ch = NC - 1; ch >= 0; --ch) {
        const int t0 = ch * C;
        const int Cc = min(C, p.T - t0);
        const size_t tok0 = (size_t)b * p.T + t0;
        const bool staged = can_stage && ch < NC - 1;
        if (staged) cp_async_wait_all();
        __syncthreads();
        // ---- 1. load the chunk and the state entering it -------------------
        // (the state and value rows in batches of kLoadBatch elements per
        // thread whose loads are all issued before the first shared-memory store)
        if (staged) {
            // full chunk (only the last chunk can be ragged, and it is never staged)
            const int c = tid & 127;
            const float bias = (p.gate_in && p.dt_bias) ? p.dt_bias[bias_index(0, hv, 128, c)] : 0.f;
#pragma unroll 4
            for (int r = tid >> 7; r < C; r += kThreads / 128) {
                const float gz = __bfloat162float(raw[(2 * C + r) * Dk + c]);
                Qs[r * L + c] = __bfloat162float(raw[r * Dk + c]);
                Ks[r * L + c] = __bfloat162float(raw[(C + r) * Dk + c]);
                Gs[r * L + c] = p.gate_in ? kda_gate(p.gate_in, gz, bias, ea, p.g_min) : gz;
            }
        } else for (int idx = tid; idx < Cc * Dk; idx += kThreads) {
            const int r = idx / Dk, c = idx % Dk;
            const size_t tok = tok0 + r;
            Qs[r * L + c] = ld_act(q, (tok * p.H + h) * Dk + c);
            Ks[r * L + c] = ld_act(k, (tok * p.H + h) * Dk + c);
            float gz = ld_act(g, gate_index(p.g_per_head, tok, p.HV, hv, Dk, c));
            if (p.gate_in) {
                const float bias = p.dt_bias ? p.dt_bias[bias_index(p.g_per_head, hv, Dk, c)] : 0.f;
                gz = kda_gate(p.gate_in, gz, bias, ea, p.g_min);
            }
            Gs[r * L + c] = gz;
        }
        for (int base = tid; base < Dk * kVT; base += kLoadBatch * kThreads) {
            float sv[kLoadBatch];
#pragma unroll
            for (int u = 0; u < kLoadBatch; ++u) {
                const int idx = base + u * kThreads, c = idx / kVT, col = col0 + idx % kVT;
                sv[u] = (idx < Dk * kVT && col < Dv) ? p.S_chunks[(((size_t)chain * NC + ch) * Dk + c) * Dv + col] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kLoadBatch; ++u) {
                const int idx = base + u * kThreads;
                if (idx < Dk * kVT) Ss[(idx % kVT) * SL + idx / kVT] = sv[u];
            }
        }
        if (staged) __syncthreads();       // the staged g rows lie under X, written next
        for (int base = tid; base < Cc * kVT; base += (kLoadBatch / 2) * kThreads) {
            float vv[kLoadBatch / 2], ov[kLoadBatch / 2];
#pragma unroll
            for (int u = 0; u < kLoadBatch / 2; ++u) {
                const int idx = base + u * kThreads, r = idx / kVT, col = col0 + idx % kVT;
                const bool in = idx < Cc * kVT && col < Dv;
                const size_t tok = tok0 + r;
                vv[u] = in ? ld_act(v, (tok * p.HV + hv) * Dv + col) : 0.f;
                ov[u] = in ? p.scale * ld_act(dout, (tok * p.HV + hv) * Dv + col) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kLoadBatch / 2; ++u) {
                const int idx = base + u * kThreads;
                if (idx < Cc * kVT) {
                    Xs[idx] = vv[u];
                    dOs[idx] = ov[u];
                }
            }
        }
        for (int r = tid; r < Cc; r += kThreads) {
            const float x = ld_act(bt, (tok0 + r) * p.HV + hv);
            bet[r] = p.beta_sigmoid ? sigmoidf_(x) : x;
            dbet[r] = 0.f;
        }
        // the next chunk's (ch - 1) rows into L2 while this one is worked on
        if (ch > 0) {
            const size_t ptok = tok0 - C;
            const int qlines = (Dk * (int)sizeof(Tin) + 127) / 128;
            for (int e = tid; e < C * qlines; e += kThreads) {
                const size_t off = ((ptok + e / qlines) * p.H + h) * Dk * sizeof(Tin) + (size_t)(e % qlines) * 128;
                prefetch_l2(reinterpret_cast<const char *>(q) + off);
                prefetch_l2(reinterpret_cast<const char *>(k) + off);
                if (!p.g_per_head)
                    prefetch_l2(reinterpret_cast<const char *>(g) + ((ptok + e / qlines) * p.HV + hv) * Dk * sizeof(Tin) +
                                (size_t)(e % qlines) * 128);
            }
            for (int e = tid; e < 2 * C + Dk; e += kThreads) {
                if (e < C) {
                    prefetch_l2(v + ((ptok + e) * p.HV + hv) * Dv + col0);
                } else if (e < 2 * C) {
                    prefetch_l2(dout + ((ptok + e - C) * p.HV + hv) * Dv + col0);
                } else {
                    prefetch_l2(p.S_chunks + (((size_t)chain * NC + ch - 1) * Dk + (e - 2 * C)) * Dv + col0);
                }
            }
        }
        __syncthreads();
        // ---- 2. L2 norms of q, k rows; in-chunk cumulative sum of g ----------
        if (p.l2norm) {
            for (int r = warp; r < Cc; r += kThreads / 32) {
                float sq = 0.f, sk = 0.f;
                for (int c = lane; c < Dk; c += 32) {
                    const float a = Qs[r * L + c], bb = Ks[r * L + c];
                    sq = fmaf(a, a, sq);
                    sk = fmaf(bb, bb, sk);
                }
                for (int off = 16; off > 0; off >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                }
                const float rq = rsqrtf(sq + p.l2_eps), rk = rsqrtf(sk + p.l2_eps);
                for (int c = lane; c < Dk; c += 32) {
                    Qs[r * L + c] *= rq;
                    Ks[r * L + c] *= rk;
                }
            }
        }
        // G is kept in log2 units from here on: every use below is a power
        // 2^(G_a - G_b) (or 2^G), one special-function instruction each.
        for (int c = tid; c < Dk; c += kThreads) {
            float run = 0.f;
            for (int r = 0; r < Cc; ++r) {
                run += Gs[r * L + c];
                Gs[r * L + c] = run * kLog2E;
            }
            Glast[c] = run * kLog2E;
        }
        __syncthreads();
        // ---- 3. A, P and X = V - (K*exp(G)) S -------------------------------
        if (kAnchored) {
            // A[r][i] = sum_c (q_rc 2^(G_rc - P_R)) (k_ic 2^(P_R - G_ic)), R = tile of r
            // (P likewise with k_rc), every factor within 2^+-116.  Of the 20
            // half-blocks (row tile R, column tile J <= R, 8 rows), warp w takes
            // half-block w over all channels and a quarter of the channels of
            // half-block 16 + w % 4 (summed below), 20 eight-channel steps per
            // warp; it stages its own factors in its scratch row (no CTA
            // barrier): [8 ch][8 rows] of q and k, [8 ch][16 columns], and
            // multiplies them on the tensor cores.  The quarter sums go to the
            // U and dU tiles, free until step 4.
            const int ntile = (Cc + 15) >> 4;
            float *Qw = wb, *Kw = wb + 64, *Kcw = wb + 128;
#pragma unroll 1
            for (int t = 0; t < 2; ++t) {
                const int hbi = t == 0 ? warp : 16 + (warp & 3);   // (R, J) in order, then half
                const int cbeg = t == 0 ? 0 : 32 * (warp >> 2), cend = t == 0 ? Dk : cbeg + 32;
                const int blk = hbi >> 1;
                int R = 0;
                while (blk >= (R + 1) * (R + 2) / 2) ++R;
                const int J = blk - R * (R + 1) / 2, rw0 = 16 * R + 8 * (hbi & 1);
                if (R >= ntile) continue;
                // the block product transposed, D[i][r] = sum_c Khat[i][c] Q~[r][c]
                // (M = 16 columns, N = 8 rows, K = 8 channels per step) on the
                // tensor cores; lane (g, t) = (lane / 4, lane % 4) holds
                // D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1]
                float dA[4] = {0.f, 0.f, 0.f, 0.f}, dP[4] = {0.f, 0.f, 0.f, 0.f};
                const int g8 = lane >> 2, t4 = lane & 3;
                for (int c0 = cbeg; c0 < cend; c0 += 8) {
                    // rows: (cc = e & 7, row e >> 3), two per lane; columns: four per lane
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int e = lane + 32 * u, cc = e & 7, rr = rw0 + (e >> 3), c = c0 + cc;
                        const float PR = R == 0 ? 0.f : Gs[(16 * R - 1) * L + c];
                        const float f = ex2f_(Gs[rr * L + c] - PR);
                        Qw[cc * 8 + (e >> 3)] = Qs[rr * L + c] * f;
                        Kw[cc * 8 + (e >> 3)] = Ks[rr * L + c] * f;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int e = lane + 32 * u, cc = e >> 4, i = 16 * J + (e & 15), c = c0 + cc;
                        const float PR = R == 0 ? 0.f : Gs[(16 * R - 1) * L + c];
                        Kcw[cc * 16 + (e & 15)] = Ks[i * L + c] * ex2f_(PR - Gs[i * L + c]);
                    }
                    __syncwarp();
                    {
                        uint32_t ah[4], al[4], bh[2], bl[2];
                        split_tf32(Kcw[t4 * 16 + g8], ah[0], al[0]);
                        split_tf32(Kcw[t4 * 16 + g8 + 8], ah[1], al[1]);
                        split_tf32(Kcw[(t4 + 4) * 16 + g8], ah[2], al[2]);
                        split_tf32(Kcw[(t4 + 4) * 16 + g8 + 8], ah[3], al[3]);
                        split_tf32(Qw[t4 * 8 + g8], bh[0], bl[0]);
                        split_tf32(Qw[(t4 + 4) * 8 + g8], bh[1], bl[1]);
                        mma3_tf32(dA, ah, al, bh, bl);
                        split_tf32(Kw[t4 * 8 + g8], bh[0], bl[0]);
                        split_tf32(Kw[(t4 + 4) * 8 + g8], bh[1], bl[1]);
                        mma3_tf32(dP, ah, al, bh, bl);
                    }
                    __syncwarp();
                }
                if (t == 1) {                       // a quarter sum: [quarter][half-block][lane][8]
                    const int q = warp >> 2;
                    float *part = (q < 2 ? Us + q * 1024 : dUs + (q - 2) * 1024) + ((hbi - 16) * 32 + lane) * 8;
                    *reinterpret_cast<float4 *>(part) = make_float4(dA[0], dA[1], dA[2], dA[3]);
                    *reinterpret_cast<float4 *>(part + 4) = make_float4(dP[0], dP[1], dP[2], dP[3]);
                    continue;
                }
                // stores: A lower with the diagonal, P strictly lower, zeros above;
                // value v of the lane is row rw0 + 2t + (v & 1), column 16J + g + 8 (v >> 1)
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int r = rw0 + 2 * t4 + (v & 1), i = 16 * J + g8 + 8 * (v >> 1);
                    if (r >= Cc || i >= Cc) continue;
                    Aqk[r * C + i] = i <= r ? dA[v] : 0.f;
                    Pkk[r * C + i] = i < r ? dP[v] : 0.f;
                }
            }
            // the blocks above the diagonal tiles
            for (int e = tid; e < Cc * Cc; e += kThreads) {
                const int r = e / Cc, i = e % Cc;
                if ((i >> 4) > (r >> 4)) {
                    Aqk[r * C + i] = 0.f;
                    Pkk[r * C + i] = 0.f;
                }
            }
            __syncthreads();
            // half-blocks 16..19 (row tile 3, column tiles 2 and 3): the sums of
            // the four quarters, [half-block][lane][4 A values, 4 P values]
            if (ntile == 4) {
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    const int idx = tid + kThreads * m;
                    const float v = (Us[idx] + Us[1024 + idx]) + (dUs[idx] + dUs[1024 + idx]);
                    const int hbi = 16 + (idx >> 8), ln = (idx >> 3) & 31, u = idx & 3;
                    const int r = 48 + 8 * (hbi & 1) + 2 * (ln & 3) + (u & 1);
                    const int i = 16 * ((hbi >> 1) - 6) + (ln >> 2) + 8 * (u >> 1);
                    if (r < Cc && i < Cc) {
                        if ((idx & 4) == 0) Aqk[r * C + i] = i <= r ? v : 0.f;
                        else Pkk[r * C + i] = i < r ? v : 0.f;
                    }
                }
            }
        } else {
            for (int pidx = tid; pidx < Cc * Cc; pidx += kThreads) {
                const int r = pidx / Cc, i = pidx % Cc;
                float a = 0.f, pk = 0.f;
                if (i <= r) {
                    const float *kr = Ks + r * L, *ki = Ks + i * L, *qr = Qs + r * L;
                    const float *gr = Gs + r * L, *gi = Gs + i * L;
                    for (int c = 0; c < Dk; ++c) {
                        const float kie = ki[c] * ex2f_(gr[c] - gi[c]);
                        a = fmaf(qr[c], kie, a);
                        pk = fmaf(kr[c], kie, pk);
                    }
                    if (i == r) pk = 0.f;
                }
                Aqk[r * C + i] = a;
                Pkk[r * C + i] = pk;
            }
        }
        if (kAnchored) {
            __syncthreads();                   // the quarter sums were read from the U and dU tiles
            // warp w takes rows w, w + 16, w + 32, w + 48 (their factor rows in
            // its scratch row and in its rows of the U and dU tiles, free until
            // step 4); lane = value column: one load of S^T per lane and four
            // channels serves all four rows
            float *wr[4] = {wb, wb + 128, Us + warp * 128, dUs + warp * 128};
            int rs[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) rs[q] = warp + 16 * q < Cc ? warp + 16 * q : warp;
            if (warp < Cc) {
                for (int c = lane; c < Dk; c += 32) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) wr[q][c] = -Ks[rs[q] * L + c] * ex2f_(Gs[rs[q] * L + c]);
                }
                __syncwarp();
                float2 acc[4][2];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[q][0] = make_float2(Xs[rs[q] * kVT + lane], 0.f);
                    acc[q][1] = make_float2(0.f, 0.f);
                }
                const float *srow = Ss + lane * SL;
                for (int c = 0; c < Dk; c += 4) {
                    const float4 s4 = *reinterpret_cast<const float4 *>(srow + c);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 w4 = *reinterpret_cast<const float4 *>(wr[q] + c);
                        acc[q][0] = __ffma2_rn(make_float2(w4.x, w4.y), make_float2(s4.x, s4.y), acc[q][0]);
                        acc[q][1] = __ffma2_rn(make_float2(w4.z, w4.w), make_float2(s4.z, s4.w), acc[q][1]);
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (warp + 16 * q < Cc)
                        Xs[rs[q] * kVT + lane] = (acc[q][0].x + acc[q][0].y) + (acc[q][1].x + acc[q][1].y);
            }
        } else
        // warp w takes the row pairs (r, r + 16), r = w, w + 32, ...; lane = value
        // column (one load of S^T per lane and four channels for both rows);
        // channel pairs (c, c + 1) in one packed FMA
        for (int r = warp; r < Cc; r += 2 * (kThreads / 32)) {
            const int r2 = r + kThreads / 32;
            const bool has2 = r2 < Cc;
            const int rb = has2 ? r2 : r;
            for (int c = lane; c < Dk; c += 32) {
                wb[c] = -Ks[r * L + c] * ex2f_(Gs[r * L + c]);
                wb[128 + c] = -Ks[rb * L + c] * ex2f_(Gs[rb * L + c]);
            }
            __syncwarp();
            float2 a0 = make_float2(Xs[r * kVT + lane], 0.f), a1 = make_float2(0.f, 0.f);
            float2 b0 = make_float2(Xs[rb * kVT + lane], 0.f), b1 = make_float2(0.f, 0.f);
            const float *srow = Ss + lane * SL;
            int c = 0;
            for (; c + 3 < Dk; c += 4) {
                const float4 s4 = *reinterpret_cast<const float4 *>(srow + c);
                const float4 wa = *reinterpret_cast<const float4 *>(wb + c);
                const float4 wc = *reinterpret_cast<const float4 *>(wb + 128 + c);
                a0 = __ffma2_rn(make_float2(wa.x, wa.y), make_float2(s4.x, s4.y), a0);
                a1 = __ffma2_rn(make_float2(wa.z, wa.w), make_float2(s4.z, s4.w), a1);
                b0 = __ffma2_rn(make_float2(wc.x, wc.y), make_float2(s4.x, s4.y), b0);
                b1 = __ffma2_rn(make_float2(wc.z, wc.w), make_float2(s4.z, s4.w), b1);
            }
            for (; c < Dk; ++c) {
                a0.x = fmaf(wb[c], srow[c], a0.x);
                b0.x = fmaf(wb[128 + c], srow[c], b0.x);
            }
            Xs[r * kVT + lane] = (a0.x + a0.y) + (a1.x + a1.y);
            if (has2) Xs[r2 * kVT + lane] = (b0.x + b0.y) + (b1.x + b1.y);
            __syncwarp();
        }
        __syncthreads();
        // ---- 4. U = (I + Diag(beta) P)^-1 Diag(beta) X by 16-row tiles: the
        //         diagonal block by forward substitution (warp 0, lane = value
        //         column), then its contribution taken off every later row (all
        //         threads); U is built in place over a copy of X ------------------
        for (int idx = tid; idx < Cc * kVT; idx += kThreads) Us[idx] = Xs[idx];
        // the exp(G_last) dS'.S term of the last row's dG (independent of U)
        for (int c = tid; c < Dk; c += kThreads) {
            float acc = 0.f;
            for (int j = 0; j < kVT; ++j) acc = fmaf(Ss[j * SL + c], dSs[j * SL + c], acc);
            dlast[c] = ex2f_(Glast[c]) * acc;
        }
        __syncthreads();
        for (int R0 = 0; R0 < Cc; R0 += 16) {
            const int R1 = min(R0 + 16, Cc);
            if (warp == 0) {
                // the block's column lane in registers; row a takes the finished
                // rows above it (row of P contiguous, two partial sums)
                float u[16];
#pragma unroll
                for (int a = 0; a < 16; ++a) u[a] = (R0 + a < R1) ? Us[(R0 + a) * kVT + lane] : 0.f;
#pragma unroll
                for (int a = 0; a < 16; ++a) {
                    if (R0 + a >= R1) break;
                    const float *pr = Pkk + (R0 + a) * C + R0;
                    float acc0 = u[a], acc1 = 0.f;
#pragma unroll
                    for (int i = 0; i < a; ++i) {
                        if (i & 1) acc1 = fmaf(-pr[i], u[i], acc1);
                        else acc0 = fmaf(-pr[i], u[i], acc0);
                    }
                    u[a] = bet[R0 + a] * (acc0 + acc1);
                }
#pragma unroll
                for (int a = 0; a < 16; ++a)
                    if (R0 + a < R1) Us[(R0 + a) * kVT + lane] = u[a];
            }
            __syncthreads();
            if (R1 < Cc) {
                for (int idx = tid; idx < (Cc - R1) * kVT; idx += kThreads) {
                    const int r = R1 + idx / kVT, jj = idx % kVT;
                    float acc = Us[r * kVT + jj];
                    if ((C & 3) == 0 && R1 == R0 + 16) {     // the row of P as four float4s
                        const float4 *prow = reinterpret_cast<const float4 *>(Pkk + r * C + R0);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const float4 pv = prow[q4];
                            acc = fmaf(-pv.x, Us[(R0 + 4 * q4) * kVT + jj], acc);
                            acc = fmaf(-pv.y, Us[(R0 + 4 * q4 + 1) * kVT + jj], acc);
                            acc = fmaf(-pv.z, Us[(R0 + 4 * q4 + 2) * kVT + jj], acc);
                            acc = fmaf(-pv.w, Us[(R0 + 4 * q4 + 3) * kVT + jj], acc);
                        }
                    } else {
#pragma unroll
                        for (int a = 0; a < 16; ++a)
                            if (R0 + a < R1) acc = fmaf(-Pkk[r * C + R0 + a], Us[(R0 + a) * kVT + jj], acc);
                    }
                    Us[r * kVT + jj] = acc;
                }
                __syncthreads();
            }
        }
        // ---- 5. dU = A^T dO + (K*exp(G_last - G)) dS' ------------------------
        // row pairs (r, r + 16) as in X: A^T dO with (A[rr][r], A[rr][r + 16])
        // in one packed FMA (A is zero above the diagonal), then the dS' terms
        for (int r = warp; r < Cc; r += 2 * (kThreads / 32)) {
            const int r2 = r + kThreads / 32;
            const bool has2 = r2 < Cc;
            const int rb = has2 ? r2 : r;
            for (int c = lane; c < Dk; c += 32) {
                wb[c] = Ks[r * L + c] * ex2f_(Glast[c] - Gs[r * L + c]);
                wb[128 + c] = Ks[rb * L + c] * ex2f_(Glast[c] - Gs[rb * L + c]);
            }
            __syncwarp();
            float2 ab = make_float2(0.f, 0.f);
            for (int rr = r; rr < Cc; ++rr) {
                const float o = dOs[rr * kVT + lane];
                ab = __ffma2_rn(make_float2(Aqk[rr * C + r], Aqk[rr * C + rb]), make_float2(o, o), ab);
            }
            const float *drow = dSs + lane * SL;
            float2 a0 = make_float2(ab.x, 0.f), a1 = make_float2(0.f, 0.f);
            float2 b0 = make_float2(ab.y, 0.f), b1 = make_float2(0.f, 0.f);
            int c = 0;
            for (; c + 3 < Dk; c += 4) {
                const float4 d4 = *reinterpret_cast<const float4 *>(drow + c);
                const float4 wa = *reinterpret_cast<const float4 *>(wb + c);
                const float4 wc = *reinterpret_cast<const float4 *>(wb + 128 + c);
                a0 = __ffma2_rn(make_float2(wa.x, wa.y), make_float2(d4.x, d4.y), a0);
                a1 = __ffma2_rn(make_float2(wa.z, wa.w), make_float2(d4.z, d4.w), a1);
                b0 = __ffma2_rn(make_float2(wc.x, wc.y), make_float2(d4.x, d4.y), b0);
                b1 = __ffma2_rn(make_float2(wc.z, wc.w), make_float2(d4.z, d4.w), b1);
            }
            for (; c < Dk; ++c) {
                a0.x = fmaf(wb[c], drow[c], a0.x);
                b0.x = fmaf(wb[128 + c], drow[c], b0.x);
            }
            dUs[r * kVT + lane] = (a0.x + a0.y) + (a1.x + a1.y);
            if (has2) dUs[r2 * kVT + lane] = (b0.x + b0.y) + (b1.x + b1.y);
            __syncwarp();
        }
        __syncthreads();
        // ---- 6. dZ = (I + Diag(beta) P)^-T dU in place, by 16-row tiles from
        //         the last: the diagonal block by back substitution (warp 0), then
        //         its contribution taken off every earlier row (all threads) ----
        for (int T = (Cc - 1) >> 4; T >= 0; --T) {
            const int R0 = 16 * T, R1 = min(R0 + 16, Cc);
            if (warp == 0) {
                // right-looking from the bottom: once dZ_b is final every earlier
                // row of the block takes its term
                float z[16];
#pragma unroll
                for (int a = 0; a < 16; ++a) z[a] = (R0 + a < R1) ? dUs[(R0 + a) * kVT + lane] : 0.f;
#pragma unroll
                for (int b = 15; b >= 0; --b) {
                    if (R0 + b >= R1) continue;
                    const float zb = bet[R0 + b] * z[b];
#pragma unroll
                    for (int a = 0; a < b; ++a) z[a] = fmaf(-Pkk[(R0 + b) * C + R0 + a], zb, z[a]);
                }
#pragma unroll
                for (int a = 0; a < 16; ++a)
                    if (R0 + a < R1) dUs[(R0 + a) * kVT + lane] = z[a];
            }
            __syncthreads();
            if (R0 > 0) {
                for (int idx = tid; idx < R0 * kVT; idx += kThreads) {
                    const int r = idx / kVT, jj = idx % kVT;
                    float acc = dUs[idx];
#pragma unroll
                    for (int a = 0; a < 16; ++a)
                        if (R0 + a < R1)
                            acc = fmaf(-bet[R0 + a] * Pkk[(R0 + a) * C + r], dUs[(R0 + a) * kVT + jj], acc);
                    dUs[idx] = acc;
                }
                __syncthreads();
            }
        }
        // ---- 7. dA, dP, dbeta and dV ------------------------------------------
        // Warp w takes rows w, w + 16, ...: lane = column i (rounds of 32),
        // then lane = value column for dV; the row's dbeta is a warp sum.  The
        // value-column pairs start at a lane-dependent offset so that the lanes
        // of a half-warp read different shared-memory banks.
        for (int r = warp; r < Cc; r += kThreads / 32) {
            float db = 0.f;
            // columns i = lane and i + 32 in one pass over the value columns of
            // rows r of dO and dZ (the second only where it is on or below the
            // diagonal: r >= 32)
            const int i1 = lane + 32;
            const bool two = r >= 32;
            float2 da = make_float2(0.f, 0.f), dm = make_float2(0.f, 0.f);
            float2 da1 = da, dm1 = da;
            if (lane <= r) {
                for (int j0 = 0; j0 < kVT; j0 += 2) {
                    const int j = (j0 + 2 * lane) & (kVT - 1);
                    const float2 o2 = *reinterpret_cast<const float2 *>(dOs + r * kVT + j);
                    const float2 z2 = *reinterpret_cast<const float2 *>(dUs + r * kVT + j);
                    const float2 u = *reinterpret_cast<const float2 *>(Us + lane * kVT + j);
                    da = __ffma2_rn(o2, u, da);
                    dm = __ffma2_rn(z2, u, dm);
                    if (two) {
                        const float2 u1 = *reinterpret_cast<const float2 *>(Us + i1 * kVT + j);
                        da1 = __ffma2_rn(o2, u1, da1);
                        dm1 = __ffma2_rn(z2, u1, dm1);
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = h ? i1 : lane;
                if (i >= Cc) continue;
                const float2 a2 = h ? da1 : da, m2 = h ? dm1 : dm;
                const float dms = (i <= r) ? -(m2.x + m2.y) : 0.f;
                if (i < r) {
                    db = fmaf(dms, Pkk[r * C + i], db);
                    Pkk[r * C + i] = bet[r] * dms;
                } else {
                    Pkk[r * C + i] = 0.f;
                }
                Aqk[r * C + i] = (i <= r) ? a2.x + a2.y : 0.f;
            }
            const float dz = dUs[r * kVT + lane];
            db = fmaf(dz, Xs[r * kVT + lane], db);
            if (col0 + lane < Dv) p.dv[((tok0 + r) * p.HV + hv) * Dv + col0 + lane] = bet[r] * dz;
            for (int off = 16; off > 0; off >>= 1) db += __shfl_xor_sync(0xffffffffu, db, off);
            if (lane == 0) dbet[r] = db;
        }
        __syncthreads();
        // ---- 8. per (r, c): dq, dk (atomics) and dG (registers) --------------
        float dG[kElemsPerThread];
        if (kAnchored) {
            // Thread (tile R, 8-row half h, channels c and c + 64): rows
            // r = 16R + 8h + a, a < 8, so every row of dA, dP, dO, dZ and U read
            // by a warp serves two channels.  Pairwise sums with tile anchors
            // P_J = G at the row before tile J (0 for J = 0):
            //   aq_r = 2^(G_r - P_R) sum_{i <= r} dA[r][i] k_i 2^(P_R - G_i)
            //   ak_r = sum_{J >= R} 2^(P_J - G_r) sum_{rr in J, rr >= r} dA[rr][r] q_rr 2^(G_rr - P_J)
            // (pr, pc likewise with dP and k).  Entries of dA / dP above the
            // diagonal are zero, so the sums run over whole tiles.  dG[8 ch + a].
            const int R = tid >> 7, hh = (tid >> 6) & 1, cl = tid & 63, r0 = 16 * R, ra = r0 + 8 * hh;
            const int ntile = (Cc + 15) >> 4;
            float dq[2][8], dk[2][8];
            float dl[2] = {0.f, 0.f};                // this thread's shares of dlast[c]
            if (R >= ntile || ra >= Cc) {
#pragma unroll
                for (int n = 0; n < 16; ++n) dG[n] = 0.f;
            } else {
                float PR[2];
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) PR[ch] = R == 0 ? 0.f : Gs[(r0 - 1) * L + cl + 64 * ch];
                {
                    // column pairs (i, i + 1) in one packed FMA per row and channel
                    float2 sa[2][8], sp[2][8];
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                        for (int a = 0; a < 8; ++a) sa[ch][a] = sp[ch][a] = make_float2(0.f, 0.f);
                    const int iend = min(r0 + 16, Cc);
                    int i = 0;
                    for (; i + 1 < iend; i += 2) {
                        float2 kc[2];
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch) {
                            const int c = cl + 64 * ch;
                            kc[ch] = make_float2(Ks[i * L + c] * ex2f_(PR[ch] - Gs[i * L + c]),
                                                 Ks[(i + 1) * L + c] * ex2f_(PR[ch] - Gs[(i + 1) * L + c]));
                        }
#pragma unroll
                        for (int a = 0; a < 8; ++a) {
                            const float2 av = *reinterpret_cast<const float2 *>(Aqk + (ra + a) * C + i);
                            const float2 pv = *reinterpret_cast<const float2 *>(Pkk + (ra + a) * C + i);
#pragma unroll
                            for (int ch = 0; ch < 2; ++ch) {
                                sa[ch][a] = __ffma2_rn(av, kc[ch], sa[ch][a]);
                                sp[ch][a] = __ffma2_rn(pv, kc[ch], sp[ch][a]);
                            }
                        }
                    }
                    if (i < iend) {                  // an odd last column
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch) {
                            const int c = cl + 64 * ch;
                            const float kc = Ks[i * L + c] * ex2f_(PR[ch] - Gs[i * L + c]);
#pragma unroll
                            for (int a = 0; a < 8; ++a) {
                                sa[ch][a].x = fmaf(Aqk[(ra + a) * C + i], kc, sa[ch][a].x);
                                sp[ch][a].x = fmaf(Pkk[(ra + a) * C + i], kc, sp[ch][a].x);
                            }
                        }
                    }
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                        for (int a = 0; a < 8; ++a) {
                            const int c = cl + 64 * ch, r = ra + a, n = 8 * ch + a;
                            dq[ch][a] = dk[ch][a] = dG[n] = 0.f;
                            if (r >= Cc) continue;
                            const float fr = ex2f_(Gs[r * L + c] - PR[ch]);
                            const float aq = fr * (sa[ch][a].x + sa[ch][a].y), pr = fr * (sp[ch][a].x + sp[ch][a].y);
                            dq[ch][a] = aq;
                            dk[ch][a] = pr;
                            dG[n] = Qs[r * L + c] * aq + Ks[r * L + c] * pr;
                        }
                }
                for (int J = R; J < ntile; ++J) {
                    float PJ[2];
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch) PJ[ch] = J == 0 ? 0.f : Gs[(16 * J - 1) * L + cl + 64 * ch];
                    // rows (2m, 2m + 1) of ak + pc in one packed FMA, per channel
                    float2 s2[2][4];
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                        for (int m = 0; m < 4; ++m) s2[ch][m] = make_float2(0.f, 0.f);
                    const int rend = min(16 * J + 16, Cc);
                    for (int rr = 16 * J; rr < rend; ++rr) {
                        const float4 *arow = reinterpret_cast<const float4 *>(Aqk + rr * C + ra);
                        const float4 *prow = reinterpret_cast<const float4 *>(Pkk + rr * C + ra);
                        const float4 a0 = arow[0], a1 = arow[1], p0 = prow[0], p1 = prow[1];
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch) {
                            const int c = cl + 64 * ch;
                            const float e = ex2f_(Gs[rr * L + c] - PJ[ch]);
                            const float qe = Qs[rr * L + c] * e, ke = Ks[rr * L + c] * e;
                            const float2 qe2 = make_float2(qe, qe), ke2 = make_float2(ke, ke);
                            s2[ch][0] = __ffma2_rn(make_float2(a0.x, a0.y), qe2, s2[ch][0]);
                            s2[ch][1] = __ffma2_rn(make_float2(a0.z, a0.w), qe2, s2[ch][1]);
                            s2[ch][2] = __ffma2_rn(make_float2(a1.x, a1.y), qe2, s2[ch][2]);
                            s2[ch][3] = __ffma2_rn(make_float2(a1.z, a1.w), qe2, s2[ch][3]);
                            s2[ch][0] = __ffma2_rn(make_float2(p0.x, p0.y), ke2, s2[ch][0]);
                            s2[ch][1] = __ffma2_rn(make_float2(p0.z, p0.w), ke2, s2[ch][1]);
                            s2[ch][2] = __ffma2_rn(make_float2(p1.x, p1.y), ke2, s2[ch][2]);
                            s2[ch][3] = __ffma2_rn(make_float2(p1.z, p1.w), ke2, s2[ch][3]);
                        }
                    }
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                        for (int a = 0; a < 8; ++a) {
                            const int c = cl + 64 * ch, r = ra + a;
                            if (r >= Cc) continue;
                            const float f = ex2f_(PJ[ch] - Gs[r * L + c]);
                            const float akpc = f * ((a & 1) ? s2[ch][a >> 1].y : s2[ch][a >> 1].x);   // ak + pc
                            dk[ch][a] += akpc;
                            dG[8 * ch + a] -= Ks[r * L + c] * akpc;
                        }
                }
                // elementwise factors: dQg = dO S^T, dKw = -dX S^T, dKd = U dS'^T,
                // four rows at a time: the value columns j .. j+3 of a row are one
                // broadcast float4 serving both channels; the two channels' S and
                // dS' entries are one conflict-free load each
#pragma unroll
                for (int hb = 0; hb < 2; ++hb) {
                    float dqg[2][4], dkw[2][4], dkd[2][4];
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                        for (int a = 0; a < 4; ++a) dqg[ch][a] = dkw[ch][a] = dkd[ch][a] = 0.f;
                    for (int j = 0; j < kVT; j += 4) {
                        float sv[2][4], dv[2][4];
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                sv[ch][u] = Ss[(j + u) * SL + cl + 64 * ch];
                                dv[ch][u] = dSs[(j + u) * SL + cl + 64 * ch];
                            }
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            const int r = ra + 4 * hb + a;
                            const float4 o4 = *reinterpret_cast<const float4 *>(dOs + r * kVT + j);
                            const float4 u4 = *reinterpret_cast<const float4 *>(dUs + r * kVT + j);
                            const float4 v4 = *reinterpret_cast<const float4 *>(Us + r * kVT + j);
#pragma unroll
                            for (int ch = 0; ch < 2; ++ch) {
                                dqg[ch][a] = fmaf(o4.x, sv[ch][0], fmaf(o4.y, sv[ch][1], fmaf(o4.z, sv[ch][2], fmaf(o4.w, sv[ch][3], dqg[ch][a]))));
                                dkw[ch][a] = fmaf(u4.x, sv[ch][0], fmaf(u4.y, sv[ch][1], fmaf(u4.z, sv[ch][2], fmaf(u4.w, sv[ch][3], dkw[ch][a]))));
                                dkd[ch][a] = fmaf(v4.x, dv[ch][0], fmaf(v4.y, dv[ch][1], fmaf(v4.z, dv[ch][2], fmaf(v4.w, dv[ch][3], dkd[ch][a]))));
                            }
                        }
                    }
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            const int aa = 4 * hb + a, r = ra + aa, c = cl + 64 * ch;
                            if (r >= Cc) continue;
                            const float grc = Gs[r * L + c], qrc = Qs[r * L + c], krc = Ks[r * L + c];
                            const float vqg = dqg[ch][a], vkd = dkd[ch][a];
                            const float kw = -bet[r] * dkw[ch][a];
                            const float eg = ex2f_(grc), ed = ex2f_(Glast[c] - grc);
                            dq[ch][aa] = fmaf(eg, vqg, dq[ch][aa]);
                            dk[ch][aa] += eg * kw + ed * vkd;
                            dG[8 * ch + aa] += eg * (vqg * qrc + kw * krc) - ed * vkd * krc;
                            dl[ch] = fmaf(ed * vkd, krc, dl[ch]);
                        }
                }
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
                    for (int a = 0; a < 8; ++a) {
                        if (ra + a >= Cc) continue;
                        const size_t tq = ((tok0 + ra + a) * p.H + h) * Dk + cl + 64 * ch;
                        atomicAdd(&p.dq[tq], dq[ch][a]);
                        atomicAdd(&p.dk[tq], dk[ch][a]);
                    }
                    atomicAdd(&dlast[cl + 64 * ch], dl[ch]);
                }
            }
        } else {
#pragma unroll
            for (int n = 0; n < kElemsPerThread; ++n) {
                const int idx = tid + n * kThreads;
                dG[n] = 0.f;
                if (idx >= Cc * Dk) continue;
                const int r = idx / Dk, c = idx % Dk;
                const float qrc = Qs[r * L + c], krc = Ks[r * L + c], grc = Gs[r * L + c];
                // pairwise sums: row r against earlier tokens, then later tokens against r
                float aq = 0.f, pr = 0.f;
                for (int i = 0; i <= r; ++i) {
                    const float kie = Ks[i * L + c] * ex2f_(grc - Gs[i * L + c]);
                    aq = fmaf(Aqk[r * C + i], kie, aq);
                    pr = fmaf(Pkk[r * C + i], kie, pr);
                }
                float ak = 0.f, pc = 0.f;
                for (int rr = r; rr < Cc; ++rr) {
                    const float e = ex2f_(Gs[rr * L + c] - grc);
                    ak = fmaf(Aqk[rr * C + r], Qs[rr * L + c] * e, ak);
                    pc = fmaf(Pkk[rr * C + r], Ks[rr * L + c] * e, pc);
                }
                // elementwise factors: dQg = dO S^T, dKw = -dX S^T, dKd = U dS'^T
                float dqg = 0.f, dkw = 0.f, dkd = 0.f;
                const float br = bet[r];
                for (int j = 0; j < kVT; ++j) {
                    const float s = Ss[j * SL + c];
                    dqg = fmaf(dOs[r * kVT + j], s, dqg);
                    dkw = fmaf(-br * dUs[r * kVT + j], s, dkw);
                    dkd = fmaf(Us[r * kVT + j], dSs[j * SL + c], dkd);
                }
                const float eg = ex2f_(grc), ed = ex2f_(Glast[c] - grc);
                const size_t tq = ((tok0 + r) * p.H + h) * Dk + c;
                atomicAdd(&p.dq[tq], fmaf(eg, dqg, aq));
                atomicAdd(&p.dk[tq], ak + pr + pc + eg * dkw + ed * dkd);
                dG[n] = qrc * aq - krc * ak + krc * pr - krc * pc + eg * (dqg * qrc + dkw * krc) - ed * dkd * krc;
                atomicAdd(&dlast[c], ed * dkd * krc);
            }
        }
        __syncthreads();
        if (can_stage && ch > 0) {
            // q, k, g rows of chunk ch - 1 (full: C rows of 256 bytes) into the
            // free A/P/X/U tiles, 16 bytes per copy
            const size_t ptok = tok0 - C;
            uint8_t *dst = reinterpret_cast<uint8_t *>(Aqk);
            for (int e = tid; e < 3 * C * 16; e += kThreads) {
                const int tsr = e / (C * 16), rest = e % (C * 16), r = rest >> 4, q16 = rest & 15;
                const size_t tok = ptok + r;
                const uint8_t *src =
                    tsr == 0   ? reinterpret_cast<const uint8_t *>(q + (tok * p.H + h) * 128)
                    : tsr == 1 ? reinterpret_cast<const uint8_t *>(k + (tok * p.H + h) * 128)
                               : reinterpret_cast<const uint8_t *>(g + (tok * p.HV + hv) * 128);
                cp_async16(dst + ((size_t)(tsr * C + r) * 128) * 2 + 16 * q16, src + 16 * q16);
            }
            cp_async_commit();
        }
        // ---- 9. dS entering the chunk (in place) -----------------------------
        // thread = (key channel c, eight value columns j0 .. j0+7): the factors
        // e^G q and -e^G k beta of (r, c) once per thread, the value columns of
        // rows r of dO and dZ as broadcast float4s; each thread reads and then
        // overwrites only its own entries of dS'
        {
            const int c = tid & 127, j0 = 8 * (tid >> 7);
            if (c < Dk) {
                const float el = ex2f_(Glast[c]);
                float2 acc[4];
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    acc[m] = make_float2(el * dSs[(j0 + 2 * m) * SL + c], el * dSs[(j0 + 2 * m + 1) * SL + c]);
                for (int r = 0; r < Cc; ++r) {
                    const float e = ex2f_(Gs[r * L + c]);
                    const float w1 = e * Qs[r * L + c], w2 = -e * Ks[r * L + c] * bet[r];
                    const float2 w1p = make_float2(w1, w1), w2p = make_float2(w2, w2);
                    const float4 o0 = *reinterpret_cast<const float4 *>(dOs + r * kVT + j0);
                    const float4 o1 = *reinterpret_cast<const float4 *>(dOs + r * kVT + j0 + 4);
                    const float4 z0 = *reinterpret_cast<const float4 *>(dUs + r * kVT + j0);
                    const float4 z1 = *reinterpret_cast<const float4 *>(dUs + r * kVT + j0 + 4);
                    acc[0] = __ffma2_rn(make_float2(o0.x, o0.y), w1p, acc[0]);
                    acc[1] = __ffma2_rn(make_float2(o0.z, o0.w), w1p, acc[1]);
                    acc[2] = __ffma2_rn(make_float2(o1.x, o1.y), w1p, acc[2]);
                    acc[3] = __ffma2_rn(make_float2(o1.z, o1.w), w1p, acc[3]);
                    acc[0] = __ffma2_rn(make_float2(z0.x, z0.y), w2p, acc[0]);
                    acc[1] = __ffma2_rn(make_float2(z0.z, z0.w), w2p, acc[1]);
                    acc[2] = __ffma2_rn(make_float2(z1.x, z1.y), w2p, acc[2]);
                    acc[3] = __ffma2_rn(make_float2(z1.z, z1.w), w2p, acc[3]);
                }
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    dSs[(j0 + 2 * m) * SL + c] = acc[m].x;
                    dSs[(j0 + 2 * m + 1) * SL + c] = acc[m].y;
                }
            }
        }
        __syncthreads();
        if (kAnchored) {
            const int ra = 16 * (tid >> 7) + 8 * ((tid >> 6) & 1), cl = tid & 63;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                for (int a = 0; a < 8; ++a)
                    if (ra + a < Cc) Gs[(ra + a) * L + cl + 64 * ch] = dG[8 * ch + a];
        } else {
#pragma unroll
            for (int n = 0; n < kElemsPerThread; ++n) {
                const int idx = tid + n * kThreads;
                if (idx < Cc * Dk) Gs[(idx / Dk) * L + idx % Dk] = dG[n];
            }
        }
        __syncthreads();
        // ---- 10. dg = reverse cumulative sum of dG; dbeta --------------------
        for (int c = tid; c < Dk; c += kThreads) {
            float acc = dlast[c];
            for (int r = Cc - 1; r >= 0; --r) {
                acc += Gs[r * L + c];
                if (p.g_per_head) Gs[r * L + c] = acc;
                else atomicAdd(&p.dg[((tok0 + r) * p.HV + hv) * Dk + c], acc);
            }
        }
        for (int r = tid; r < Cc; r += kThreads) atomicAdd(&p.dbeta[(tok0 + r) * p.HV + hv], dbet[r]);
        if (p.g_per_head) {
            // one decay per (token, head): its gradient sums over the key channels
            __syncthreads();
            for (int r = warp; r < Cc; r += kThreads / 32) {
                float sum = 0.f;
                for (int c = lane; c < Dk; c += 32) sum += Gs[r * L + c];
                for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
                if (lane == 0) atomicAdd(&p.dg[(tok0 + r) * p.HV + hv], sum);
            }
        }
    }
    __syncthreads();
    if (p.dS0) {
        for (int idx = tid; idx < Dk * kVT; idx += kThreads) {
            const int c = idx / kVT, col = col0 + idx % kVT;
            if (col < Dv) p.dS0[((size_t)chain * Dk + c) * Dv + col] = dSs[(idx % kVT) * SL + c];
        }
    }
}

// dq, dk through q <- q / sqrt(|q|^2 + eps): warp per (token, head) row.
template <typename Tin>
__global__ void __launch_bounds__(kRowThreads)
bwd_l2norm_kernel(BwdParams p) {
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5);
    const long long rows = (long long)p.B * p.T * p.H;
    if (row >= rows) return;
    const Tin *xs[2] = {static_cast<const Tin *>(p.q), static_cast<const Tin *>(p.k)};
    float *ds[2] = {p.dq, p.dk};
    for (int w = 0; w < 2; ++w) {
        const size_t base = (size_t)row * p.Dk;
        float xx = 0.f, xy = 0.f;
        for (int c = lane; c < p.Dk; c += 32) {
            const float x = ld_act(xs[w], base + c), y = ds[w][base + c];
            xx = fmaf(x, x, xx);
            xy = fmaf(x, y, xy);
        }
        for (int off = 16; off > 0; off >>= 1) {
            xx += __shfl_xor_sync(0xffffffffu, xx, off);
            xy += __shfl_xor_sync(0xffffffffu, xy, off);
        }
        const float rn = rsqrtf(xx + p.l2_eps);
        const float coef = xy * rn * rn * rn;
        for (int c = lane; c < p.Dk; c += 32) {
            const float x = ld_act(xs[w], base + c);
            ds[w][base + c] = fmaf(ds[w][base + c], rn, -x * coef);
        }
    }
}

// Backward of the in-kernel gate at one element: returns dz for the upstream
// gradient dg of the log-decay and adds this element's share of the sums over
// tokens of dA_log (acc_a) and ddt_bias (acc_b).
__device__ __forceinline__ float gate_backward(int mode, float z, float bias, float ea, float g_min, float dg,
                                               float &acc_a, float &acc_b) {
    float dz;
    if (mode == 2) {             // g = -ea softplus(x), x = z + bias: dg/dx = -ea sigmoid(x), dg/dA_log = g
        const float x = z + bias;
        dz = -dg * ea * sigmoidf_(x);
        acc_a = fmaf(dg, -ea * softplusf_(x), acc_a);
    } else {                     // g = g_min sigmoid(pre), pre = ea (z + bias): dpre/dA_log = pre
        const float pre = ea * (z + bias), s = sigmoidf_(pre);
        const float dpre = dg * g_min * s * (1.f - s);
        dz = dpre * ea;
        acc_a = fmaf(dpre, pre, acc_a);
    }
    acc_b += dz;
    return dz;
}

__device__ __forceinline__ float block_sum_128(float v, float *red) {
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    const float total = red[0] + red[1] + red[2] + red[3];
    __syncthreads();
    return total;
}

// dbeta through the sigmoid; dg through the in-kernel gate, with the sums over
// tokens of dA_log and ddt_bias.  Block = (value head hv, kGateTokens tokens)
// of 128 threads: thread = key channel, or (one decay per head) thread = token.
constexpr int kGateTokens = 256;
template <typename Tin>
__global__ void __launch_bounds__(128)
bwd_gate_kernel(BwdParams p) {
    __shared__ float red[4];
    const int hv = blockIdx.x, tid = threadIdx.x;
    const long long n0 = (long long)blockIdx.y * kGateTokens;
    const long long ntok = (long long)p.B * p.T;
    const long long n1 = n0 + kGateTokens < ntok ? n0 + kGateTokens : ntok;
    const Tin *g = static_cast<const Tin *>(p.g);
    const Tin *bt = static_cast<const Tin *>(p.beta);
    if (p.beta_sigmoid) {
        for (long long n = n0 + tid; n < n1; n += blockDim.x) {
            const size_t i = (size_t)n * p.HV + hv;
            const float s = sigmoidf_(ld_act(bt, i));
            p.dbeta[i] *= s * (1.f - s);
        }
    }
    if (!p.gate_in) return;
    const float ea = expf(p.A_log[hv]);
    float acc_a = 0.f, acc_b = 0.f;
    if (p.g_per_head) {
        const float bias = p.dt_bias ? p.dt_bias[hv] : 0.f;
        for (long long n = n0 + tid; n < n1; n += blockDim.x) {
            const size_t i = (size_t)n * p.HV + hv;
            p.dg[i] = gate_backward(p.gate_in, ld_act(g, i), bias, ea, p.g_min, p.dg[i], acc_a, acc_b);
        }
        const float sb = block_sum_128(acc_b, red);
        if (tid == 0 && p.ddt_bias) atomicAdd(&p.ddt_bias[hv], sb);
    } else if (tid < p.Dk) {
        const float bias = p.dt_bias ? p.dt_bias[(size_t)hv * p.Dk + tid] : 0.f;
        for (long long n = n0; n < n1; ++n) {
            const size_t i = ((size_t)n * p.HV + hv) * p.Dk + tid;
            p.dg[i] = gate_backward(p.gate_in, ld_act(g, i), bias, ea, p.g_min, p.dg[i], acc_a, acc_b);
        }
        if (p.ddt_bias) atomicAdd(&p.ddt_bias[(size_t)hv * p.Dk + tid], acc_b);
    }
    const float sa = block_sum_128(acc_a, red);
    if (tid == 0 && p.dA_log) atomicAdd(&p.dA_log[hv], sa);
}

// T == 0: dS0 = dS_T (or 0).
__global__ void bwd_empty_kernel(BwdParams p) {
    const size_t n = (size_t)p.B * p.HV * p.Dk * p.Dv;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        p.dS0[i] = p.dS_T ? p.dS_T[i] : 0.f;
}

}  // namespace

// The anchored instance needs 128 key channels (thread layouts by channel),
// 64-token chunks and a decay of at most 5 per token (the anchors' bound).
inline bool bwd_anchored(const BwdParams &p) {
    return p.Dk == 128 && p.C == 64 && p.gate_in == 1 && p.g_min >= -5.0f;
}

// Dynamic shared memory of chunk_bwd_kernel (both instances use one layout;
// the anchored one also reuses the A/P/X/U tiles as its staging area).
size_t bwd_smem_bytes(int C, int Dk, bool anchored) {
    const size_t CL = ((size_t)C * (Dk | 1) + 3) & ~(size_t)3, CC = ((size_t)C * C + 3) & ~(size_t)3;
    const size_t Dk4 = ((size_t)Dk + 3) & ~(size_t)3;
    const size_t f = 3 * CL + 2 * CC + (size_t)4 * C * kVT + (size_t)2 * kVT * (Dk4 + 4) +
                     2 * (((size_t)C + 3) & ~(size_t)3) + 2 * Dk4 +
                     (size_t)(kThreads / 32) * 256;
    (void)anchored;
    return f * sizeof(float);
}

template <typename Tin, bool kAnchored>
static cudaError_t launch_bwd_main(const BwdParams &p, cudaStream_t s) {
    const size_t smem = bwd_smem_bytes(p.C, p.Dk, kAnchored);
    cudaError_t e = cudaFuncSetAttribute(chunk_bwd_kernel<Tin, kAnchored>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.B * p.HV, (p.Dv + kVT - 1) / kVT);
    chunk_bwd_kernel<Tin, kAnchored><<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <typename Tin>
static cudaError_t launch_bwd_t(const BwdParams &p, cudaStream_t s) {
    cudaError_t e = bwd_anchored(p) ? launch_bwd_main<Tin, true>(p, s) : launch_bwd_main<Tin, false>(p, s);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (p.l2norm) {
        const long long rows = (long long)p.B * p.T * p.H;
        bwd_l2norm_kernel<Tin><<<(unsigned)((rows + kRowThreads / 32 - 1) / (kRowThreads / 32)), kRowThreads, 0,
                                 s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (p.beta_sigmoid || p.gate_in) {
        const long long ntok = (long long)p.B * p.T;
        dim3 g2(p.HV, (unsigned)((ntok + kGateTokens - 1) / kGateTokens));
        bwd_gate_kernel<Tin><<<g2, 128, 0, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_chunk_bwd(const BwdParams &p, bool bf16, cudaStream_t s) {
    if (p.T == 0) {
        if (!p.dS0) return cudaSuccess;
        bwd_empty_kernel<<<148 * 4, 256, 0, s>>>(p);
        return cudaGetLastError();
    }
    return bf16 ? launch_bwd_t<__nv_bfloat16>(p, s) : launch_bwd_t<float>(p, s);
}

}  // namespace kda
