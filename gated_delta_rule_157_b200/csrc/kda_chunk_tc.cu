// tcgen05 BF16 chunk kernel for Dk = Dv = 128, chunk C = 64, warp-specialised.
//
// One CTA (384 threads) per (b, hv) chain walks the chunks in order with the
// state on chip: fp32 S^T in tensor memory (lane j = value channel, column c =
// key channel) and a packed-bf16 copy in tensor memory as the MMA A operand.
// With G the in-chunk cumulative sum of the log-decay, tiles of 16 tokens and
// P_R the cumulative sum before tile R (page "KDA 模块交互式演示" section 1.5,
// Eqs. 3-4, with the decay-weighted UT transform; page "Implémenter KDA",
// "La forme par blocs", for U = Ut - W S), the work per chunk splits in two:
//
// prep warps 0-7 (state-independent; run one chunk ahead of the state warps)
//   loads        q, k, z, v, beta of the chunk
//   prologue     L2 norm of q,k; beta = sigmoid; g = g_min sigmoid(exp(A_log)(z + dt_bias))
//   operands     bf16 tiles scaled by exp(G_r - P_R) <= 1 and exp(P_R' - G_i)
//                (<= e^80 inside a tile, <= 1 before it)
//   (I)   MMA    [K e^L ; Q e^L] x [K_R' e^{P_R'-G}]^T    -> A_kk, A_qk (all tiles at once)
//   solve        T = (I + tril(Diag(beta) A_kk, -1))^-1    (blocked, fp32)
//   (II)  MMA    Ut^T = V^T (T Diag(beta))^T              -> TMEM buffer of the chunk
//   (III) MMA    W^T  = (K Gamma)^T (T Diag(beta))^T      -> -W (MN-major smem)
// state warps 8-11 (the serial carry, one TMEM lane per value channel)
//   (IV)  MMA    U^T = Ut^T - S^T W^T        while the state is scaled by gamma_C
//   (VI)  MMA    S^T <- S^T Diag(gamma_C) + U^T K',   K' = K exp(G_C - G)
//   (V)   MMA    O^T = S^T (Q Gamma)^T + U^T A_qk^T   -> o
//
// Every exponent is bounded: inside a 16-token tile |G_r - P_R| <= 16 |g_min| = 80
// (e^80 ~ 5.5e34 < bf16/fp32 max, page "Implémenter KDA" "La décroissance
// bornée"); across tiles the factors are decays <= 1.  Exponentials use base 2:
// the log-decay is carried in log2 units.
//
// Hand-off between the two roles uses mbarriers; the operands the state warps
// read (Q Gamma, K', A_qk, gamma_C and the Ut^T accumulator) are double
// buffered, -W is single buffered and released as soon as MMA (IV) completes.
// Every wait is bounded; if one gives up, the CTA records the device error
// word, both roles leave their loops, the TMEM is freed and the CTA returns.
//
// All MMAs are cta_group::1, M = 128, BF16 x BF16 -> FP32 in TMEM; shared
// operands use the K-major (or, for W, MN-major) 128-byte-swizzle layouts of
// tc_ptx.cuh.  When M_T is requested a second CTA per chain (blockIdx.y == 1)
// runs the same recurrence on the transition columns: v = 0 and S0 = I, no o.
#include "kda_internal.cuh"
#include "tc_ptx.cuh"

namespace kda {

__device__ unsigned int g_device_error = 0;

namespace {

using namespace tc;

constexpr int kPrepThreads = 256;
constexpr int kStateThreads = 128;
constexpr int kThreads = kPrepThreads + kStateThreads;
constexpr int C = 64;
constexpr int D = 128;
constexpr int BAR_PREP = 1;
constexpr int BAR_STATE = 2;
constexpr float kLog2e = 1.4426950408889634f;

// Shared-memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_AINTRA = 0;        // [128 rows][K=128]  K e^L (rows 0-63), Q e^L (64-127)
constexpr uint32_t OFF_KRCAT = 32768;     // [160 rows][K=128]  K_R' e^{P_R'-G}, R' = 0..3
constexpr uint32_t OFF_AKK = 0;           //   alias after (I): fp32 [64][68] beta-scaled A_kk
constexpr uint32_t OFF_TINV = 17408;      //   alias after (I): fp32 [64][68] T
constexpr uint32_t OFF_KGT = 73728;       // [128 rows][K=64]   (K Gamma)^T
constexpr uint32_t OFF_VT = 90112;        // [128 rows][K=64]   V^T
constexpr uint32_t OFF_TB = 106496;       // [64 rows][K=64]    T Diag(beta)
constexpr uint32_t OFF_QG = 114688;       // 2 x [64 rows][K=128]  Q Gamma
constexpr uint32_t OFF_KP = 147456;       // 2 x [128 rows][K=64]  K'^T
constexpr uint32_t OFF_AQK = 180224;      // 2 x [64 rows][K=64]   A_qk (lower, diagonal kept)
constexpr uint32_t OFF_W = 196608;        // [128 K-rows][N=64] MN-major, -W
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t MISC_RK = 0;           // float[64]
constexpr uint32_t MISC_BETA = 256;       // float[64]
constexpr uint32_t MISC_RED = 512;        // float[8 warps][16 tokens][2]
constexpr uint32_t MISC_TSUM = 1536;      // float[4][128] tile sums (log2 units)
constexpr uint32_t MISC_GAM = 3584;       // float[2][128] gamma_C per buffer
constexpr uint32_t MISC_X = 4608;         // float[3][16][17] solve scratch
constexpr uint32_t MISC_RQ = 7872;        // float[64]
constexpr uint32_t MISC_BAR = 8192;       // 8 mbarriers
constexpr uint32_t MISC_TMEM = 8256;      // uint32
constexpr uint32_t MISC_ABORT = 8260;     // int
constexpr uint32_t SMEM_BYTES = OFF_MISC + 8320 + 1024;   // + alignment slack
constexpr int LDA = 68;                   // fp32 row stride of A_kk / T

constexpr int MB_MMA_P = 0, MB_MMA_S = 1, MB_READY = 2, MB_FREE = 4, MB_WFREE = 6;

// TMEM columns.
constexpr uint32_t COL_ST = 0;            // 128: S^T fp32
constexpr uint32_t COL_SBF = 128;         // 64: S^T packed bf16 (A operand)
constexpr uint32_t COL_UBF = 192;         // 32: U^T packed bf16 (A operand)
constexpr uint32_t COL_UT = 224;          // 2 x 64: Ut^T -> U^T -> O^T, per buffer
constexpr uint32_t COL_INTRA = 352;       // 160: A_kk / A_qk products
constexpr uint32_t COL_WT = 352;          // 64: W^T (after the A readout)
constexpr uint32_t TMEM_COLS = 512;

// Row offset of block R' in the concatenated B operand of (I): 16 * R' (R' + 1) / 2.
__host__ __device__ constexpr int kr_off(int r) { return 8 * r * (r + 1); }
constexpr uint32_t kWaitLimit = 1u << 24;

struct Ctx {
    uint8_t *sm;
    uint32_t sbase, tm;
    volatile int *abort_flag;
    int chain, b, hv, h, T, nchunks;
    bool trans;
};

__device__ __forceinline__ uint32_t bar_addr(const Ctx &x, int i) {
    return x.sbase + OFF_MISC + MISC_BAR + 8u * (uint32_t)i;
}

// Bounded wait that also gives up when the other role has aborted.
__device__ __forceinline__ bool wait_bar(const Ctx &x, uint32_t mbar, uint32_t parity) {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (mbar_try_wait(mbar, parity)) return true;
        if (*x.abort_flag) return false;
        if (i >= 16) __nanosleep(128);
    }
    *x.abort_flag = 1;
    return false;
}

__device__ __forceinline__ void st_u32(uint8_t *base, uint32_t off, uint32_t v) {
    *reinterpret_cast<uint32_t *>(base + off) = v;
}
__device__ __forceinline__ void st_u128(uint8_t *base, uint32_t off, uint4 v) {
    *reinterpret_cast<uint4 *>(base + off) = v;
}
__device__ __forceinline__ uint4 pack8(const float *v) {
    uint4 w;
    w.x = pack_bf16x2(v[0], v[1]);
    w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]);
    w.w = pack_bf16x2(v[6], v[7]);
    return w;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// =====================================================================
// Prep role: warps 0-7.
// =====================================================================
__device__ __forceinline__ void prep_role(const ChunkParams &p, const Ctx &x, int tid) {
    uint8_t *sm = x.sm;
    const int lane = tid & 31, warp = tid >> 5;
    const int R = tid >> 6;                 // 16-token tile
    const int cp = tid & 63;                // channel pair
    const int c0 = 2 * cp;
    const int kb = c0 >> 6;                 // K block of this channel pair in K=128 tiles
    const uint32_t sw_base = (uint32_t)((c0 & 63) >> 3);
    const uint32_t within = (uint32_t)((c0 & 7) * 2);
    float *rk_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_RK);
    float *rq_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_RQ);
    float *beta_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_BETA);
    float *red_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_RED);
    float *tsum_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_TSUM);
    float *gam_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_GAM);
    float *X_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_X);
    float *Akk = reinterpret_cast<float *>(sm + OFF_AKK);
    float *Tm = reinterpret_cast<float *>(sm + OFF_TINV);
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(p.q);
    const __nv_bfloat16 *k = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *v = static_cast<const __nv_bfloat16 *>(p.v);
    const __nv_bfloat16 *gz = static_cast<const __nv_bfloat16 *>(p.g);
    const __nv_bfloat16 *bl = static_cast<const __nv_bfloat16 *>(p.beta);

    // Gate in log2 units: g2 = g_min log2(e) / (1 + 2^-(A1 z + B1)), A1 = exp(A_log) log2(e).
    const float A1 = p.gate_in ? expf(p.A_log[x.hv]) * kLog2e : 0.f;
    const float b0 = (p.gate_in && p.dt_bias) ? p.dt_bias[(size_t)x.hv * D + c0] : 0.f;
    const float b1 = (p.gate_in && p.dt_bias) ? p.dt_bias[(size_t)x.hv * D + c0 + 1] : 0.f;
    const float B10 = b0 * A1, B11 = b1 * A1;
    const float gmin2 = p.g_min * kLog2e;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t ph_mma = 0;

    for (int m = 0; m < x.nchunks; ++m) {
        const int t0 = m * C;
        const int Cc = min(C, x.T - t0);
        const int buf = m & 1;

        // ---------------- loads + gate + norm partials --------------------
        uint32_t qw[16], kw[16], vw[16];
        float g2[16][2];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int t = R * 16 + i;
            uint32_t a = 0, bb = 0, z = 0, vv = 0;
            if (t < Cc) {
                const size_t tok = (size_t)x.b * x.T + t0 + t;
                a = *reinterpret_cast<const uint32_t *>(q + (tok * p.H + x.h) * D + c0);
                bb = *reinterpret_cast<const uint32_t *>(k + (tok * p.H + x.h) * D + c0);
                z = *reinterpret_cast<const uint32_t *>(gz + (tok * p.HV + x.hv) * D + c0);
                if (!x.trans)
                    vv = *reinterpret_cast<const uint32_t *>(v + (tok * p.HV + x.hv) * D + c0);
            }
            qw[i] = a;
            kw[i] = bb;
            vw[i] = vv;
            const float z0 = bf_lo(z), z1 = bf_hi(z);
            float ga, gb;
            if (p.gate_in) {
                ga = gmin2 * rcp_approx(1.f + ex2_approx(-fmaf(z0, A1, B10)));
                gb = gmin2 * rcp_approx(1.f + ex2_approx(-fmaf(z1, A1, B11)));
            } else {
                ga = z0 * kLog2e;
                gb = z1 * kLog2e;
            }
            g2[i][0] = (t < Cc) ? ga : 0.f;
            g2[i][1] = (t < Cc) ? gb : 0.f;
        }
        if (p.l2norm) {
            // Per-token sums of squares over the warp's 64 channels: transpose
            // reduction, 16 values over 32 lanes in 16 shuffles per quantity.
            float sq[16], sk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float qa = bf_lo(qw[i]), qb = bf_hi(qw[i]);
                const float ka = bf_lo(kw[i]), kb2 = bf_hi(kw[i]);
                sq[i] = fmaf(qa, qa, qb * qb);
                sk[i] = fmaf(ka, ka, kb2 * kb2);
            }
#pragma unroll
            for (int step = 0; step < 4; ++step) {
                const int half = 8 >> step;            // values kept after this step
                const int bit = 16 >> step;            // lane bit exchanged
                const bool hi = (lane & bit) != 0;
#pragma unroll
                for (int i = 0; i < half; ++i) {
                    const float sq_send = hi ? sq[i] : sq[i + half];
                    const float sk_send = hi ? sk[i] : sk[i + half];
                    const float sq_keep = hi ? sq[i + half] : sq[i];
                    const float sk_keep = hi ? sk[i + half] : sk[i];
                    sq[i] = sq_keep + __shfl_xor_sync(0xffffffffu, sq_send, bit);
                    sk[i] = sk_keep + __shfl_xor_sync(0xffffffffu, sk_send, bit);
                }
            }
            sq[0] += __shfl_xor_sync(0xffffffffu, sq[0], 1);
            sk[0] += __shfl_xor_sync(0xffffffffu, sk[0], 1);
            // Lane l now holds token ((l>>4)&1)*8 + ((l>>3)&1)*4 + ((l>>2)&1)*2 + ((l>>1)&1).
            if ((lane & 1) == 0) {
                const int tok = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                                ((lane >> 1) & 1);
                red_s[(warp * 16 + tok) * 2 + 0] = sq[0];
                red_s[(warp * 16 + tok) * 2 + 1] = sk[0];
            }
        }
        float ts0 = 0.f, ts1 = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            ts0 += g2[i][0];
            ts1 += g2[i][1];
        }
        tsum_s[R * D + c0] = ts0;
        tsum_s[R * D + c0 + 1] = ts1;
        if (cp < 16) {
            const int t = R * 16 + cp;
            float bb = 0.f;
            if (t < Cc) {
                bb = __bfloat162float(bl[((size_t)x.b * x.T + t0 + t) * p.HV + x.hv]);
                if (p.beta_sigmoid) bb = rcp_approx(1.f + ex2_approx(-bb * kLog2e));
            }
            beta_s[t] = bb;
        }
        named_bar(BAR_PREP, kPrepThreads);
        if (tid < 64) {
            const int t = tid, w0 = (t >> 4) * 2, i = t & 15;
            float rq = 1.f, rk = 1.f;
            if (p.l2norm) {
                rq = rsqrtf(red_s[(w0 * 16 + i) * 2 + 0] + red_s[((w0 + 1) * 16 + i) * 2 + 0] + p.l2_eps);
                rk = rsqrtf(red_s[(w0 * 16 + i) * 2 + 1] + red_s[((w0 + 1) * 16 + i) * 2 + 1] + p.l2_eps);
            }
            rq_s[t] = rq;
            rk_s[t] = rk;
        }
        // Tile-start prefixes P_R' and the chunk total, per channel (log2 units).
        float P2[4][2], GC2[2];
#pragma unroll
        for (int xx = 0; xx < 2; ++xx) {
            float run = 0.f;
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                P2[rr][xx] = run;
                run += tsum_s[rr * D + c0 + xx];
            }
            GC2[xx] = run;
        }
        // The double-buffered operands of this chunk overwrite those of chunk m-2.
        bool ok = true;
        if (m >= 2) ok = wait_bar(x, bar_addr(x, MB_FREE + buf), (uint32_t)(((m - 2) >> 1) & 1));
        if (named_bar_any(BAR_PREP, kPrepThreads, !ok)) break;   // also orders rq/rk writes
        if (R == 0) {
            gam_s[buf * D + c0] = ex2_approx(GC2[0]);
            gam_s[buf * D + c0 + 1] = ex2_approx(GC2[1]);
        }
        float eP[2], eCP[2], Dn[4][2];
#pragma unroll
        for (int xx = 0; xx < 2; ++xx) {
            const float PR = (R == 0) ? P2[0][xx] : (R == 1) ? P2[1][xx] : (R == 2) ? P2[2][xx] : P2[3][xx];
            eP[xx] = ex2_approx(PR);
            eCP[xx] = ex2_approx(GC2[xx] - PR);
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) Dn[rr][xx] = (rr >= R) ? ex2_approx(P2[rr][xx] - PR) : 0.f;
        }

        // ---------------- operand tiles -----------------------------------
        const uint32_t rowR = (uint32_t)(R * 16 * 128);
        const uint32_t a_base = OFF_AINTRA + (uint32_t)kb * 16384u + rowR + within;
        const uint32_t kr_base = OFF_KRCAT + (uint32_t)kb * 20480u + rowR + within;
        const uint32_t qg_base = OFF_QG + (uint32_t)buf * 16384u + (uint32_t)kb * 8192u + rowR + within;
        float kg[2][8], kpv[2][8];
        uint32_t vlo[4], vhi[4];
        float L0 = 0.f, L1 = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int t = R * 16 + i;
            const uint32_t sw = ((sw_base ^ (uint32_t)(i & 7)) << 4) + (uint32_t)(i * 128);
            const float rq = rq_s[t], rk = rk_s[t];
            L0 += g2[i][0];
            L1 += g2[i][1];
            const float e0 = ex2_approx(L0), e1 = ex2_approx(L1);
            const float ei0 = ex2_approx(-L0), ei1 = ex2_approx(-L1);
            const float kh0 = bf_lo(kw[i]) * rk, kh1 = bf_hi(kw[i]) * rk;
            const float qh0 = bf_lo(qw[i]) * rq, qh1 = bf_hi(qw[i]) * rq;
            const float kl0 = kh0 * e0, kl1 = kh1 * e1;
            const float ql0 = qh0 * e0, ql1 = qh1 * e1;
            const float kr0 = kh0 * ei0, kr1 = kh1 * ei1;
            st_u32(sm, a_base + sw, pack_bf16x2(kl0, kl1));
            st_u32(sm, a_base + 8192u + sw, pack_bf16x2(ql0, ql1));
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
                if (rr >= R)
                    st_u32(sm, kr_base + (uint32_t)(kr_off(rr) * 128) + sw,
                           pack_bf16x2(kr0 * Dn[rr][0], kr1 * Dn[rr][1]));
            }
            st_u32(sm, qg_base + sw, pack_bf16x2(ql0 * eP[0], ql1 * eP[1]));
            kg[0][i & 7] = kl0 * eP[0];
            kg[1][i & 7] = kl1 * eP[1];
            kpv[0][i & 7] = kr0 * eCP[0];
            kpv[1][i & 7] = kr1 * eCP[1];
            if ((i & 1) == 1) {
                // value channels c0 (low halves) and c0+1 (high halves) of tokens i-1, i
                vlo[(i & 7) >> 1] = (vw[i - 1] & 0xFFFFu) | (vw[i] << 16);
                vhi[(i & 7) >> 1] = (vw[i - 1] >> 16) | (vw[i] & 0xFFFF0000u);
            }
            if ((i & 7) == 7) {
                const int ch = 2 * R + (i >> 3);
#pragma unroll
                for (int xx = 0; xx < 2; ++xx) {
                    const int row = c0 + xx;
                    const uint32_t o = (uint32_t)(row * 128) + (uint32_t)(((ch ^ (row & 7))) << 4);
                    st_u128(sm, OFF_KGT + o, pack8(kg[xx]));
                    st_u128(sm, OFF_KP + (uint32_t)buf * 16384u + o, pack8(kpv[xx]));
                    if (!x.trans) {
                        const uint32_t *vsrc = xx ? vhi : vlo;
                        st_u128(sm, OFF_VT + o, make_uint4(vsrc[0], vsrc[1], vsrc[2], vsrc[3]));
                    }
                }
            }
        }
        fence_async_smem();
        named_bar(BAR_PREP, kPrepThreads);

        // ---------------- (I) intra-chunk products -------------------------
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id = idesc_bf16(128, 160);
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16(x.tm + COL_INTRA, kmaj_desc(x.sbase + OFF_AINTRA, 128, s),
                         kmaj_desc(x.sbase + OFF_KRCAT, 160, s), id, s > 0);
            mma_commit(bar_addr(x, MB_MMA_P));
        }
        ok = wait_bar(x, bar_addr(x, MB_MMA_P), ph_mma);
        ph_mma ^= 1u;
        if (named_bar_any(BAR_PREP, kPrepThreads, !ok)) break;
        fence_after_sync();

        // ---------------- A_kk (fp32) and A_qk (bf16 operand) -------------
        if (warp < 4) {
            const int rr = (warp & 1) * 32 + lane;        // row of A_kk / A_qk
            const int Rr = rr >> 4;
            const bool is_qk = warp >= 2;
            const int cbeg = (warp & 1) ? 48 : 0;
            const int nld = (warp & 1) ? 7 : 3;
            const float br = beta_s[rr];
            uint8_t *aqk = sm + OFF_AQK + buf * 8192;
            for (int mm = 0; mm < nld; ++mm) {
                const int cb = cbeg + mm * 16;               // warp-uniform column
                const int Rb = cb < 16 ? 0 : cb < 48 ? 1 : cb < 96 ? 2 : 3;   // its block
                float vals[16];
                tmem_ld16(x.tm + lane_base + COL_INTRA + cb, vals);
                if (Rb == Rr) {
                    const int i0 = cb - kr_off(Rb);           // first column index i of the slice
                    if (is_qk) {
                        float vv[16];
#pragma unroll
                        for (int u = 0; u < 16; ++u) vv[u] = (i0 + u <= rr) ? vals[u] : 0.f;
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int ch = (i0 >> 3) + hh;
                            st_u128(aqk, (uint32_t)(rr * 128 + ((ch ^ (rr & 7)) << 4)), pack8(vv + 8 * hh));
                        }
                    } else {
#pragma unroll
                        for (int u4 = 0; u4 < 4; ++u4) {
                            float4 f;
                            f.x = (i0 + 4 * u4 + 0 < rr) ? br * vals[4 * u4 + 0] : 0.f;
                            f.y = (i0 + 4 * u4 + 1 < rr) ? br * vals[4 * u4 + 1] : 0.f;
                            f.z = (i0 + 4 * u4 + 2 < rr) ? br * vals[4 * u4 + 2] : 0.f;
                            f.w = (i0 + 4 * u4 + 3 < rr) ? br * vals[4 * u4 + 3] : 0.f;
                            *reinterpret_cast<float4 *>(Akk + rr * LDA + i0 + 4 * u4) = f;
                        }
                    }
                }
            }
            // Columns past this row's tile are zero.
            for (int i0 = 16 * (Rr + 1); i0 < C; i0 += 16) {
                if (is_qk) {
                    const uint4 z4 = make_uint4(0, 0, 0, 0);
                    st_u128(aqk, (uint32_t)(rr * 128 + ((((i0 >> 3) + 0) ^ (rr & 7)) << 4)), z4);
                    st_u128(aqk, (uint32_t)(rr * 128 + ((((i0 >> 3) + 1) ^ (rr & 7)) << 4)), z4);
                } else {
#pragma unroll
                    for (int u4 = 0; u4 < 4; ++u4)
                        *reinterpret_cast<float4 *>(Akk + rr * LDA + i0 + 4 * u4) = make_float4(0, 0, 0, 0);
                }
            }
        }
        fence_before_sync();
        fence_async_smem();
        named_bar(BAR_PREP, kPrepThreads);

        // ---------------- T = (I + A_kk)^-1, blocked ----------------------
        if (tid < 64) {
            const int bb = tid >> 4, j = tid & 15;
            float xv[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) xv[r] = (r == j) ? 1.f : 0.f;
#pragma unroll
            for (int r = 1; r < 16; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < r; ++i) acc = fmaf(Akk[(16 * bb + r) * LDA + 16 * bb + i], xv[i], acc);
                if (r > j) xv[r] = -acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Tm[(16 * bb + r) * LDA + 16 * bb + j] = (r >= j) ? xv[r] : 0.f;
        }
        named_bar(BAR_PREP, kPrepThreads);
        for (int d = 1; d < 4; ++d) {
            const int er = tid >> 4, ec = tid & 15;
            for (int I = d; I < 4; ++I) {
                const int J = I - d;
                float acc = 0.f;
                for (int K = J; K < I; ++K) {
#pragma unroll
                    for (int mm = 0; mm < 16; ++mm)
                        acc = fmaf(Akk[(16 * I + er) * LDA + 16 * K + mm], Tm[(16 * K + mm) * LDA + 16 * J + ec], acc);
                }
                X_s[((I - d) * 16 + er) * 17 + ec] = acc;
            }
            named_bar(BAR_PREP, kPrepThreads);
            for (int I = d; I < 4; ++I) {
                const int J = I - d;
                float acc = 0.f;
#pragma unroll
                for (int mm = 0; mm < 16; ++mm)
                    acc = fmaf(Tm[(16 * I + er) * LDA + 16 * I + mm], X_s[((I - d) * 16 + mm) * 17 + ec], acc);
                Tm[(16 * I + er) * LDA + 16 * J + ec] = -acc;
            }
            named_bar(BAR_PREP, kPrepThreads);
        }
        {
            // T Diag(beta) -> bf16 K-major [r][i]; row r, columns 16*qq .. 16*qq+15
            const int r = tid >> 2, qq = tid & 3;
            float vv[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int i = 16 * qq + u;
                vv[u] = (i <= r) ? Tm[r * LDA + i] * beta_s[i] : 0.f;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int ch = 2 * qq + hh;
                st_u128(sm, OFF_TB + (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4)), pack8(vv + 8 * hh));
            }
        }
        fence_async_smem();
        named_bar(BAR_PREP, kPrepThreads);

        // ---------------- (II) Ut^T = V^T TB^T, (III) W^T = KG^T TB^T -----
        if (tid == 0) {
            fence_after_sync();
            const uint32_t id = idesc_bf16(128, 64);
            if (!x.trans) {
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    mma_bf16(x.tm + COL_UT + 64u * (uint32_t)buf, kmaj_desc(x.sbase + OFF_VT, 128, s),
                             kmaj_desc(x.sbase + OFF_TB, 64, s), id, s > 0);
            }
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16(x.tm + COL_WT, kmaj_desc(x.sbase + OFF_KGT, 128, s),
                         kmaj_desc(x.sbase + OFF_TB, 64, s), id, s > 0);
            mma_commit(bar_addr(x, MB_MMA_P));
        }
        ok = wait_bar(x, bar_addr(x, MB_MMA_P), ph_mma);
        ph_mma ^= 1u;
        // -W overwrites the buffer MMA (IV) of chunk m-1 reads.
        if (ok && m >= 1) ok = wait_bar(x, bar_addr(x, MB_WFREE), (uint32_t)((m - 1) & 1));
        if (named_bar_any(BAR_PREP, kPrepThreads, !ok)) break;
        fence_after_sync();
        if (warp < 4) {
            const int c = warp * 32 + lane;
            for (int mm = 0; mm < C / 16; ++mm) {
                float vals[16];
                tmem_ld16(x.tm + lane_base + COL_WT + mm * 16, vals);
#pragma unroll
                for (int u = 0; u < 16; ++u) vals[u] = -vals[u];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    st_u128(sm, OFF_W + mnmaj_chunk_off(c, mm * 2 + hh), pack8(vals + 8 * hh));
            }
        }
        fence_before_sync();
        fence_async_smem();
        named_bar(BAR_PREP, kPrepThreads);
        if (tid == 0) mbar_arrive(bar_addr(x, MB_READY + buf));
    }
}

// =====================================================================
// State role: warps 8-11, thread j <-> TMEM lane j <-> value channel j.
// =====================================================================
__device__ __forceinline__ void state_role(const ChunkParams &p, const Ctx &x, int tid) {
    uint8_t *sm = x.sm;
    const int ts = tid - kPrepThreads;      // 0..127
    const int warp = tid >> 5;
    const int j = ts;                        // (warp - 8) * 32 + lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float *gam_s = reinterpret_cast<const float *>(sm + OFF_MISC + MISC_GAM);
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.o);

    // Initial state: S0^T (or the identity for the transition columns, or 0).
    for (int mm = 0; mm < D / 16; ++mm) {
        float vals[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int c = mm * 16 + u;
            float s0 = 0.f;
            if (x.trans) s0 = (c == j) ? 1.f : 0.f;
            else if (p.S0) s0 = p.S0[((size_t)x.chain * D + c) * D + j];
            vals[u] = s0;
        }
        tmem_st16(x.tm + lane_base + COL_ST + mm * 16, vals);
        uint32_t pk[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) pk[u] = pack_bf16x2(vals[2 * u], vals[2 * u + 1]);
        tmem_st8(x.tm + lane_base + COL_SBF + mm * 8, pk);
    }
    tmem_st_wait();
    fence_before_sync();
    named_bar(BAR_STATE, kStateThreads);

    uint32_t ph_s = 0;
    for (int n = 0; n < x.nchunks; ++n) {
        const int t0 = n * C;
        const int Cc = min(C, x.T - t0);
        const int buf = n & 1;
        const uint32_t col_ut = COL_UT + 64u * (uint32_t)buf;
        bool ok = wait_bar(x, bar_addr(x, MB_READY + buf), (uint32_t)((n >> 1) & 1));
        if (named_bar_any(BAR_STATE, kStateThreads, !ok)) break;
        fence_after_sync();

        // (IV) U^T = Ut^T + S^T (-W)
        if (ts == 0) {
            const uint32_t id = idesc_bf16(128, 64, false, /*b_mn_major=*/true);
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16_tmem_a(x.tm + col_ut, x.tm + COL_SBF + s * 8, mnmaj_desc(x.sbase + OFF_W, s),
                                id, (x.trans && s == 0) ? 0u : 1u);
            mma_commit(bar_addr(x, MB_MMA_S));
            mma_commit(bar_addr(x, MB_WFREE));
        }
        // Meanwhile: S^T <- S^T Diag(gamma_C) (fp32, in TMEM).
        for (int mm = 0; mm < D / 16; ++mm) {
            float vals[16];
            tmem_ld16(x.tm + lane_base + COL_ST + mm * 16, vals);
#pragma unroll
            for (int u = 0; u < 16; ++u) vals[u] *= gam_s[buf * D + mm * 16 + u];
            tmem_st16(x.tm + lane_base + COL_ST + mm * 16, vals);
        }
        tmem_st_wait();
        ok = wait_bar(x, bar_addr(x, MB_MMA_S), ph_s);
        ph_s ^= 1u;
        if (named_bar_any(BAR_STATE, kStateThreads, !ok)) break;
        fence_after_sync();

        // U^T -> packed bf16 A operand.
        for (int mm = 0; mm < C / 16; ++mm) {
            float vals[16];
            tmem_ld16(x.tm + lane_base + col_ut + mm * 16, vals);
            uint32_t pk[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) pk[u] = pack_bf16x2(vals[2 * u], vals[2 * u + 1]);
            tmem_st8(x.tm + lane_base + COL_UBF + mm * 8, pk);
        }
        tmem_st_wait();
        fence_before_sync();
        named_bar(BAR_STATE, kStateThreads);

        // (VI) S^T += U^T K'  then  (V) O^T = S^T (Q Gamma)^T + U^T A_qk^T
        if (ts == 0) {
            fence_after_sync();
            const uint32_t id2 = idesc_bf16(128, 128);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16_tmem_a(x.tm + COL_ST, x.tm + COL_UBF + s * 8,
                                kmaj_desc(x.sbase + OFF_KP + 16384u * buf, 128, s), id2, 1u);
            if (!x.trans) {
                const uint32_t id = idesc_bf16(128, 64);
#pragma unroll
                for (int s = 0; s < D / 16; ++s)
                    mma_bf16_tmem_a(x.tm + col_ut, x.tm + COL_SBF + s * 8,
                                    kmaj_desc(x.sbase + OFF_QG + 16384u * buf, 64, s), id, s > 0);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    mma_bf16_tmem_a(x.tm + col_ut, x.tm + COL_UBF + s * 8,
                                    kmaj_desc(x.sbase + OFF_AQK + 8192u * buf, 64, s), id, 1u);
            }
            mma_commit(bar_addr(x, MB_MMA_S));
        }
        ok = wait_bar(x, bar_addr(x, MB_MMA_S), ph_s);
        ph_s ^= 1u;
        if (named_bar_any(BAR_STATE, kStateThreads, !ok)) break;
        fence_after_sync();

        // New S^T as the bf16 operand of the next chunk, then the outputs.
        for (int mm = 0; mm < D / 16; ++mm) {
            float vals[16];
            tmem_ld16(x.tm + lane_base + COL_ST + mm * 16, vals);
            uint32_t pk[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) pk[u] = pack_bf16x2(vals[2 * u], vals[2 * u + 1]);
            tmem_st8(x.tm + lane_base + COL_SBF + mm * 8, pk);
        }
        if (!x.trans) {
            for (int mm = 0; mm < C / 16; ++mm) {
                float vals[16];
                tmem_ld16(x.tm + lane_base + col_ut + mm * 16, vals);
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const int t = mm * 16 + u;
                    if (t < Cc)
                        o[(((size_t)x.b * x.T + t0 + t) * p.HV + x.hv) * D + j] =
                            __float2bfloat16_rn(p.scale * vals[u]);
                }
            }
        }
        tmem_st_wait();
        fence_before_sync();
        named_bar(BAR_STATE, kStateThreads);
        if (ts == 0) mbar_arrive(bar_addr(x, MB_FREE + buf));
    }

    if (!*x.abort_flag) {
        float *out = x.trans ? p.M_T : p.S_T;
        if (out) {
            for (int mm = 0; mm < D / 16; ++mm) {
                float vals[16];
                tmem_ld16(x.tm + lane_base + COL_ST + mm * 16, vals);
#pragma unroll
                for (int u = 0; u < 16; ++u) out[((size_t)x.chain * D + mm * 16 + u) * D + j] = vals[u];
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(ChunkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    Ctx x;
    x.sm = sm;
    x.sbase = smem_addr(sm);
    x.abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + MISC_ABORT);
    x.chain = blockIdx.x;
    x.trans = blockIdx.y == 1;
    x.b = x.chain / p.HV;
    x.hv = x.chain % p.HV;
    x.h = x.hv / p.group;
    x.T = p.T;
    x.nchunks = (p.T + C - 1) / C;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + MISC_TMEM);

    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 7; ++i) mbar_init(bar_addr(x, i), 1);
        *x.abort_flag = 0;
        fence_mbar_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    x.tm = *tmem_slot;

    if (warp < kPrepThreads / 32) prep_role(p, x, tid);
    else state_role(p, x, tid);

    fence_before_sync();
    __syncthreads();
    if (tid == 0 && *x.abort_flag) atomicOr(&g_device_error, 1u);
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(x.tm, TMEM_COLS);
    }
}

}  // namespace

bool chunk_tc_supported(const ChunkParams &p, bool bf16) {
    return bf16 && p.Dk == D && p.Dv == D && p.C == C;
}

cudaError_t launch_chunk_tc(const ChunkParams &p, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(p.B * p.HV, p.M_T ? 2 : 1);
    chunk_tc_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(p);
    return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(cudaStream_t s, unsigned int *out) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(out, g_device_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace kda
