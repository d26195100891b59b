// tcgen05 BF16 chunk kernel for Dk = Dv = 128, chunk C = 64, warp-specialised.
//
// One CTA (640 threads) per (b, hv) chain walks the chunks in order with the
// state on chip: fp32 S^T in tensor memory (lane j = value channel, column c =
// key channel) and a packed-bf16 copy in tensor memory as the MMA A operand.
// With G the in-chunk cumulative sum of the log-decay, tiles of 16 tokens and
// P_R the cumulative sum before tile R (page "KDA 模块交互式演示" section 1.5,
// Eqs. 3-4, with the decay-weighted UT transform; page "Implémenter KDA",
// "La forme par blocs", for U = Ut - W S), the work per chunk splits in two:
//
// prep warps 0-15 (state-independent; run one chunk ahead of the state warps)
//   inputs       q, k, z rows of the chunk by tensor-map TMA (requested a chunk
//                ahead), beta prefetched in a register
//   prologue     L2 norm of q,k; beta = sigmoid; g = g_min sigmoid(exp(A_log)(z + dt_bias))
//   operands     bf16 tiles scaled by exp(G_r - P_R) <= 1 and exp(P_R' - G_i)
//                (<= e^80 inside a tile, <= 1 before it)
//   (I)   MMA    [K e^L ; Q e^L] x [K_R' e^{P_R'-G}]^T    -> A_kk, A_qk (all tiles at once),
//                issued by one lane of warp 15
//   solve        T = (I + tril(Diag(beta) A_kk, -1))^-1: fp32 substitution on the
//                diagonal 16 x 16 blocks, tf32 warp-level MMAs for the rest,
//                written as the bf16 operand T Diag(beta)
// state warps 16-19 (the serial carry, one TMEM lane per value channel)
//   (II)  MMA    Ut^T = V^T (T Diag(beta))^T   (V tile by swizzled TMA) -> TMEM buffer
//   (III) MMA    W^T  = (K Gamma)^T (T Diag(beta))^T, read out as -W (MN-major smem)
//   (IV)  MMA    U^T = Ut^T - S^T W^T        while the state is scaled by gamma_C
//   (VI)  MMA    S^T <- S^T Diag(gamma_C) + U^T K',   K' = K exp(G_C - G)
//   (V)   MMA    O^T = S^T (Q Gamma)^T + U^T A_qk^T   -> o
//
// Every exponent is bounded: inside a 16-token tile |G_r - P_R| <= 16 |g_min| = 80
// (e^80 ~ 5.5e34 < bf16/fp32 max, page "Implémenter KDA" "La décroissance
// bornée"); across tiles the factors are decays <= 1.  Exponentials use base 2:
// the log-decay is carried in log2 units.
//
// Hand-off between the two roles uses mbarriers (READY / FREE and the MMA
// (II)/(III) completion double-buffered by chunk parity); the operands the
// state warps read (Q Gamma, K', A_qk, gamma_C and the Ut^T accumulator) are
// double buffered.  Every wait is bounded; if one gives up, the CTA records the
// device error word, both roles leave their loops, in-flight MMAs and tensor
// copies are drained (bounded), the TMEM is freed and the CTA returns.
//
// All MMAs are cta_group::1, M = 128, BF16 x BF16 -> FP32 in TMEM; shared
// operands use the 128-byte-swizzle layouts of tc_ptx.cuh (K-major, or
// MN-major for V, K Gamma, K' and -W).  When M_T is requested a second CTA per
// chain (blockIdx.y == 1) runs the same recurrence on the transition columns:
// v = 0 and S0 = I, no o.  With o == NULL (only the states are wanted) MMA (V)
// and the o rows are skipped.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_internal.cuh"
#include "tc_ptx.cuh"

namespace kda {

__device__ unsigned int g_device_error = 0;

namespace {

using namespace tc;

constexpr int kPrepThreads = 512;
constexpr int kStateThreads = 128;
constexpr int kThreads = kPrepThreads + kStateThreads;
constexpr int C = 64;
constexpr int D = 128;
constexpr int BAR_PREP = 1;
constexpr int BAR_STATE = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Shared-memory map (bytes from a 1024-aligned base).
constexpr uint32_t OFF_AINTRA = 0;        // [128 rows][K=128]  K e^L (rows 0-63), Q e^L (64-127)
constexpr uint32_t OFF_KRCAT = 32768;     // [160 rows][K=128]  K_R' e^{P_R'-G}, R' = 0..3
constexpr uint32_t OFF_AKK = 0;           //   alias after (I): fp32 [64][68] beta-scaled A_kk
constexpr uint32_t OFF_STAGE_Z = 0;       //   alias after the solve: raw z rows of the next chunk [64][256 B]
constexpr uint32_t OFF_STAGE_Q = 36864;   //   alias after (I): raw q rows of the next chunk
constexpr uint32_t OFF_STAGE_K = 53248;   //   ... raw k rows
constexpr uint32_t OFF_TINV = 17408;      //   alias after (I): fp32 [64][68] T
constexpr uint32_t OFF_KGT = 73728;       // K Gamma, token-major (MN-major A of (III): M = 128 channels, K = 64)
constexpr uint32_t OFF_VT = 90112;        // V, token-major (MN-major A of (II)), loaded by TMA with the 128-byte swizzle
constexpr uint32_t OFF_TB = 106496;       // [64 rows][K=64]    T Diag(beta)
constexpr uint32_t OFF_QG = 114688;       // 2 x [64 rows][K=128]  Q Gamma
constexpr uint32_t OFF_KP = 147456;       // 2 x K', token-major (MN-major B of (VI): N = 128 channels, K = 64)
constexpr uint32_t OFF_AQK = 180224;      // 2 x [64 rows][K=64]   A_qk (lower, diagonal kept)
constexpr uint32_t OFF_W = 196608;        // [128 K-rows][N=64] MN-major, -W; after (IV): o rows [64][128] bf16
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t MISC_RK = 0;           // float[64]
constexpr uint32_t MISC_BETA = 256;       // float[64]
constexpr uint32_t MISC_QSUM = 512;       // float[16 quarters][128] (log2 units)
constexpr uint32_t MISC_GAM = 8704;       // float[2][128] gamma_C per buffer
constexpr uint32_t MISC_RQ = 9728;        // float[64] q norm factor times the output scale
constexpr uint32_t MISC_TSUM = 9984;      // float[4][128] tile sums (log2 units)
constexpr uint32_t MISC_BAR = 12032;      // 14 mbarriers
constexpr uint32_t MISC_TMEM = 12144;     // uint32
constexpr uint32_t MISC_ABORT = 12148;    // int
constexpr uint32_t MISC_RANGE = 12152;    // int: a caller-given log-decay was below g_min
constexpr uint32_t SMEM_BYTES = OFF_MISC + 12160 + 1024;   // + alignment slack
constexpr int LDA = 68;                   // fp32 row stride of A_kk / T

// Barriers used by both roles in every chunk are double-buffered by chunk
// parity (READY, FREE, MMA_W), so neither role can fall two phases behind.
constexpr int MB_MMA_P = 0, MB_MMA_S = 1, MB_READY = 2, MB_FREE = 4, MB_MMA_W = 6, MB_ODONE = 8;
constexpr int MB_LZV = 9, MB_LQK = 10, MB_LV = 11;  // raw z rows / raw q, k rows / V tile of a chunk
constexpr int MB_WTFREE = 12;             // W^T read out of TMEM by the state warps
constexpr int MB_DRAIN = 13;              // exit: every MMA the state warps issued is complete
constexpr int kNumBars = 14;

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

// Kernel parameters: the chunk arguments plus tensor maps of q, k (per key head)
// and z, v, o (per value head), each viewed as [B*T tokens][heads][128 channels]
// with a [64 tokens][1][128] box.
struct TcParams {
    ChunkParams p;
    CUtensorMap tm[5];   // q, k, z, v, o
    int o_tma;           // o rows of whole chunks leave by tensor store through tm[4]
};

struct Ctx {
    uint8_t *sm;
    uint32_t sbase, tm;
    volatile int *abort_flag;
    int chain, b, hv, h, T, nchunks;
    bool trans;     // the transition CTA of a chain (v = 0, S0 = I)
    bool want_o;    // o is written (not for the transition CTA, nor when o == NULL)
};

__device__ __forceinline__ uint32_t bar_addr(const Ctx &x, int i) {
    return x.sbase + OFF_MISC + MISC_BAR + 8u * (uint32_t)i;
}

// Bounded wait that also gives up when the other role has aborted: spins on
// the mbarrier for at most about two seconds of SM clock.  The exit drains
// below use the suspend hint (kSuspendNs per try, kWaitTries tries).
constexpr uint32_t kSuspendNs = 500000;
constexpr uint32_t kWaitTries = 4000;
constexpr long long kWaitCycles = 4000000000LL;
__device__ __forceinline__ bool wait_bar(const Ctx &x, uint32_t mbar, uint32_t parity) {
    if (mbar_try_wait(mbar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(mbar, parity)) {
        if (*x.abort_flag) return false;
        if (clock64() - t0 > kWaitCycles) {
            *x.abort_flag = 1;
            return false;
        }
    }
    return true;
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
// Prep role: warps 0-15.  Thread (R, qt, cq) owns tokens 16R + 4qt .. +3 and
// key/value channels 4cq .. 4cq+3 of each chunk; warp w = (R, qt) covers whole
// 128-channel rows, so every global load is one contiguous 256-byte row.
// =====================================================================
__device__ __forceinline__ uint2 pack4(float a, float b, float c, float d) {
    return make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
}
// Elementwise bf16 x bf16 product of two packed 4-element groups (rounded to nearest).
__device__ __forceinline__ uint2 bmul4(uint2 a, uint2 b) {
    __nv_bfloat162 r0 = __hmul2(*reinterpret_cast<__nv_bfloat162 *>(&a.x), *reinterpret_cast<__nv_bfloat162 *>(&b.x));
    __nv_bfloat162 r1 = __hmul2(*reinterpret_cast<__nv_bfloat162 *>(&a.y), *reinterpret_cast<__nv_bfloat162 *>(&b.y));
    return make_uint2(*reinterpret_cast<uint32_t *>(&r0), *reinterpret_cast<uint32_t *>(&r1));
}
__device__ __forceinline__ void st_u64(uint8_t *base, uint32_t off, uint2 v) {
    *reinterpret_cast<uint2 *>(base + off) = v;
}

// One warp: d (a 16x8 tile) += A (16 x 8KS) B (8KS x 8), both fp32 in shared
// memory with row stride LDA, on the tensor cores in tf32 (mma.sync m16n8k8).
template <int KS>
__device__ __forceinline__ void warp_mm16x8(float d[4], const float *A, const float *B, int lane) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
        const float *a = A + g * LDA + 8 * kk + t;
        const float *b = B + (8 * kk + t) * LDA + g;
        const uint32_t af[4] = {to_tf32(a[0]), to_tf32(a[8 * LDA]), to_tf32(a[4]), to_tf32(a[8 * LDA + 4])};
        const uint32_t bf[2] = {to_tf32(b[0]), to_tf32(b[4 * LDA])};
        mma_tf32_16x8x8(d, af, bf);
    }
}
// Element (r, i) of the bf16 K-major 64 x 64 tile T Diag(beta).
__device__ __forceinline__ uint32_t tb_off(int r, int i) {
    return OFF_TB + (uint32_t)(r * 128 + ((((i >> 3) ^ (r & 7))) << 4) + (i & 7) * 2);
}
// A 16x8 fragment of T (rows row0.., columns col0..), times -1 and Diag(beta),
// into the bf16 tile (one 32-bit store per row pair of columns).
__device__ __forceinline__ void warp_tb16x8(uint8_t *sm, int row0, int col0, const float d[4], const float *beta_s,
                                            int lane) {
    const int g = lane >> 2, t = lane & 3, c = col0 + 2 * t;
    const float b0 = beta_s[c], b1 = beta_s[c + 1];
    *reinterpret_cast<uint32_t *>(sm + tb_off(row0 + g, c)) = pack_bf16x2(-d[0] * b0, -d[1] * b1);
    *reinterpret_cast<uint32_t *>(sm + tb_off(row0 + g + 8, c)) = pack_bf16x2(-d[2] * b0, -d[3] * b1);
}
// D (16x8 tile in shared memory) = sgn * d, or D += sgn * d.
__device__ __forceinline__ void warp_st16x8(float *D, const float d[4], float sgn, bool accumulate, int lane) {
    const int g = lane >> 2, t = lane & 3;
    float2 *p0 = reinterpret_cast<float2 *>(D + g * LDA + 2 * t);
    float2 *p1 = reinterpret_cast<float2 *>(D + (g + 8) * LDA + 2 * t);
    float2 v0 = make_float2(sgn * d[0], sgn * d[1]), v1 = make_float2(sgn * d[2], sgn * d[3]);
    if (accumulate) {
        const float2 o0 = *p0, o1 = *p1;
        v0.x += o0.x; v0.y += o0.y; v1.x += o1.x; v1.y += o1.y;
    }
    *p0 = v0;
    *p1 = v1;
}

__device__ __forceinline__ void prep_role(const ChunkParams &p, const CUtensorMap *tmaps, const Ctx &x, int tid) {
    uint8_t *sm = x.sm;
    const int lane = tid & 31, warp = tid >> 5;
    const int R = warp >> 2;                // 16-token tile
    const int qt = warp & 3;                // quarter of the tile: tokens 16R + 4qt .. +3
    const int cq = lane;                    // channel quad: 4cq .. 4cq+3
    const int c0 = 4 * cq;
    const int kb = cq >> 4;                 // K block of the quad in K=128 tiles
    const uint32_t chunk_c = (uint32_t)((cq & 15) >> 1);
    const uint32_t within = (uint32_t)((cq & 1) * 8);
    const int tq = R * 16 + qt * 4;         // first token of this thread
    float *rk_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_RK);
    float *rq_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_RQ);
    float *beta_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_BETA);
    float *qsum_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_QSUM);
    float *tsum_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_TSUM);
    float *gam_s = reinterpret_cast<float *>(sm + OFF_MISC + MISC_GAM);
    float *Akk = reinterpret_cast<float *>(sm + OFF_AKK);
    float *Tm = reinterpret_cast<float *>(sm + OFF_TINV);
    const __nv_bfloat16 *bl = static_cast<const __nv_bfloat16 *>(p.beta);

    // Gate in log2 units, A1 = exp(A_log) log2(e): bounded, g2 = g_min log2(e) /
    // (1 + 2^-(A1 z + B1)) with B1 = A1 dt_bias; softplus, g2 = -A1 softplus(z + B1)
    // with B1 = dt_bias.
    const float A1 = p.gate_in ? expf(p.A_log[x.hv]) * kLog2e : 0.f;
    float B1[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
        B1[u] = (p.gate_in && p.dt_bias)
                    ? p.dt_bias[p.g_per_head ? (size_t)x.hv : (size_t)x.hv * D + c0 + u] * (p.gate_in == 1 ? A1 : 1.f)
                    : 0.f;
    const float gmin2 = p.g_min * kLog2e;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t ph_mma = 0;
    bool below_gmin = false;

    // Raw rows of each chunk arrive in shared memory by tensor-map copies (one
    // [64 x 128] box per tensor) issued one chunk ahead: q, k as soon as MMA (I)
    // has finished with its operand tiles (counted on MB_LQK), z, v once the
    // solve no longer needs its workspace (MB_LZV).  Whole boxes are counted,
    // rows past the tensor included (zero-filled).
    // Issued by one lane of the last prep warp, which has no part in the
    // diagonal blocks of the solve nor in issuing MMAs.
    auto issue_rows = [&](int mc, bool zv) {
        if (tid != kPrepThreads - 32) return;
        const int row0 = x.b * x.T + mc * C;
        if (zv) {
            const uint32_t bar = bar_addr(x, MB_LZV);
            if (p.g_per_head) {          // one gate value per token: read directly by read_z
                mbar_arrive(bar);
            } else {
                mbar_arrive_expect_tx(bar, (uint32_t)(C * D * 2));
                tma_load_3d(x.sbase + OFF_STAGE_Z, &tmaps[2], 0, x.hv, row0, bar);
            }
        } else {
            const uint32_t bar = bar_addr(x, MB_LQK);
            mbar_arrive_expect_tx(bar, (uint32_t)(2 * C * D * 2));
            tma_load_3d(x.sbase + OFF_STAGE_Q, &tmaps[0], 0, x.h, row0, bar);
            tma_load_3d(x.sbase + OFF_STAGE_K, &tmaps[1], 0, x.h, row0, bar);
        }
    };
    // V goes straight into the operand tile of MMA (II): two [64 tokens x 64
    // channels] boxes whose 128-byte swizzle is the operand layout.
    auto issue_v = [&](int mc) {
        if (tid != kPrepThreads - 32 || x.trans) return;
        const int row0 = x.b * x.T + mc * C;
        const uint32_t bar = bar_addr(x, MB_LV);
        mbar_arrive_expect_tx(bar, (uint32_t)(C * D * 2));
        tma_load_3d(x.sbase + OFF_VT, &tmaps[3], 0, x.hv, row0, bar);
        tma_load_3d(x.sbase + OFF_VT + 8192u, &tmaps[3], 64, x.hv, row0, bar);
    };
    uint2 qw[4], kw[4], zw[4];
    auto read_z = [&](int mc, int lCc) {
        if (p.g_per_head) {              // the token's one value, in all four channel slots
            const uint16_t *gz = static_cast<const uint16_t *>(p.g);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = tq + i;
                const uint32_t bits = t < lCc ? gz[((size_t)x.b * x.T + (size_t)mc * C + t) * p.HV + x.hv] : 0u;
                zw[i] = make_uint2(bits | (bits << 16), bits | (bits << 16));
            }
            return;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = tq + i;
            const uint32_t off = (uint32_t)t * 256u + 8u * (uint32_t)cq;
            zw[i] = t < lCc ? *reinterpret_cast<const uint2 *>(sm + OFF_STAGE_Z + off) : make_uint2(0, 0);
        }
    };
    auto read_qk = [&](int lCc) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = tq + i;
            const uint32_t off = (uint32_t)t * 256u + 8u * (uint32_t)cq;
            const bool in = t < lCc;
            qw[i] = in ? *reinterpret_cast<const uint2 *>(sm + OFF_STAGE_Q + off) : make_uint2(0, 0);
            kw[i] = in ? *reinterpret_cast<const uint2 *>(sm + OFF_STAGE_K + off) : make_uint2(0, 0);
        }
    };
    // Chunks whose rows were requested / have arrived, per barrier.
    int issued = 0;                        // chunks whose rows were requested
    int v_issued = 0;                      // chunks whose V tile was requested
    int mi_issued = 0;                     // chunks whose MMA (I) was issued (by this thread)
    if (tid == kPrepThreads - 32)
        for (int i = 0; i < 4; ++i)
            if (i != 2 || !p.g_per_head) prefetch_tensormap(&tmaps[i]);
    if (x.nchunks > 0) {
        issue_rows(0, true);
        issue_rows(0, false);
        issue_v(0);
        issued = v_issued = 1;
    }
    // beta of this thread's token (lanes 28-31), loaded one chunk ahead.
    auto load_beta = [&](int mc) {
        const int t = mc * C + tq + (lane - 28);
        return (lane >= 28 && t < x.T) ? bl[((size_t)x.b * x.T + t) * p.HV + x.hv] : __float2bfloat16_rn(0.f);
    };
    __nv_bfloat16 beta_next = load_beta(0);
    // T Diag(beta) keeps a zero upper triangle; the solve writes only the lower one.
    st_u128(sm, OFF_TB + 16u * (uint32_t)tid, make_uint4(0, 0, 0, 0));   // 512 x 16 B
    for (int m = 0; m < x.nchunks; ++m) {
        const int t0 = m * C;
        const int Cc = min(C, x.T - t0);
        const int buf = m & 1;
        // This chunk's raw q, k rows have landed; the double-buffered operands
        // (and the Ut^T accumulator) of chunk m-2 are free once the state warps
        // have finished that chunk.
        bool ok = wait_bar(x, bar_addr(x, MB_LQK), (uint32_t)(m & 1));
        if (ok && m >= 2) ok = wait_bar(x, bar_addr(x, MB_FREE + buf), (uint32_t)(((m - 2) >> 1) & 1));
        if (named_bar_any(BAR_PREP, kPrepThreads, !ok)) break;
        fence_after_sync();
        read_qk(Cc);

        // ---------------- norms, gate, quarter sums ----------------------
        if (p.l2norm) {
            // Per-token sums of squares over the warp's 128 channels: 4 values
            // over 32 lanes by transpose reduction (6 shuffles per quantity).
            float sq[4], sk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float q0 = bf_lo(qw[i].x), q1 = bf_hi(qw[i].x), q2 = bf_lo(qw[i].y), q3 = bf_hi(qw[i].y);
                const float k0 = bf_lo(kw[i].x), k1 = bf_hi(kw[i].x), k2 = bf_lo(kw[i].y), k3 = bf_hi(kw[i].y);
                sq[i] = fmaf(q0, q0, fmaf(q1, q1, fmaf(q2, q2, q3 * q3)));
                sk[i] = fmaf(k0, k0, fmaf(k1, k1, fmaf(k2, k2, k3 * k3)));
            }
#pragma unroll
            for (int step = 0; step < 2; ++step) {
                const int half = 2 >> step;
                const int bit = 16 >> step;
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
#pragma unroll
            for (int bit = 4; bit > 0; bit >>= 1) {
                sq[0] += __shfl_xor_sync(0xffffffffu, sq[0], bit);
                sk[0] += __shfl_xor_sync(0xffffffffu, sk[0], bit);
            }
            // Lane l holds token ((l >> 4) & 1) * 2 + ((l >> 3) & 1) of this thread's four.
            if ((lane & 7) == 0) {
                const int t = tq + ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
                rq_s[t] = rsqrtf(sq[0] + p.l2_eps) * p.scale;
                rk_s[t] = rsqrtf(sk[0] + p.l2_eps);
            }
        } else if (lane < 4) {
            rq_s[tq + lane] = p.scale;
            rk_s[tq + lane] = 1.f;
        }
        // The z rows (requested after the previous chunk's solve) arrive while
        // the norms are computed.
        const bool ok_zv = wait_bar(x, bar_addr(x, MB_LZV), (uint32_t)(m & 1));
        read_z(m, Cc);
        float g2[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float zz[4] = {bf_lo(zw[i].x), bf_hi(zw[i].x), bf_lo(zw[i].y), bf_hi(zw[i].y)};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float g;
                if (p.gate_in == 1) {
                    g = gmin2 * rcp_approx(1.f + ex2_approx(-fmaf(zz[u], A1, B1[u])));
                } else {
                    if (p.gate_in == 2) {
                        // softplus(x) = max(x, 0) + ln(1 + e^-|x|), unbounded below
                        const float xx = zz[u] + B1[u];
                        g = -A1 * (fmaxf(xx, 0.f) + kLn2 * lg2_approx(1.f + ex2_approx(-fabsf(xx) * kLog2e)));
                    } else {
                        g = zz[u] * kLog2e;
                    }
                    // the exponent bound needs g >= g_min: clamped, and reported
                    below_gmin = below_gmin || (tq + i < Cc && g < gmin2);
                    g = fmaxf(g, gmin2);
                }
                g2[i][u] = (tq + i < Cc) ? g : 0.f;
            }
        }
        {
            float4 qs;
            qs.x = g2[0][0] + g2[1][0] + g2[2][0] + g2[3][0];
            qs.y = g2[0][1] + g2[1][1] + g2[2][1] + g2[3][1];
            qs.z = g2[0][2] + g2[1][2] + g2[2][2] + g2[3][2];
            qs.w = g2[0][3] + g2[1][3] + g2[2][3] + g2[3][3];
            *reinterpret_cast<float4 *>(qsum_s + (R * 4 + qt) * D + c0) = qs;
        }
        if (lane >= 28) {
            const int t = tq + (lane - 28);
            float bb = 0.f;
            if (t < Cc) {
                bb = __bfloat162float(beta_next);
                if (p.beta_sigmoid) bb = rcp_approx(1.f + ex2_approx(-bb * kLog2e));
            }
            beta_s[t] = bb;
        }
        if (named_bar_any(BAR_PREP, kPrepThreads, !ok_zv)) break;

        // Per channel: tile-start prefixes P_R', the chunk total, and the start of
        // this thread's quarter inside its tile (log2 units).
        if (qt == 0) {
            // Tile sums of this warp's tile, for all 128 channels.
            float4 ts = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                const float4 s4 = *reinterpret_cast<const float4 *>(qsum_s + (R * 4 + qq) * D + c0);
                ts.x += s4.x; ts.y += s4.y; ts.z += s4.z; ts.w += s4.w;
            }
            *reinterpret_cast<float4 *>(tsum_s + R * D + c0) = ts;
        }
        float Lst[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int qq = 0; qq < 3; ++qq) {
            if (qq < qt) {
                const float4 s4 = *reinterpret_cast<const float4 *>(qsum_s + (R * 4 + qq) * D + c0);
                Lst[0] += s4.x; Lst[1] += s4.y; Lst[2] += s4.z; Lst[3] += s4.w;
            }
        }
        // ---------------- operand tiles -----------------------------------
        // Base operands in fp32, rounded once: K e^L, Q e^L, K e^-L (tile anchors).
        // They need only this tile's prefix, so they are built while the tile
        // sums of the other warps land; the anchored block of this tile
        // (factor e^0 = 1) is stored with them.  Derived operands are bf16 x
        // bf16 products with the decay factors: K_R' (x e^{P_R'-P_R}, R' > R)
        // below, Q Gamma and K Gamma (x e^{P_R}), K' (x e^{G_C-P_R}) while MMA (I) runs.
        const uint32_t a_base = OFF_AINTRA + (uint32_t)kb * 16384u + within;
        const uint32_t kr_base = OFF_KRCAT + (uint32_t)kb * 20480u + within;
        const uint32_t qg_base = OFF_QG + (uint32_t)buf * 16384u + (uint32_t)kb * 8192u + within;
        uint2 klp[4], qlp[4], krp[4];
        {
            float L[4] = {Lst[0], Lst[1], Lst[2], Lst[3]};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = tq + i;
                const uint32_t roff = (uint32_t)(t * 128) + ((chunk_c ^ (uint32_t)(t & 7)) << 4);
                const float rq = rq_s[t], rk = rk_s[t];
                const float kv4[4] = {bf_lo(kw[i].x), bf_hi(kw[i].x), bf_lo(kw[i].y), bf_hi(kw[i].y)};
                const float qv4[4] = {bf_lo(qw[i].x), bf_hi(qw[i].x), bf_lo(qw[i].y), bf_hi(qw[i].y)};
                float kl[4], ql[4], kr[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    L[u] += g2[i][u];
                    const float e = ex2_approx(L[u]), ei = ex2_approx(-L[u]);
                    const float kh = kv4[u] * rk;
                    kl[u] = kh * e;
                    ql[u] = qv4[u] * rq * e;
                    kr[u] = kh * ei;
                }
                klp[i] = pack4(kl[0], kl[1], kl[2], kl[3]);
                qlp[i] = pack4(ql[0], ql[1], ql[2], ql[3]);
                krp[i] = pack4(kr[0], kr[1], kr[2], kr[3]);
                st_u64(sm, a_base + roff, klp[i]);
                st_u64(sm, a_base + 8192u + roff, qlp[i]);
                st_u64(sm, kr_base + (uint32_t)(kr_off(R) * 128) + roff, krp[i]);
            }
        }
        named_bar(BAR_PREP, kPrepThreads);
        float Pc[4][4], GC[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
            const float4 t4 = *reinterpret_cast<const float4 *>(tsum_s + rr * D + c0);
            Pc[rr][0] = GC[0]; Pc[rr][1] = GC[1]; Pc[rr][2] = GC[2]; Pc[rr][3] = GC[3];
            GC[0] += t4.x; GC[1] += t4.y; GC[2] += t4.z; GC[3] += t4.w;
        }
        // Decay factors, packed as bf16 pairs for the derived operands.
        uint2 ePp, eCPp, Dnp[4];
        {
            float eP[4], eCP[4], Dn[4][4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float PR = (R == 0) ? Pc[0][u] : (R == 1) ? Pc[1][u] : (R == 2) ? Pc[2][u] : Pc[3][u];
                eP[u] = ex2_approx(PR);
                eCP[u] = ex2_approx(GC[u] - PR);
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) Dn[rr][u] = (rr > R) ? ex2_approx(Pc[rr][u] - PR) : 0.f;
                if (R == 0 && qt == 0) gam_s[buf * D + c0 + u] = ex2_approx(GC[u]);
            }
            ePp = pack4(eP[0], eP[1], eP[2], eP[3]);
            eCPp = pack4(eCP[0], eCP[1], eCP[2], eCP[3]);
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) Dnp[rr] = pack4(Dn[rr][0], Dn[rr][1], Dn[rr][2], Dn[rr][3]);
        }
        // The later tiles' anchored blocks K_R' (R' > R) of this thread's tokens.
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int t = tq + i;
            const uint32_t roff = (uint32_t)(t * 128) + ((chunk_c ^ (uint32_t)(t & 7)) << 4);
#pragma unroll
            for (int rr = 1; rr < 4; ++rr)
                if (rr > R) st_u64(sm, kr_base + (uint32_t)(kr_off(rr) * 128) + roff, bmul4(krp[i], Dnp[rr]));
        }
        fence_async_smem();
        named_bar(BAR_PREP, kPrepThreads);

        // ---------------- (I) intra-chunk products -------------------------
        // Issued by lane 0 of the last prep warp, whose own share of the work
        // below overlaps the MMA.  MMA (I) overwrites the TMEM columns of W^T:
        // the state warps must have read out chunk m-1's.
        if (tid == kPrepThreads - 32 &&
            (m == 0 || wait_bar(x, bar_addr(x, MB_WTFREE), (uint32_t)((m - 1) & 1)))) {
            fence_after_sync();
            const uint32_t id = idesc_bf16(128, 160);
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16(x.tm + COL_INTRA, kmaj_desc(x.sbase + OFF_AINTRA, 128, s),
                         kmaj_desc(x.sbase + OFF_KRCAT, 160, s), id, s > 0);
            mma_commit(bar_addr(x, MB_MMA_P));
            mi_issued = m + 1;
        }
        // Meanwhile: Q Gamma, K Gamma and K', all token-major (K Gamma and K'
        // serve as MN-major operands, whose byte image is the same).  K Gamma
        // and V were read by MMAs (II)/(III) of chunk m-1, finished long ago.
        if (m >= 1) {
            // MMA (II) of chunk m-1 has released the V tile: load this chunk's.
            if (wait_bar(x, bar_addr(x, MB_MMA_W + ((m - 1) & 1)), (uint32_t)(((m - 1) >> 1) & 1))) {
                issue_v(m);
                v_issued = m + 1;
            }
        }
        {
            const uint32_t kg_base = OFF_KGT + (uint32_t)kb * 8192u + within;
            const uint32_t kp_base = OFF_KP + (uint32_t)buf * 16384u + (uint32_t)kb * 8192u + within;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = tq + i;
                const uint32_t roff = (uint32_t)(t * 128) + ((chunk_c ^ (uint32_t)(t & 7)) << 4);
                st_u64(sm, qg_base + roff, bmul4(qlp[i], ePp));
                st_u64(sm, kg_base + roff, bmul4(klp[i], ePp));
                st_u64(sm, kp_base + roff, bmul4(krp[i], eCPp));
            }
        }
        fence_async_smem();
        ok = wait_bar(x, bar_addr(x, MB_MMA_P), ph_mma);
        ph_mma ^= 1u;
        if (named_bar_any(BAR_PREP, kPrepThreads, !ok)) break;
        fence_after_sync();

        // ---------------- A_kk (fp32) and A_qk (bf16 operand) -------------
        {
            // All 16 warps: warp w reads TMEM lane quarter q = w % 4 (A_kk rows for
            // q < 2, A_qk rows for q >= 2) and column blocks sub, sub + 4 of that
            // quarter's range (rows 0-31 need blocks 0-2, rows 32-63 blocks 3-9).
            const int q = warp & 3, sub = warp >> 2;
            const int rr = (q & 1) * 32 + lane;           // row of A_kk / A_qk
            const int Rr = rr >> 4;
            const bool is_qk = q >= 2;
            const int nblk = (q & 1) ? 7 : 3;
            const int cb0 = (q & 1) ? 48 : 0;
            const float br = beta_s[rr];
            uint8_t *aqk = sm + OFF_AQK + buf * 8192;
            auto emit = [&](int cb, const float (&vals)[16]) {
                const int Rb = cb < 16 ? 0 : cb < 48 ? 1 : cb < 96 ? 2 : 3;   // block of the slice
                if (Rb != Rr) return;
                const int i0 = cb - kr_off(Rb);               // first column index i of the slice
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
                    // Only the strictly lower part is read by the solve.
#pragma unroll
                    for (int u4 = 0; u4 < 4; ++u4)
                        *reinterpret_cast<float4 *>(Akk + rr * LDA + i0 + 4 * u4) =
                            make_float4(br * vals[4 * u4 + 0], br * vals[4 * u4 + 1],
                                        br * vals[4 * u4 + 2], br * vals[4 * u4 + 3]);
                }
            };
            if (sub + 4 < nblk) {
                float v0[16], v1[16];
                const int cba = cb0 + 16 * sub, cbb = cb0 + 16 * (sub + 4);
                tmem_ld16x2(x.tm + lane_base + COL_INTRA + cba, x.tm + lane_base + COL_INTRA + cbb, v0, v1);
                emit(cba, v0);
                emit(cbb, v1);
            } else if (sub < nblk) {
                float v0[16];
                const int cba = cb0 + 16 * sub;
                tmem_ld16(x.tm + lane_base + COL_INTRA + cba, v0);
                emit(cba, v0);
            }
            // A_qk columns past this row's tile are zero.
            if (is_qk && sub == 3) {
                for (int i0 = 16 * (Rr + 1); i0 < C; i0 += 16) {
                    const uint4 z4 = make_uint4(0, 0, 0, 0);
                    st_u128(aqk, (uint32_t)(rr * 128 + ((((i0 >> 3) + 0) ^ (rr & 7)) << 4)), z4);
                    st_u128(aqk, (uint32_t)(rr * 128 + ((((i0 >> 3) + 1) ^ (rr & 7)) << 4)), z4);
                }
            }
        }
        // (A_qk reaches the async proxy through the fence before the READY hand-off.)
        fence_before_sync();
        named_bar(BAR_PREP, kPrepThreads);
        if (m + 1 < x.nchunks) {           // MMA (I) is done with its operand tiles
            issue_rows(m + 1, false);
        }

        beta_next = load_beta(m + 1);     // in flight during the solve (beta_s holds this chunk's)

        // ---------------- T = (I + A_kk)^-1, blocked ----------------------
        // Diagonal 16x16 blocks T_II = (I + A_II)^-1 first; the rest follows from
        // (I + A) T = I, i.e. T_IJ = -T_II sum_{J<=K<I} A_IK T_KJ, in three steps:
        //   (1) X10 = A10 T00, X32 = A32 T22, Xc = A_{23,01} T_{01,01} without its T10 term;
        //   (2) T10 = -T11 X10, T32 = -T33 X32, Xc[:, 0:16] -= Xc[:, 16:32] X10
        //       (the missing term A_{23,1} T10 equals -(A_{23,1} T11) X10);
        //   (3) T_{23,01} = -T_{23,23} Xc.
        // The products run on the tensor cores in tf32 (warp-level mma); X10, X32
        // and Xc live in the upper triangle of T, which is never read as T.  Each
        // block of T goes to the bf16 operand T Diag(beta) as it is produced; the
        // operand's upper triangle is zeroed once, before the first chunk.
        if (warp < 2) {
            // Diagonal blocks: lane = (block 2 warp + lane / 16, column j = lane % 16),
            // right-looking substitution down the column: once x_i is final, every
            // later row takes its term, so the dependent chain is one FMA per row.
            const int b = 2 * warp + (lane >> 4), j = lane & 15;
            const float *Ab = Akk + 16 * b * LDA + 16 * b;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) x[r] = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                x[i] = (i == j) ? 1.f : x[i];                // rows above j stay 0
#pragma unroll
                for (int r = i + 1; r < 16; ++r) x[r] = fmaf(-Ab[r * LDA + i], x[i], x[r]);
            }
            const int col = 16 * b + j;
            const float bj = beta_s[col];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                Tm[(16 * b + r) * LDA + col] = x[r];
                *reinterpret_cast<__nv_bfloat16 *>(sm + tb_off(16 * b + r, col)) = __float2bfloat16_rn(x[r] * bj);
            }
        }
        named_bar(BAR_PREP, kPrepThreads);
        if (warp < 12) {
            // (1) one 16x8 tile per warp: X10 = A10 T00, X32 = A32 T22,
            //     Xc[:, 16:32] = A_{23,1} T11, Xc[:, 0:16] = A_{23,0} T00.
            const int blk = warp >> 1, nh = (warp & 1) * 8;
            const int arow = blk == 0 ? 16 : blk == 1 ? 48 : (blk == 2 || blk == 4) ? 32 : 48;
            const int kc = blk == 1 ? 32 : (blk == 2 || blk == 3) ? 16 : 0;
            const int drow = blk == 1 ? 32 : (blk == 3 || blk == 5) ? 16 : 0;
            const int dcol = blk == 0 ? 16 : blk == 4 || blk == 5 ? 32 : 48;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            warp_mm16x8<2>(d, Akk + arow * LDA + kc, Tm + kc * LDA + kc + nh, lane);
            warp_st16x8(Tm + drow * LDA + dcol + nh, d, 1.f, false, lane);
        }
        named_bar(BAR_PREP, kPrepThreads);
        if (warp < 8) {
            // (2) T10 = -T11 X10, T32 = -T33 X32, Xc[:, 0:16] -= Xc[:, 16:32] X10.
            const int task = warp >> 1, nh = (warp & 1) * 8;
            const int arow = task == 0 ? 16 : task == 1 ? 48 : 16 * (task - 2);
            const int acol = task == 0 ? 16 : 48;
            const int brow = task == 1 ? 32 : 0;
            const int bcol = task == 1 ? 48 : 16;
            const int drow = task == 0 ? 16 : task == 1 ? 48 : 16 * (task - 2);
            const int dcol = task == 0 ? 0 : 32;
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            warp_mm16x8<2>(d, Tm + arow * LDA + acol, Tm + brow * LDA + bcol + nh, lane);
            if (task != 0) warp_st16x8(Tm + drow * LDA + dcol + nh, d, -1.f, task >= 2, lane);
            if (task < 2) warp_tb16x8(sm, drow, dcol + nh, d, beta_s, lane);   // T10, T32
        }
        named_bar(BAR_PREP, kPrepThreads);
        if (warp < 8) {
            // (3) T_{23,01} = -T_{23,23} Xc, 16x8 tiles; rows 32-47 of T_{23,23}
            //     reach only K = 16 (their upper-right block holds X32).
            const int mt = warp >> 2, n0 = 8 * (warp & 3);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            const float *A = Tm + (32 + 16 * mt) * LDA + 32;
            const float *B = Tm + 32 + n0;
            if (mt == 0) warp_mm16x8<2>(d, A, B, lane);
            else warp_mm16x8<4>(d, A, B, lane);
            warp_tb16x8(sm, 32 + 16 * mt, n0, d, beta_s, lane);
        }
        fence_async_smem();
        named_bar(BAR_PREP, kPrepThreads);
        if (m + 1 < x.nchunks) {           // the solve workspace is free
            issue_rows(m + 1, true);
            issued = m + 2;
        }

        // Everything of chunk m is in shared memory: the state warps take the
        // chunk, starting with MMAs (II)/(III).
        if (tid == 0 && !p.withhold_ready) mbar_arrive(bar_addr(x, MB_READY + buf));
    }
    if (below_gmin) *reinterpret_cast<volatile int *>(sm + OFF_MISC + MISC_RANGE) = 1;
    // After an abort, tensor copies may still be writing into shared memory: let
    // the last requested phase of each load barrier complete (bounded) before
    // the CTA can exit.  (Waiting on a phase that already completed returns at
    // once.)
    if (tid == kPrepThreads - 32 && mi_issued > 0) {
        for (uint32_t i = 0; i < kWaitTries; ++i)
            if (mbar_try_wait_suspend(bar_addr(x, MB_MMA_P), (uint32_t)((mi_issued - 1) & 1), kSuspendNs)) break;
    }
    if (tid == kPrepThreads - 32 && issued > 0) {
        const int bars[3] = {MB_LQK, MB_LZV, MB_LV};
        const int last[3] = {issued, issued, v_issued};
        for (int b = 0; b < (x.trans ? 2 : 3); ++b) {
            const uint32_t par = (uint32_t)((last[b] - 1) & 1);
            for (uint32_t i = 0; i < kWaitTries; ++i)
                if (mbar_try_wait_suspend(bar_addr(x, bars[b]), par, kSuspendNs)) break;
        }
    }
}

// =====================================================================
// State role: warps 16-19, thread j <-> TMEM lane j <-> value channel j.
// =====================================================================
__device__ __forceinline__ void state_role(const ChunkParams &p, const CUtensorMap *tmaps, bool o_tma, const Ctx &x,
                                           int tid) {
    uint8_t *sm = x.sm;
    const int ts = tid - kPrepThreads;      // 0..127
    const int warp = tid >> 5;
    const int j = ts;                        // (warp - 8) * 32 + lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float *gam_s = reinterpret_cast<const float *>(sm + OFF_MISC + MISC_GAM);

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

    // Descriptors: start-address fields advance by compile-time offsets per k-step.
    const uint64_t dW0 = mnmaj_desc(x.sbase + OFF_W, 0);
    const uint32_t id_iv = idesc_bf16(128, 64, false, /*b_mn_major=*/true);
    const uint32_t id_vi = idesc_bf16(128, 128, false, /*b_mn_major=*/true);
    const uint32_t id_v = idesc_bf16(128, 64);
    const uint32_t id_w = idesc_bf16(128, 64, false, false, /*a_mn_major=*/true);
    uint32_t ph_s = 0, ph_o = 0;
    for (int n = 0; n < x.nchunks; ++n) {
        const int buf = n & 1;
        const uint32_t col_ut = COL_UT + 64u * (uint32_t)buf;
        bool ok = wait_bar(x, bar_addr(x, MB_READY + buf), (uint32_t)((n >> 1) & 1));
        // (II) Ut^T = V^T TB^T and (III) W^T = (K Gamma)^T TB^T of this chunk,
        // once its V tile has landed.
        if (ts == 0 && ok) {
            if (!x.trans) ok = wait_bar(x, bar_addr(x, MB_LV), (uint32_t)(n & 1));
            if (ok) {
                fence_after_sync();
                if (!x.trans) {
#pragma unroll
                    for (int s = 0; s < C / 16; ++s)
                        mma_bf16(x.tm + col_ut, mnmaj_desc(x.sbase + OFF_VT, s), kmaj_desc(x.sbase + OFF_TB, 64, s),
                                 id_w, s > 0);
                }
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    mma_bf16(x.tm + COL_WT, mnmaj_desc(x.sbase + OFF_KGT, s), kmaj_desc(x.sbase + OFF_TB, 64, s),
                             id_w, s > 0);
                mma_commit(bar_addr(x, MB_MMA_W + buf));
            }
        }
        if (ok) ok = wait_bar(x, bar_addr(x, MB_MMA_W + buf), (uint32_t)((n >> 1) & 1));
        // The previous chunk's o rows in the -W tile have been read by their tensor store.
        if (ts == 0) bulk_wait_read<0>();
        if (named_bar_any(BAR_STATE, kStateThreads, !ok)) break;
        fence_after_sync();

        // -W^T (row j = TMEM lane j) -> MN-major bf16 operand; then the W^T
        // columns are free for the prep warps' next MMA (I).
        {
            float v0[16], v1[16];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                tmem_ld16x2(x.tm + lane_base + COL_WT + hf * 32, x.tm + lane_base + COL_WT + hf * 32 + 16, v0, v1);
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    v0[u] = -v0[u];
                    v1[u] = -v1[u];
                }
                st_u128(sm, OFF_W + mnmaj_chunk_off(j, 4 * hf + 0), pack8(v0));
                st_u128(sm, OFF_W + mnmaj_chunk_off(j, 4 * hf + 1), pack8(v0 + 8));
                st_u128(sm, OFF_W + mnmaj_chunk_off(j, 4 * hf + 2), pack8(v1));
                st_u128(sm, OFF_W + mnmaj_chunk_off(j, 4 * hf + 3), pack8(v1 + 8));
            }
        }
        fence_async_smem();
        fence_before_sync();
        named_bar(BAR_STATE, kStateThreads);

        // (IV) U^T = Ut^T + S^T (-W)
        if (ts == 0) {
            fence_after_sync();
            mbar_arrive(bar_addr(x, MB_WTFREE));
#pragma unroll
            for (int s = 0; s < D / 16; ++s)
                mma_bf16_tmem_a(x.tm + col_ut, x.tm + COL_SBF + s * 8, dW0 + (uint64_t)(s * 2048 / 16),
                                id_iv, (x.trans && s == 0) ? 0u : 1u);
            mma_commit(bar_addr(x, MB_MMA_S));
        }
        // Meanwhile: S^T <- S^T Diag(gamma_C) (fp32, in TMEM); the state entering
        // this chunk goes to S_chunks first when it is asked for.
        float *sck = (p.S_chunks && !x.trans) ? p.S_chunks + ((size_t)x.chain * x.nchunks + n) * D * D + j
                                              : nullptr;
        for (int mm = 0; mm < D / 16; ++mm) {
            // gamma_C of these 16 columns (a broadcast read) is in flight with the TMEM load
            const float4 *g4p = reinterpret_cast<const float4 *>(gam_s + buf * D + mm * 16);
            const float4 g4[4] = {g4p[0], g4p[1], g4p[2], g4p[3]};
            float vals[16];
            tmem_ld16(x.tm + lane_base + COL_ST + mm * 16, vals);
            if (sck) {
#pragma unroll
                for (int u = 0; u < 16; ++u) sck[(size_t)(mm * 16 + u) * D] = vals[u];
            }
#pragma unroll
            for (int u4 = 0; u4 < 4; ++u4) {
                vals[4 * u4 + 0] *= g4[u4].x;
                vals[4 * u4 + 1] *= g4[u4].y;
                vals[4 * u4 + 2] *= g4[u4].z;
                vals[4 * u4 + 3] *= g4[u4].w;
            }
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

        // (VI) S^T += U^T K' (the serial carry), then (V) O^T = S^T (Q Gamma)^T + U^T A_qk^T
        // with its own completion barrier so the next S^T operand is built meanwhile.
        if (ts == 0) {
            fence_after_sync();
            const uint64_t dKP = mnmaj_desc(x.sbase + OFF_KP + 16384u * buf, 0);
#pragma unroll
            for (int s = 0; s < C / 16; ++s)
                mma_bf16_tmem_a(x.tm + COL_ST, x.tm + COL_UBF + s * 8, dKP + (uint64_t)(s * 2048 / 16), id_vi, 1u);
            mma_commit(bar_addr(x, MB_MMA_S));
            if (x.want_o) {
                const uint64_t dQG = kmaj_desc(x.sbase + OFF_QG + 16384u * buf, 64, 0);
                const uint64_t dAQ = kmaj_desc(x.sbase + OFF_AQK + 8192u * buf, 64, 0);
#pragma unroll
                for (int s = 0; s < D / 16; ++s)
                    mma_bf16_tmem_a(x.tm + col_ut, x.tm + COL_SBF + s * 8,
                                    dQG + (uint64_t)(((s >> 2) * 64 * 128 + (s & 3) * 32) / 16), id_v, s > 0);
#pragma unroll
                for (int s = 0; s < C / 16; ++s)
                    mma_bf16_tmem_a(x.tm + col_ut, x.tm + COL_UBF + s * 8, dAQ + (uint64_t)(s * 32 / 16), id_v, 1u);
            }
            mma_commit(bar_addr(x, MB_ODONE));
        }
        ok = wait_bar(x, bar_addr(x, MB_MMA_S), ph_s);
        ph_s ^= 1u;
        if (named_bar_any(BAR_STATE, kStateThreads, !ok)) break;
        fence_after_sync();
        // The new S^T as the bf16 operand of the next chunk.  (V) still reads
        // the old operand: wait for it before overwriting.
        ok = wait_bar(x, bar_addr(x, MB_ODONE), ph_o);
        ph_o ^= 1u;
        if (named_bar_any(BAR_STATE, kStateThreads, !ok)) break;
        fence_after_sync();
        for (int mm = 0; mm < D / 16; ++mm) {
            float vals[16];
            tmem_ld16(x.tm + lane_base + COL_ST + mm * 16, vals);
            uint32_t pk[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) pk[u] = pack_bf16x2(vals[2 * u], vals[2 * u + 1]);
            tmem_st8(x.tm + lane_base + COL_SBF + mm * 8, pk);
        }
        // o rows of this chunk (the output scale is in q's norm factor): thread j
        // holds value channel j of each token.  A whole chunk goes through the -W
        // tile (free since (IV) completed) as [64 tokens][128 channels] bf16 rows
        // and leaves in one tensor store; a partial last chunk is stored directly.
        const int t0 = n * C, Cc = min(C, x.T - t0);
        const bool o_staged = x.want_o && o_tma && Cc == C;
        if (o_staged) {
#pragma unroll 1
            for (int mm = 0; mm < C / 16; ++mm) {
                float vals[16];
                tmem_ld16(x.tm + lane_base + col_ut + mm * 16, vals);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t w = pack_bf16x2(vals[2 * u], vals[2 * u + 1]);
                    uint8_t *row = sm + OFF_W + (uint32_t)(mm * 16 + 2 * u) * 256u + 2u * (uint32_t)j;
                    *reinterpret_cast<uint16_t *>(row) = (uint16_t)(w & 0xFFFFu);
                    *reinterpret_cast<uint16_t *>(row + 256) = (uint16_t)(w >> 16);
                }
            }
            fence_async_smem();
        } else if (x.want_o) {
            __nv_bfloat16 *orow = static_cast<__nv_bfloat16 *>(p.o) +
                                  (((size_t)x.b * x.T + t0) * p.HV + x.hv) * D + j;
            const size_t tstride = (size_t)p.HV * D;
            for (int mm = 0; mm < C / 16; ++mm) {
                float vals[16];
                tmem_ld16(x.tm + lane_base + col_ut + mm * 16, vals);
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    if (mm * 16 + u < Cc) orow[(mm * 16 + u) * tstride] = __float2bfloat16_rn(vals[u]);
            }
        }
        tmem_st_wait();
        fence_before_sync();
        named_bar(BAR_STATE, kStateThreads);
        if (ts == 0) {
            if (o_staged) {
                tma_store_3d(&tmaps[4], 0, x.hv, x.b * x.T + t0, x.sbase + OFF_W);
                bulk_commit();
            }
            mbar_arrive(bar_addr(x, MB_FREE + buf));
        }
    }

    // Every MMA this role issued ((II)-(VI)) must be complete before the TMEM
    // can be freed, after an abort too: one more commit arrives once all of
    // them are (at once if none is in flight); wait for it (bounded).
    if (ts == 0) {
        bulk_wait<0>();                    // o tensor stores complete (shared rows read, global written)
        mma_commit(bar_addr(x, MB_DRAIN));
        for (uint32_t i = 0; i < kWaitTries; ++i)
            if (mbar_try_wait_suspend(bar_addr(x, MB_DRAIN), 0u, kSuspendNs)) break;
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
chunk_tc_kernel(const __grid_constant__ TcParams tp) {
    const ChunkParams &p = tp.p;
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
    x.want_o = !x.trans && p.o != nullptr;
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
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar_addr(x, i), 1);
        *x.abort_flag = 0;
        *reinterpret_cast<volatile int *>(sm + OFF_MISC + MISC_RANGE) = 0;
        fence_mbar_init();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    x.tm = *tmem_slot;

    if (warp < kPrepThreads / 32) prep_role(p, tp.tm, x, tid);
    else state_role(p, tp.tm, tp.o_tma != 0, x, tid);

    fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        unsigned int word = 0;
        if (*x.abort_flag) word |= 1u;                                                   // a wait gave up
        if (*reinterpret_cast<volatile int *>(sm + OFF_MISC + MISC_RANGE)) word |= 2u;  // g clamped
        if (word) atomicOr(&g_device_error, word);
    }
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(x.tm, TMEM_COLS);
    }
}

}  // namespace

bool chunk_tc_supported(const ChunkParams &p, bool bf16) {
    return bf16 && p.Dk == D && p.Dv == D && p.C == C;
}

// Tensor map of a [B*T][heads][128] bf16 tensor with a [64][1][128] box, or
// with a [64][1][64] box in the 128-byte swizzle (the MMA operand layout).
static cudaError_t make_row_map(CUtensorMap *map, const void *base, int heads, long long rows,
                                bool swizzle128 = false) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
    const cuuint32_t box[3] = {(cuuint32_t)(swizzle128 ? 64 : D), 1, (cuuint32_t)C};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_chunk_tc(const ChunkParams &p, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    TcParams tp;
    tp.p = p;
    const long long rows = (long long)p.B * p.T;
    if ((e = make_row_map(&tp.tm[0], p.q, p.H, rows)) != cudaSuccess) return e;
    if ((e = make_row_map(&tp.tm[1], p.k, p.H, rows)) != cudaSuccess) return e;
    if (p.g_per_head) memset(&tp.tm[2], 0, sizeof(tp.tm[2]));      // z is read directly
    else if ((e = make_row_map(&tp.tm[2], p.g, p.HV, rows)) != cudaSuccess) return e;
    if ((e = make_row_map(&tp.tm[3], p.v, p.HV, rows, /*swizzle128=*/true)) != cudaSuccess) return e;
    // o by tensor stores when its map can be made (16-byte aligned base), else by plain stores
    tp.o_tma = (p.o && make_row_map(&tp.tm[4], p.o, p.HV, rows) == cudaSuccess) ? 1 : 0;
    if (!tp.o_tma) memset(&tp.tm[4], 0, sizeof(tp.tm[4]));
    dim3 grid(p.B * p.HV, p.M_T ? 2 : 1);
    chunk_tc_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(tp);
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
