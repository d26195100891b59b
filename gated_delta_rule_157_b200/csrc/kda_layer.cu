// Layer prologue and epilogue around the KDA core (page "KDA 模块交互式演示",
// sections 1.1 ShortConv and 1.7 the complete layer; page "Implémenter KDA",
// "La paramétrisation" and "La porte de sortie de rang plein"):
//
//   short_conv_kernel   u = bias + causal depthwise K-tap convolution of x,
//                       y = SiLU(u) (optional), L2-normalised per 128-channel
//                       head (optional); carries a K-1 token window across
//                       calls (decode, or a sequence run in pieces).
//   output_gate_kernel  y = sigmoid(gate) * weight * o / sqrt(mean(o^2) + eps)
//                       per (token, head) of 128 channels.
//
// Both are HBM-bound streams: contiguous 8- or 16-byte loads and stores per
// lane (256 or 512 contiguous bytes per warp and token), per-head reductions
// by warp shuffles, and nothing read twice.  For rows of a multiple of 256
// channels the short convolution streams [128 tokens x 256 channels] tiles
// through shared memory by tensor-map copies (short_conv_tma_kernel).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <string.h>

#include "kda_internal.cuh"
#include "tc_ptx.cuh"

namespace kda {
namespace {

constexpr int kConvTokens = 64;     // tokens per warp (sliding window in registers)
constexpr int kLayerThreads = 256;

__device__ __forceinline__ void unpack4(uint2 w, float (&f)[4]) {
    f[0] = __uint_as_float(w.x << 16);
    f[1] = __uint_as_float(w.x & 0xFFFF0000u);
    f[2] = __uint_as_float(w.y << 16);
    f[3] = __uint_as_float(w.y & 0xFFFF0000u);
}
__device__ __forceinline__ uint2 pack4(const float (&f)[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(f[2], f[3]);
    return make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float silu(float u) { return __fdividef(u, 1.f + __expf(-u)); }

// Warp w of the grid: batch b, 256-channel group grp (lane = 8 channels, one
// 16-byte load per token row; a 128-channel head is a half-warp), tokens
// [t0, t0 + kConvTokens) (only the K-1 halo tokens before t0 are read twice).
// A group of 128 channels at the end of a row leaves the upper half-warp idle.
__host__ __device__ inline long long conv_grid_warps(const ConvParams &p) {
    const long long nblk = p.T > 0 ? (p.T + kConvTokens - 1) / kConvTokens : 1;
    return (long long)p.B * ((p.C + 255) / 256) * nblk;
}

__device__ __forceinline__ void unpack8(uint4 w, float (&f)[8]) {
    const uint32_t r[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(r[i] << 16);
        f[2 * i + 1] = __uint_as_float(r[i] & 0xFFFF0000u);
    }
}
// The same eight channels as four (even, odd) channel pairs.
__device__ __forceinline__ void unpack8x2(uint4 w, float2 (&f)[4]) {
    const uint32_t r[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = make_float2(__uint_as_float(r[i] << 16), __uint_as_float(r[i] & 0xFFFF0000u));
}
__device__ __forceinline__ uint4 pack8x2(const float2 (&f)[4]) {
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 a = __floats2bfloat162_rn(f[i].x, f[i].y);
        r[i] = *reinterpret_cast<uint32_t *>(&a);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    uint32_t r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 a = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        r[i] = *reinterpret_cast<uint32_t *>(&a);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

template <int K>
__global__ void __launch_bounds__(kLayerThreads, 2)
short_conv_kernel(ConvParams p) {
    const int lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * (kLayerThreads / 32) + (threadIdx.x >> 5);
    const int ngrp = (p.C + 255) / 256;
    const int nblk = p.T > 0 ? (p.T + kConvTokens - 1) / kConvTokens : 1;
    if (gw >= conv_grid_warps(p)) return;
    // Consecutive warps take consecutive channel groups of the same tokens, so
    // a thread block streams whole contiguous spans of each token row.
    const int grp = (int)(gw % ngrp);
    const int blk = (int)((gw / ngrp) % nblk);
    const int b = (int)(gw / ((long long)nblk * ngrp));
    const int c0 = grp * 256 + 8 * lane;
    const bool act = c0 < p.C;                   // the upper half-warp of a 128-channel tail group idles
    const int t0 = blk * kConvTokens, t1 = min(p.T, t0 + kConvTokens);
    const __nv_bfloat16 *x = static_cast<const __nv_bfloat16 *>(p.x);
    const __nv_bfloat16 *sin = static_cast<const __nv_bfloat16 *>(p.state_in);
    __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(p.y);

    float w[8][4], bias[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        bias[u] = (act && p.bias) ? p.bias[c0 + u] : 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) w[u][j] = (act && j < K) ? p.w[(size_t)(c0 + u) * K + j] : 0.f;
    }
    auto row = [&](int tok) { return *reinterpret_cast<const uint4 *>(x + ((size_t)b * p.T + tok) * p.C + c0); };
    // win[s]: token t - 3 + s, s = 0..2 (only the last K-1 slots are used).
    auto fetch = [&](int tok, float (&f)[8]) {
        uint4 r = make_uint4(0, 0, 0, 0);
        if (act && tok >= 0) r = row(tok);
        else if (act && sin && tok >= -(K - 1))
            r = *reinterpret_cast<const uint4 *>(sin + ((size_t)b * (K - 1) + (K - 1) + tok) * p.C + c0);
        unpack8(r, f);
    };
    float win[3][8];
#pragma unroll
    for (int s = 0; s < 3; ++s) fetch(t0 - 3 + s, win[s]);

    // Groups of 2 tokens, double-buffered: the 2 row loads of the next group
    // are in flight while the current group is computed.  Rows past the block
    // are computed from zeros and not stored.  state_out (the last K-1 tokens of
    // state_in ++ x, oldest first) is written at the sequence's last token.
    constexpr int G = 2;
    __nv_bfloat16 *so = static_cast<__nv_bfloat16 *>(p.state_out);
    auto put_state = [&](const float (&s0)[8], const float (&s1)[8], const float (&s2)[8]) {
        const float *rows[3] = {s0, s1, s2};
#pragma unroll
        for (int r = 0; r < K - 1; ++r) {
            const float *src = rows[4 - K + r];
            float f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = src[u];
            if (act) *reinterpret_cast<uint4 *>(so + ((size_t)b * (K - 1) + r) * p.C + c0) = pack8(f);
        }
    };
    auto load_group = [&](int tg, uint4 (&r)[G]) {
#pragma unroll
        for (int i = 0; i < G; ++i) r[i] = (act && tg + i < t1) ? row(tg + i) : make_uint4(0, 0, 0, 0);
    };
    auto process = [&](int tg, const uint4 (&r)[G]) {
#pragma unroll
        for (int i = 0; i < G; ++i) {
            float cur[8];
            unpack8(r[i], cur);
            float out[8];
            float ss = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                // taps j = 0..K-2 read win[4 - K + j]; tap K-1 reads the current token
                float acc = bias[u];
#pragma unroll
                for (int j = 0; j < 3; ++j)
                    if (j < K - 1) acc = fmaf(w[u][j], win[4 - K + j][u], acc);
                acc = fmaf(w[u][K - 1], cur[u], acc);
                out[u] = p.silu ? silu(acc) : acc;
                ss = fmaf(out[u], out[u], ss);
            }
            if (p.head_dim) {
                // the head's 128 channels are this half-warp's 16 lanes
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                const float rn = rsqrtf(ss + p.l2_eps);
#pragma unroll
                for (int u = 0; u < 8; ++u) out[u] *= rn;
            }
            if (act && tg + i < t1) *reinterpret_cast<uint4 *>(y + ((size_t)b * p.T + tg + i) * p.C + c0) = pack8(out);
            if (so && tg + i + 1 == p.T) put_state(win[1], win[2], cur);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                win[0][u] = win[1][u];
                win[1][u] = win[2][u];
                win[2][u] = cur[u];
            }
        }
    };
    uint4 ra[G], rb[G];
    if (t0 < t1) load_group(t0, ra);
    for (int tg = t0; tg < t1; tg += 2 * G) {
        if (tg + G < t1) load_group(tg + G, rb);
        process(tg, ra);
        if (tg + G < t1) {
            if (tg + 2 * G < t1) load_group(tg + 2 * G, ra);
            process(tg + G, rb);
        }
    }
    if (so && p.T == 0) put_state(win[0], win[1], win[2]);   // no token: state_in passes through
}

// Warp per 4 consecutive (row n, head h) pairs, lane = 4 channels of the
// head's 128; the 8 loads of the four pairs are in flight together.
constexpr int kGateRows = 4;
__global__ void __launch_bounds__(kLayerThreads)
output_gate_kernel(GateParams p) {
    const int lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * (kLayerThreads / 32) + (threadIdx.x >> 5);
    const long long rows = (long long)p.N * p.HV;
    const long long r0 = gw * kGateRows;
    if (r0 >= rows) return;
    float wv[4] = {1.f, 1.f, 1.f, 1.f};
    if (p.weight) {
#pragma unroll
        for (int u = 0; u < 4; ++u) wv[u] = p.weight[4 * lane + u];
    }
    const __nv_bfloat16 *po = static_cast<const __nv_bfloat16 *>(p.o);
    const __nv_bfloat16 *pg = static_cast<const __nv_bfloat16 *>(p.gate);
    uint2 ro[kGateRows], rg[kGateRows];
#pragma unroll
    for (int i = 0; i < kGateRows; ++i) {
        const bool in = r0 + i < rows;
        const size_t off = (size_t)(r0 + i) * p.D + 4 * lane;
        ro[i] = in ? *reinterpret_cast<const uint2 *>(po + off) : make_uint2(0, 0);
        rg[i] = in ? *reinterpret_cast<const uint2 *>(pg + off) : make_uint2(0, 0);
    }
#pragma unroll
    for (int i = 0; i < kGateRows; ++i) {
        float o[4], g[4];
        unpack4(ro[i], o);
        unpack4(rg[i], g);
        const float ms = warp_sum(o[0] * o[0] + o[1] * o[1] + o[2] * o[2] + o[3] * o[3]) * (1.f / 128.f);
        const float r = rsqrtf(ms + p.eps);
        float out[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) out[u] = __fdividef(o[u] * r * wv[u], 1.f + __expf(-g[u]));
        if (r0 + i < rows)
            *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.y) + (size_t)(r0 + i) * p.D + 4 * lane) = pack4(out);
    }
}


// ---------------------------------------------------------------------------
// short_conv_tma_kernel: the same convolution for C a multiple of 256, as a
// stream of tiles (batch row b, 256 channels, 128 tokens) through shared
// memory.  Persistent CTAs of 512 threads, one per SM; each takes a contiguous
// range of tiles in the order channel group, batch row, token block (the
// weights are reloaded only when the group changes).
// Each tile arrives as one [131 rows x 256 channels] box of a 3-D tensor map
// (tokens t0-3 .. t0+127; rows before the sequence or past its end read as
// zeros) in a three-stage ring, two tiles (134 KB) ahead of the one computed,
// enough bytes in flight per SM to cover the memory latency at full
// bandwidth; output rows go straight from registers to global memory, 512
// contiguous bytes per warp and token.  Warp w computes tokens t0 + 8w .. +7 with
// its 3-token window in registers (16 warps per SM keep enough independent
// work in flight for the per-token latency chain: taps, tanh, head-norm
// shuffles, rsqrt), lane = 8 channels (16-byte shared loads,
// a 128-channel head is a half-warp).  SiLU(u) = u sigmoid(u) with
// sigmoid(u) = (1 + tanh(u/2)) / 2 on one special-function instruction.
constexpr int kConvThreads = 512;                        // 16 warps
constexpr int kTokPerWarp = 8;                           // kTT / 16
constexpr int kTT = 128;                                 // tokens per tile
static_assert(kTT == kTokPerWarp * (kConvThreads / 32), "the warps cover a tile");
constexpr int kTC = 256;                                 // channels per tile
constexpr int kHalo = 3;                                 // K - 1 <= 3 earlier tokens
constexpr uint32_t kRowBytes = kTC * 2;                  // 512
constexpr uint32_t kInBytes = (kTT + kHalo) * kRowBytes; // 67,072
constexpr int kStages = 3;
constexpr uint32_t TS_IN = 0;                            // kStages input tiles (128-byte aligned)
constexpr uint32_t TS_BAR = kStages * kInBytes;          // kStages mbarriers
constexpr uint32_t TS_SMEM = TS_BAR + 64;
constexpr long long kConvWaitCycles = 4000000000LL;      // about two seconds of SM clock

__device__ unsigned int g_conv_error = 0;                // bit 0: a stage wait gave up

struct ConvTmaParams {
    ConvParams p;
    CUtensorMap tx;          // x as [B][T][C]: boxes of [1][131][256]
};

// SiLU(2h) = h + h tanh(h): the tiled kernel keeps its taps and bias halved,
// so its convolution yields h = u / 2 directly.
__device__ __forceinline__ float silu_of_half(float h) {
    float th;
#ifdef __CUDA_ARCH__
    asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(h));
#else
    th = tanhf(h);
#endif
    return fmaf(h, th, h);
}
// Both channels of a pair: tanh per channel, the product-add packed.
__device__ __forceinline__ float2 silu_of_half2(float2 h) {
    float2 th;
#ifdef __CUDA_ARCH__
    asm("tanh.approx.f32 %0, %1;" : "=f"(th.x) : "f"(h.x));
    asm("tanh.approx.f32 %0, %1;" : "=f"(th.y) : "f"(h.y));
#else
    th = make_float2(tanhf(h.x), tanhf(h.y));
#endif
    return __ffma2_rn(h, th, h);
}

template <int K>
__global__ void __launch_bounds__(kConvThreads, 1)
short_conv_tma_kernel(const __grid_constant__ ConvTmaParams tp) {
    const ConvParams &p = tp.p;
    extern __shared__ __align__(1024) float smem[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(smem);
    const uint32_t sbase = tc::smem_addr(sm);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nblk = (p.T + kTT - 1) / kTT;
    const int ntiles = p.B * (p.C / kTC) * nblk;      // below 2^31 (checked by the launcher)
    // This CTA's tiles are the contiguous range [n0, n1) of the order channel
    // group (slowest), batch row, token block (fastest): moving to the next
    // tile is an increment, and the weights change only at a group boundary.
    const int n0 = (int)((long long)ntiles * blockIdx.x / gridDim.x);
    const int my = (int)((long long)ntiles * (blockIdx.x + 1) / gridDim.x) - n0;
    struct Cursor {
        int g, b, blk;
    };
    auto first = [&]() {
        Cursor c;
        const int rows = p.B * nblk;
        c.g = n0 / rows;
        c.b = (n0 % rows) / nblk;
        c.blk = n0 % nblk;
        return c;
    };
    auto advance = [&](Cursor &c) {
        if (++c.blk == nblk) {
            c.blk = 0;
            if (++c.b == p.B) {
                c.b = 0;
                ++c.g;
            }
        }
    };
    auto bar = [&](int st) { return sbase + TS_BAR + 8u * (uint32_t)st; };
    Cursor ic = first();                              // the next tile to request (thread 0)
    int ii = 0;
    auto issue = [&]() {
        const int st = ii % kStages;
        tc::mbar_arrive_expect_tx(bar(st), kInBytes);
        tc::tma_load_3d(sbase + TS_IN + (uint32_t)st * kInBytes, &tp.tx, ic.g * kTC, ic.blk * kTT - kHalo, ic.b,
                        bar(st));
        advance(ic);
        ++ii;
    };
    if (tid == 0) {
        for (int st = 0; st < kStages; ++st) tc::mbar_init(bar(st), 1);
        tc::fence_mbar_init();
        tc::prefetch_tensormap(&tp.tx);
    }
    __syncthreads();
    if (tid == 0)
        while (ii < my && ii < kStages - 1) issue();
    const __nv_bfloat16 *sin = static_cast<const __nv_bfloat16 *>(p.state_in);
    __nv_bfloat16 *so = static_cast<__nv_bfloat16 *>(p.state_out);
    float2 w[4][4], bias[4];                          // channel pairs (8 lane, 8 lane + 1), ...
    int wg = -1;                                      // channel group whose weights are loaded
    int i = 0;
    bool aborted = false;
    Cursor cc = first();                              // the tile computed
    for (; i < my; ++i, advance(cc)) {
        const int b = cc.b, g = cc.g, blk = cc.blk;
        const int st = i % kStages;
        // its stage was read by tile i - 1, finished before the barrier that ended it
        if (tid == 0 && ii < my) issue();
        bool ok = tc::mbar_try_wait(bar(st), (uint32_t)((i / kStages) & 1));
        if (!ok) {
            const long long c0 = clock64();
            while (!(ok = tc::mbar_try_wait(bar(st), (uint32_t)((i / kStages) & 1))))
                if (clock64() - c0 > kConvWaitCycles) break;
        }
        if (__syncthreads_or(!ok)) {
            aborted = true;
            break;
        }
        if (g != wg) {
            wg = g;
            const int c = g * kTC + 8 * lane;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                // halved (exact in binary floating point): the convolution gives u / 2
                bias[u] = p.bias ? make_float2(0.5f * p.bias[c + 2 * u], 0.5f * p.bias[c + 2 * u + 1])
                                 : make_float2(0.f, 0.f);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    w[u][j] = j < K ? make_float2(0.5f * p.w[(size_t)(c + 2 * u) * K + j],
                                                  0.5f * p.w[(size_t)(c + 2 * u + 1) * K + j])
                                    : make_float2(0.f, 0.f);
            }
        }
        const int t0 = blk * kTT, t1 = min(p.T, t0 + kTT);
        uint8_t *in = sm + TS_IN + (uint32_t)st * kInBytes;            // row r: token t0 - 3 + r
        const int tw = kTokPerWarp * warp;
        __nv_bfloat16 *yr = static_cast<__nv_bfloat16 *>(p.y) + ((size_t)b * p.T + t0 + tw) * p.C + g * kTC + 8 * lane;
        if (t0 == 0 && sin) {
            // the window before the sequence: the carried K-1 tokens (oldest first)
            for (int idx = tid; idx < (K - 1) * (kTC / 8); idx += kConvThreads) {
                const int r = idx / (kTC / 8), l8 = idx % (kTC / 8);
                *reinterpret_cast<uint4 *>(in + (uint32_t)(kHalo - (K - 1) + r) * kRowBytes + 16u * l8) =
                    *reinterpret_cast<const uint4 *>(sin + ((size_t)b * (K - 1) + r) * p.C + g * kTC + 8 * l8);
            }
            __syncthreads();
        }
        // channel pairs in packed FP32x2 arithmetic (one instruction per pair)
        float2 win[3][4];
#pragma unroll
        for (int s = 0; s < 3; ++s)
            unpack8x2(*reinterpret_cast<const uint4 *>(in + (uint32_t)(tw + s) * kRowBytes + 16u * lane), win[s]);
#pragma unroll
        for (int k = 0; k < kTokPerWarp; ++k) {
            float2 cur[4];
            unpack8x2(*reinterpret_cast<const uint4 *>(in + (uint32_t)(tw + kHalo + k) * kRowBytes + 16u * lane), cur);
            float2 o[4];
            float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                // taps j = 0..K-2 read win[4 - K + j]; tap K-1 reads the current token
                float2 acc = bias[u];
#pragma unroll
                for (int j = 0; j < 3; ++j)
                    if (j < K - 1) acc = __ffma2_rn(w[u][j], win[4 - K + j][u], acc);
                acc = __ffma2_rn(w[u][K - 1], cur[u], acc);
                o[u] = p.silu ? silu_of_half2(acc) : __fadd2_rn(acc, acc);
                ss2 = __ffma2_rn(o[u], o[u], ss2);
            }
            if (p.head_dim) {
                float ss = ss2.x + ss2.y;
#pragma unroll
                for (int m = 8; m > 0; m >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
                const float rn = rsqrtf(ss + p.l2_eps);
#pragma unroll
                for (int u = 0; u < 4; ++u) o[u] = __fmul2_rn(o[u], make_float2(rn, rn));
            }
            if (t0 + tw + k < t1) *reinterpret_cast<uint4 *>(yr + (size_t)k * p.C) = pack8x2(o);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                win[0][u] = win[1][u];
                win[1][u] = win[2][u];
                win[2][u] = cur[u];
            }
        }
        // state_out: the last K-1 tokens of state_in ++ x, still in the input tile
        if (so && t1 == p.T && warp == 0) {
            for (int r = 0; r < K - 1; ++r) {
                const int row = p.T - t0 + kHalo - (K - 1) + r;
                *reinterpret_cast<uint4 *>(so + ((size_t)b * (K - 1) + r) * p.C + g * kTC + 8 * lane) =
                    *reinterpret_cast<const uint4 *>(in + (uint32_t)row * kRowBytes + 16u * lane);
            }
        }
        __syncthreads();                              // stage st is free for tile i + kStages
    }
    if (tid == 0 && aborted) {
        atomicOr(&g_conv_error, 1u);
        // tiles i .. i + kStages - 2 may still be arriving: let them land (bounded)
        for (int j = i; j < ii; ++j)
            for (int tries = 0; tries < 4000; ++tries)
                if (tc::mbar_try_wait_suspend(bar((int)(j % kStages)), (uint32_t)((j / kStages) & 1), 500000u))
                    break;
    }
}

}  // namespace

// The tiled kernel, when the shape and buffers allow it (defined below).
cudaError_t launch_short_conv_tma(const ConvParams &p, cudaStream_t s, bool &launched);

cudaError_t launch_short_conv(const ConvParams &p, cudaStream_t s) {
    bool launched = false;
    const cudaError_t e0 = launch_short_conv_tma(p, s, launched);
    if (e0 != cudaSuccess || launched) return e0;
    const long long warps = conv_grid_warps(p);
    if (warps == 0) return cudaSuccess;
    const long long blocks = (warps + kLayerThreads / 32 - 1) / (kLayerThreads / 32);
    switch (p.K) {
        case 1: short_conv_kernel<1><<<(unsigned)blocks, kLayerThreads, 0, s>>>(p); break;
        case 2: short_conv_kernel<2><<<(unsigned)blocks, kLayerThreads, 0, s>>>(p); break;
        case 3: short_conv_kernel<3><<<(unsigned)blocks, kLayerThreads, 0, s>>>(p); break;
        default: short_conv_kernel<4><<<(unsigned)blocks, kLayerThreads, 0, s>>>(p); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_output_gate(const GateParams &p, cudaStream_t s) {
    const long long warps = ((long long)p.N * p.HV + kGateRows - 1) / kGateRows;
    if (warps == 0) return cudaSuccess;
    const long long blocks = (warps + kLayerThreads / 32 - 1) / (kLayerThreads / 32);
    output_gate_kernel<<<(unsigned)blocks, kLayerThreads, 0, s>>>(p);
    return cudaGetLastError();
}

// Tensor map of a bf16 [B][T][C] tensor (channels innermost) with a box of
// [1][rows][256] channels.
static bool make_conv_map(CUtensorMap *map, const void *base, const ConvParams &p, int rows) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return false;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[3] = {(cuuint64_t)p.C, (cuuint64_t)p.T, (cuuint64_t)p.B};
    const cuuint64_t strides[2] = {(cuuint64_t)p.C * 2, (cuuint64_t)p.T * p.C * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kTC, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tiled kernel takes rows of a multiple of 256 channels, K <= 4, at least
// one token, and 16-byte aligned state buffers; everything else the warp kernel.
static bool conv_tma_eligible(const ConvParams &p) {
    return p.C % kTC == 0 && p.T > 0 && p.K >= 1 && p.K <= 4 && (p.head_dim == 0 || p.head_dim == 128) &&
           ((uintptr_t)p.state_in % 16 == 0) && ((uintptr_t)p.state_out % 16 == 0);
}

cudaError_t launch_short_conv_tma(const ConvParams &p, cudaStream_t s, bool &launched) {
    launched = false;
    if (!conv_tma_eligible(p)) return cudaSuccess;
    ConvTmaParams tp;
    tp.p = p;
    if (!make_conv_map(&tp.tx, p.x, p, kTT + kHalo) || (uintptr_t)p.y % 16 != 0) return cudaSuccess;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long ntiles = (long long)p.B * (p.C / kTC) * ((p.T + kTT - 1) / kTT);
    if (ntiles >= (1LL << 31)) return cudaSuccess;                 // the warp kernel takes it
    const long long grid = ntiles < sms ? ntiles : sms;
    switch (p.K) {
#define KDA_CONV_TMA(KK)                                                                                      \
    case KK:                                                                                                  \
        if ((e = cudaFuncSetAttribute(short_conv_tma_kernel<KK>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                      (int)TS_SMEM)) != cudaSuccess)                                          \
            return e;                                                                                         \
        short_conv_tma_kernel<KK><<<(unsigned)grid, kConvThreads, TS_SMEM, s>>>(tp);                         \
        break;
        KDA_CONV_TMA(1)
        KDA_CONV_TMA(2)
        KDA_CONV_TMA(3)
        default: KDA_CONV_TMA(4)
#undef KDA_CONV_TMA
    }
    launched = true;
    return cudaGetLastError();
}

cudaError_t read_and_clear_conv_error(unsigned int *out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_conv_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_conv_error, &zero, sizeof(unsigned int));
}

}  // namespace kda
