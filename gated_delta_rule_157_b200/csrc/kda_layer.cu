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
// by warp shuffles, and nothing read twice.
#include <cuda_bf16.h>
#include <stdint.h>

#include "kda_internal.cuh"

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

}  // namespace

cudaError_t launch_short_conv(const ConvParams &p, cudaStream_t s) {
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

}  // namespace kda
