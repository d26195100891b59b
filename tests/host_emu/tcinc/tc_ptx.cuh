// Host model of the sm_100a instructions wrapped by the library's tc_ptx.cuh
// (same names and signatures), for running the tensor-core chunk kernel with
// one std::thread per CUDA thread: shared memory is the CTA's byte array and a
// shared address is an offset into it; tensor memory is a 128-lane x 512-column
// array of 32-bit cells; tcgen05.mma, tensor-map loads and tcgen05.commit run
// to completion in the issuing thread (their mbarrier arrivals follow at once);
// mbarriers keep arrival count, transaction bytes and phase; named barriers
// count their participants.
#pragma once
#include <stdint.h>

#include <atomic>
#include <chrono>
#include <cmath>
#include <condition_variable>
#include <cstring>
#include <mutex>
#include <thread>

namespace kda {
namespace tc {

// ---- the CTA being run (blocks run one after another) ----------------------
struct EmuMBar {
    int expected = 0, pending = 0;
    long long tx = 0;
    std::atomic<int> phase{0};
};
struct EmuNamedBar {
    std::mutex m;
    std::condition_variable cv;
    int arrived = 0;
    unsigned gen = 0;
    bool any = false, result = false;
};
struct EmuCta {
    uint8_t *smem = nullptr;       // shared address 0
    size_t smem_bytes = 0;
    uint32_t tmem[128][512];
    EmuMBar *bars = nullptr;       // one per 8 bytes of shared memory
    std::mutex bar_mutex;
    EmuNamedBar named[16];
};
extern EmuCta *g_cta;

inline uint8_t *shared_ptr(uint32_t addr) { return g_cta->smem + addr; }

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(static_cast<const uint8_t *>(p) - g_cta->smem);
}

// ---- descriptors (identical encodings) ---------------------------------------
__device__ __forceinline__ uint64_t kmaj_desc(uint32_t base, int rows, int s) {
    const uint32_t addr = base + (uint32_t)((s >> 2) * rows * 128 + (s & 3) * 32);
    uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}
__device__ __forceinline__ uint32_t mnmaj_chunk_off(int krow, int chunk) {
    return (uint32_t)(krow * 128 + ((chunk ^ (krow & 7)) << 4));
}
__device__ __forceinline__ uint64_t mnmaj_desc(uint32_t base, int s) {
    const uint32_t addr = base + (uint32_t)(s * 2048);
    uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)(8192u >> 4) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool negate_a = false,
                                                  bool b_mn_major = false, bool a_mn_major = false) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((negate_a ? 1u : 0u) << 13) | ((a_mn_major ? 1u : 0u) << 15) |
           ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---- operand reads -------------------------------------------------------------
inline float emu_bf16_at(uint32_t addr) {
    // 128-byte swizzle: the 16-byte chunk index (address bits 4-6) is XORed
    // with the 128-byte row index within the 1024-byte atom (bits 7-9).
    const uint32_t sw = addr ^ (((addr >> 7) & 7u) << 4);
    uint16_t h;
    std::memcpy(&h, shared_ptr(sw), 2);
    const uint32_t u = (uint32_t)h << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}
struct EmuDesc {
    uint32_t start, lbo, sbo;
};
inline EmuDesc emu_desc(uint64_t d) {
    return EmuDesc{(uint32_t)(d & 0x3FFFu) << 4, (uint32_t)((d >> 16) & 0x3FFFu) << 4,
                   (uint32_t)((d >> 32) & 0x3FFFu) << 4};
}
// Element (row `mn`, k-element `e` of the 16 of this k-step) of an SW128 operand.
inline float emu_operand(const EmuDesc &d, bool mn_major, int mn, int e) {
    if (!mn_major)   // K-major: rows of 128 B, 8-row atoms SBO apart
        return emu_bf16_at(d.start + (uint32_t)(mn >> 3) * d.sbo + (uint32_t)(mn & 7) * 128u + (uint32_t)e * 2u);
    // MN-major: 64-element MN blocks LBO apart; K-rows of 128 B, 8-row groups SBO apart
    return emu_bf16_at(d.start + (uint32_t)(mn >> 6) * d.lbo + (uint32_t)(e >> 3) * d.sbo +
                       (uint32_t)(e & 7) * 128u + (uint32_t)(mn & 63) * 2u);
}
inline float emu_tmem_bf16(uint32_t lane, uint32_t col, int e) {
    const uint32_t w = g_cta->tmem[lane][col + (uint32_t)(e >> 1)];
    const uint32_t u = (e & 1) ? (w & 0xFFFF0000u) : (w << 16);
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}
inline void emu_mma(uint32_t d_tmem, bool a_in_tmem, uint32_t a_tmem, uint64_t a_desc, uint64_t b_desc,
                    uint32_t idesc, uint32_t accumulate) {
    const int N = (int)((idesc >> 17) & 0x3Fu) << 3, M = (int)((idesc >> 24) & 0x1Fu) << 4;
    const bool neg = (idesc >> 13) & 1u, a_mn = (idesc >> 15) & 1u, b_mn = (idesc >> 16) & 1u;
    const EmuDesc A = emu_desc(a_desc), B = emu_desc(b_desc);
    const uint32_t dl = d_tmem >> 16, dc = d_tmem & 0xFFFFu, al = a_tmem >> 16, ac = a_tmem & 0xFFFFu;
    for (int m = 0; m < M; ++m) {
        float a[16];
        for (int e = 0; e < 16; ++e) {
            a[e] = a_in_tmem ? emu_tmem_bf16(al + (uint32_t)m, ac, e) : emu_operand(A, a_mn, m, e);
            if (neg) a[e] = -a[e];
        }
        for (int n = 0; n < N; ++n) {
            float acc = 0.f;
            for (int e = 0; e < 16; ++e) acc = std::fma(a[e], emu_operand(B, b_mn, n, e), acc);
            uint32_t &cell = g_cta->tmem[dl + (uint32_t)m][dc + (uint32_t)n];
            float old;
            std::memcpy(&old, &cell, 4);
            const float r = accumulate ? old + acc : acc;
            std::memcpy(&cell, &r, 4);
        }
    }
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    emu_mma(d_tmem, false, 0, a_desc, b_desc, idesc, accumulate);
}
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
    emu_mma(d_tmem, true, a_tmem, 0, b_desc, idesc, accumulate);
}

// ---- mbarriers -------------------------------------------------------------------
inline EmuMBar &emu_bar(uint32_t mbar) { return g_cta->bars[mbar >> 3]; }
inline void emu_bar_complete_if_done(EmuMBar &b) {
    if (b.pending == 0 && b.tx == 0) {
        b.pending = b.expected;
        b.phase.fetch_xor(1);
    }
}
__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
    std::lock_guard<std::mutex> l(g_cta->bar_mutex);
    EmuMBar &b = emu_bar(mbar);
    b.expected = b.pending = (int)count;
    b.tx = 0;
    b.phase.store(0);
}
__device__ __forceinline__ void fence_mbar_init() {}
__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
    std::lock_guard<std::mutex> l(g_cta->bar_mutex);
    EmuMBar &b = emu_bar(mbar);
    --b.pending;
    emu_bar_complete_if_done(b);
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t mbar, uint32_t bytes) {
    std::lock_guard<std::mutex> l(g_cta->bar_mutex);
    EmuMBar &b = emu_bar(mbar);
    b.tx += bytes;
    --b.pending;
    emu_bar_complete_if_done(b);
}
inline void emu_complete_tx(uint32_t mbar, uint32_t bytes) {
    std::lock_guard<std::mutex> l(g_cta->bar_mutex);
    EmuMBar &b = emu_bar(mbar);
    b.tx -= bytes;
    emu_bar_complete_if_done(b);
}
// The phase with this parity has completed once the current phase differs.
__device__ __forceinline__ bool mbar_try_wait(uint32_t mbar, uint32_t parity) {
    if (emu_bar(mbar).phase.load() != (int)parity) return true;
    std::this_thread::yield();
    return false;
}
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t mbar, uint32_t parity, uint32_t) {
    return mbar_try_wait(mbar, parity);
}
__device__ __forceinline__ void mma_commit(uint32_t mbar) { mbar_arrive(mbar); }

// ---- fences and tensor memory ------------------------------------------------------
__device__ __forceinline__ void fence_before_sync() { std::atomic_thread_fence(std::memory_order_seq_cst); }
__device__ __forceinline__ void fence_after_sync() { std::atomic_thread_fence(std::memory_order_seq_cst); }
__device__ __forceinline__ void fence_async_smem() { std::atomic_thread_fence(std::memory_order_seq_cst); }
// Warp-collective: one write of the address (column 0 of lane 0) for the warp.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t) {
    if ((threadIdx.x & 31u) == 0) {
        const uint32_t zero = 0;
        std::memcpy(shared_ptr(dst_smem), &zero, 4);
    }
    __syncwarp();
}
__device__ __forceinline__ void tmem_relinquish() {}
__device__ __forceinline__ void tmem_dealloc(uint32_t, uint32_t) {}
inline uint32_t emu_lane() { return threadIdx.x & 31u; }
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    const uint32_t lane = (taddr >> 16) + emu_lane(), col = taddr & 0xFFFFu;
    for (int i = 0; i < 16; ++i) std::memcpy(&v[i], &g_cta->tmem[lane][col + i], 4);
}
__device__ __forceinline__ void tmem_ld16x2(uint32_t t0, uint32_t t1, float (&v0)[16], float (&v1)[16]) {
    tmem_ld16(t0, v0);
    tmem_ld16(t1, v1);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    const uint32_t lane = (taddr >> 16) + emu_lane(), col = taddr & 0xFFFFu;
    for (int i = 0; i < 16; ++i) std::memcpy(&g_cta->tmem[lane][col + i], &v[i], 4);
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
    const uint32_t lane = (taddr >> 16) + emu_lane(), col = taddr & 0xFFFFu;
    for (int i = 0; i < 8; ++i) g_cta->tmem[lane][col + i] = v[i];
}
__device__ __forceinline__ void tmem_st_wait() { std::atomic_thread_fence(std::memory_order_seq_cst); }

// ---- named barriers ----------------------------------------------------------------
inline bool emu_named(int id, int nthreads, bool pred) {
    EmuNamedBar &b = g_cta->named[id];
    std::unique_lock<std::mutex> l(b.m);
    const unsigned gen = b.gen;
    b.any = b.any || pred;
    if (++b.arrived == nthreads) {
        b.result = b.any;
        b.any = false;
        b.arrived = 0;
        ++b.gen;
        b.cv.notify_all();
        return b.result;
    }
    b.cv.wait(l, [&] { return b.gen != gen; });
    return b.result;
}
__device__ __forceinline__ void named_bar(int id, int nthreads) { emu_named(id, nthreads, false); }
__device__ __forceinline__ bool named_bar_any(int id, int nthreads, bool pred) {
    return emu_named(id, nthreads, pred);
}

// ---- tensor-map loads ----------------------------------------------------------------
// The emulated CUtensorMap carries: base, dims[3], byte strides of dims 1 and 2,
// box[3], 128-byte swizzle flag (bf16 elements, zero fill out of range).
struct EmuTensorMap {
    const uint8_t *base;
    uint64_t dims[3], strides[2];
    uint32_t box[3];
    uint32_t swizzle128;
};
__device__ __forceinline__ void tma_load_3d(uint32_t dst_smem, const void *tmap, int c0, int c1, int c2,
                                            uint32_t mbar) {
    EmuTensorMap m;
    std::memcpy(&m, tmap, sizeof m);
    uint32_t off = 0;
    for (uint32_t z = 0; z < m.box[2]; ++z)
        for (uint32_t y = 0; y < m.box[1]; ++y)
            for (uint32_t x = 0; x < m.box[0]; ++x, off += 2) {
                const long long gx = (long long)c0 + x, gy = (long long)c1 + y, gz = (long long)c2 + z;
                uint16_t h = 0;
                if (gx >= 0 && gy >= 0 && gz >= 0 && gx < (long long)m.dims[0] && gy < (long long)m.dims[1] &&
                    gz < (long long)m.dims[2])
                    std::memcpy(&h, m.base + gz * m.strides[1] + gy * m.strides[0] + gx * 2, 2);
                uint32_t a = dst_smem + off;
                if (m.swizzle128) a ^= ((a >> 7) & 7u) << 4;
                std::memcpy(shared_ptr(a), &h, 2);
            }
    emu_complete_tx(mbar, off);
}
// Tensor store of one box: shared rows -> the tensor, elements outside it skipped
// (completes at once; the bulk-group waits below are then no-ops).
__device__ __forceinline__ void tma_store_3d(const void *tmap, int c0, int c1, int c2, uint32_t src_smem) {
    EmuTensorMap m;
    std::memcpy(&m, tmap, sizeof m);
    uint32_t off = 0;
    for (uint32_t z = 0; z < m.box[2]; ++z)
        for (uint32_t y = 0; y < m.box[1]; ++y)
            for (uint32_t x = 0; x < m.box[0]; ++x, off += 2) {
                const long long gx = (long long)c0 + x, gy = (long long)c1 + y, gz = (long long)c2 + z;
                if (gx < 0 || gy < 0 || gz < 0 || gx >= (long long)m.dims[0] || gy >= (long long)m.dims[1] ||
                    gz >= (long long)m.dims[2])
                    continue;
                uint32_t a = src_smem + off;
                if (m.swizzle128) a ^= ((a >> 7) & 7u) << 4;
                std::memcpy(const_cast<uint8_t *>(m.base) + gz * m.strides[1] + gy * m.strides[0] + gx * 2,
                            shared_ptr(a), 2);
            }
}
__device__ __forceinline__ void prefetch_tensormap(const void *) {}
__device__ __forceinline__ void tma_prefetch_3d(const void *, int, int, int) {}
// Bulk copies complete at once (the load's mbarrier arrival follows).
__device__ __forceinline__ void bulk_load(uint32_t dst_smem, const void *src, uint32_t bytes, uint32_t mbar) {
    std::memcpy(shared_ptr(dst_smem), src, bytes);
    emu_complete_tx(mbar, bytes);
}
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src_smem, uint32_t bytes) {
    std::memcpy(dst, shared_ptr(src_smem), bytes);
}
__device__ __forceinline__ void bulk_commit() {}
template <int N>
__device__ __forceinline__ void bulk_wait_read() {}
template <int N>
__device__ __forceinline__ void bulk_wait() {}

// ---- special functions, conversions, warp-level tf32 mma -------------------------------
__device__ __forceinline__ float ex2_approx(float x) { return std::exp2(x); }
__device__ __forceinline__ float rcp_approx(float x) { return 1.0f / x; }
__device__ __forceinline__ float lg2_approx(float x) { return std::log2(x); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return ((uint32_t)__float2bfloat16_rn(hi).x << 16) | (uint32_t)__float2bfloat16_rn(lo).x;
}
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t u;
    std::memcpy(&u, &x, 4);
    if ((u & 0x7F800000u) != 0x7F800000u) u += 0x1000u;    // round half away from zero
    return u & 0xFFFFE000u;
}
struct EmuTf32Slots {
    float a[32][4], b[32][2], d[32][4];
};
extern EmuTf32Slots g_tf32[32];
__device__ __forceinline__ void mma_tf32_16x8x8(float d[4], const uint32_t a[4], const uint32_t b[2]) {
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    EmuTf32Slots &s = g_tf32[w];
    for (int i = 0; i < 4; ++i) std::memcpy(&s.a[l][i], &a[i], 4);
    for (int i = 0; i < 2; ++i) std::memcpy(&s.b[l][i], &b[i], 4);
    for (int i = 0; i < 4; ++i) s.d[l][i] = d[i];
    __syncwarp();
    // A[16][8], B[8][8] from the fragments (g = lane / 4, t = lane % 4)
    const int g = l >> 2, t = l & 3;
    auto Aat = [&](int r, int k) {
        const int ll = (r & 7) * 4 + (k & 3);
        return s.a[ll][(r >> 3) + 2 * (k >> 2)];
    };
    auto Bat = [&](int k, int n) { return s.b[n * 4 + (k & 3)][k >> 2]; };
    float out[4];
    const int rows[4] = {g, g, g + 8, g + 8}, cols[4] = {2 * t, 2 * t + 1, 2 * t, 2 * t + 1};
    for (int i = 0; i < 4; ++i) {
        float acc = d[i];
        for (int k = 0; k < 8; ++k) acc = std::fma(Aat(rows[i], k), Bat(k, cols[i]), acc);
        out[i] = acc;
    }
    __syncwarp();
    for (int i = 0; i < 4; ++i) d[i] = out[i];
}

}  // namespace tc
}  // namespace kda
