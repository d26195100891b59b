// One CUDA block = blockDim.x std::threads; __syncthreads / __syncwarp are
// std::barriers, a thread that leaves the kernel drops out of them (as an
// exited GPU thread does), __shfl_xor_sync exchanges through per-warp slots.
#include <atomic>
#include <barrier>
#include <functional>
#include <memory>
#include <thread>
#include <vector>

#include "cuda_runtime.h"

thread_local uint3 threadIdx, blockIdx;
thread_local dim3 blockDim, gridDim;

namespace {
std::unique_ptr<std::barrier<>> g_block;
std::vector<std::unique_ptr<std::barrier<>>> g_warp;
float g_slots[32][32];
}

void __syncthreads() { g_block->arrive_and_wait(); }
// Barrier with an OR of the threads' predicates.  Call k (counted per thread,
// the same k in every thread of the block) accumulates in slot k % 3; after
// the barrier thread 0 clears slot (k + 2) % 3, whose last reads were before
// this barrier and whose next writes come after the next one.
static std::atomic<int> g_or_acc[3];
thread_local unsigned g_or_calls = 0;
int __syncthreads_or(int pred) {
    const unsigned k = g_or_calls++ % 3;
    if (pred) g_or_acc[k].fetch_or(1);
    g_block->arrive_and_wait();
    const int r = g_or_acc[k].load();
    if (threadIdx.x == 0) g_or_acc[(k + 2) % 3].store(0);
    return r;
}
void __syncwarp(unsigned) { g_warp[threadIdx.x / 32]->arrive_and_wait(); }
float __shfl_xor_sync(unsigned, float v, int off) {
    const int w = threadIdx.x / 32, l = threadIdx.x % 32;
    g_slots[w][l] = v;
    g_warp[w]->arrive_and_wait();
    const float r = g_slots[w][l ^ off];
    g_warp[w]->arrive_and_wait();
    return r;
}

// Runs fn(block) on every thread of every block of the grid, blocks in order;
// on_block(bx, by) runs before each block's threads start.
void emu_launch_cb(dim3 grid, dim3 block, const std::function<void(unsigned, unsigned)> &on_block,
                   const std::function<void()> &fn);
void emu_launch(dim3 grid, dim3 block, const std::function<void()> &fn) {
    emu_launch_cb(grid, block, [](unsigned, unsigned) {}, fn);
}
void emu_launch_cb(dim3 grid, dim3 block, const std::function<void(unsigned, unsigned)> &on_block,
                   const std::function<void()> &fn) {
    const unsigned nt = block.x;
    for (unsigned by = 0; by < grid.y; ++by)
        for (unsigned bx = 0; bx < grid.x; ++bx) {
            on_block(bx, by);
            for (auto &a : g_or_acc) a.store(0);
            g_block = std::make_unique<std::barrier<>>(nt);
            g_warp.clear();
            for (unsigned w = 0; w < (nt + 31) / 32; ++w)
                g_warp.push_back(std::make_unique<std::barrier<>>(std::min(32u, nt - 32 * w)));
            std::vector<std::thread> th;
            for (unsigned t = 0; t < nt; ++t)
                th.emplace_back([=, &fn] {
                    threadIdx = uint3{t, 0, 0};
                    blockIdx = uint3{bx, by, 0};
                    blockDim = block;
                    gridDim = grid;
                    fn();
                    g_warp[t / 32]->arrive_and_drop();
                    g_block->arrive_and_drop();
                });
            for (auto &x : th) x.join();
        }
}
