// tcgen05 BF16 chunk kernel (placeholder until the tensor-core path lands) and
// the device error word used by bounded waits.
#include "kda_internal.cuh"

namespace kda {

__device__ unsigned int g_device_error = 0;

bool chunk_tc_supported(const ChunkParams &p, bool bf16) {
    (void)p;
    (void)bf16;
    return false;
}

cudaError_t launch_chunk_tc(const ChunkParams &p, cudaStream_t s) {
    (void)p;
    (void)s;
    return cudaErrorNotSupported;
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
