// mx_gemm.cu -- block-scaled GEMM (placeholder until the tcgen05 kernel lands).
#include <cuda_runtime.h>

#include "mx.h"
#include "mx_internal.h"

// Device status word: kernels that give up a bounded wait record MX_ERR_TIMEOUT here.
__device__ int g_mx_status;

int mx_launch_gemm(const MxGemmArgs &, cudaStream_t) { return MX_ERR_UNSUPPORTED; }

int mx_read_device_status(cudaStream_t st) {
    if (cudaStreamSynchronize(st) != cudaSuccess) return MX_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_mx_status, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_mx_status, &zero, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    return v;
}
