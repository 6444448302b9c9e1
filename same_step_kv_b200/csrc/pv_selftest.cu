// Self-test entry point: the polynomial exp2 of pv_math.cuh, elementwise.
#include "pv_internal.h"
#include "pv_math.cuh"

namespace pv {
namespace {

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, size_t n) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x)
        y[i] = exp2_poly(x[i]);
}

}  // namespace
}  // namespace pv

extern "C" pv_status pv_selftest_exp2_poly(const float* x, float* y, size_t n, void* cuda_stream) {
    if (n == 0) return PV_OK;
    if (!x || !y) return pv::report_error(PV_ERR_INVALID_ARG, "pv_selftest_exp2_poly: NULL pointer");
    const int grid = (int)std::min<size_t>((n + 255) / 256, 4096);
    pv::exp2_poly_kernel<<<grid, 256, 0, (cudaStream_t)cuda_stream>>>(x, y, n);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return pv::report_error(PV_ERR_CUDA, cudaGetErrorString(e));
    return PV_OK;
}
