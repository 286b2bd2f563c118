// hs2_selftest.cu -- diagnostics: evaluate the library's exp2 implementations
// on caller-given points, so tests can bound their error on the device.
#include "exp2_poly.cuh"
#include "hs2_kernels.h"

namespace hs2 {
namespace {
__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float v = x[i];
    y[i] = ex2(v);
    y[n + i] = exp2_poly<3>(v);
    y[2 * n + i] = exp2_poly<5>(v);
    // the packed form, fed (x, x/2) so both lanes see varied inputs
    const float2 r = exp2_poly5_x2(make_float2(v, 0.5f * v));
    y[3 * n + i] = r.x;
    y[4 * n + i] = r.y;
}
}  // namespace
}  // namespace hs2

extern "C" hs2_status hs2_selftest_exp2(const float* x, float* y, int n, hs2_stream_t stream) {
    if (n < 0 || (n > 0 && (x == nullptr || y == nullptr))) return HS2_ERR_INVALID_ARG;
    if (n == 0) return HS2_OK;
    hs2::exp2_selftest_kernel<<<(n + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
    hs2::count_launch();
    return cudaGetLastError() == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}
