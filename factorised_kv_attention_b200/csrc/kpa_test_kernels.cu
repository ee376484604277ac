// kpa_test_kernels.cu -- small kernels that expose a device helper of the library to
// its tests, so that the helper's numbers can be checked on their own.
#include "kpa_f32x2.cuh"
#include "kpa_internal.cuh"

namespace kpa {
namespace {

// y = 2^x through exp2_poly2 (the prefill's FMA-pipe exponential), one pair per thread
__global__ void exp2_poly_kernel(const float *x, float *y, int64_t n) {
    const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const bool pair = i + 1 < n;
    const float2 r = f32x2::exp2_poly2(make_float2(x[i], pair ? x[i + 1] : x[i]));
    y[i] = r.x;
    if (pair) y[i + 1] = r.y;
}

}  // namespace
}  // namespace kpa

extern "C" kpa_status kpa_test_exp2_poly(const float *x, float *y, int64_t n, kpa_stream stream) {
    if (n < 0 || (n > 0 && (!x || !y))) return KPA_ERR_INVALID_ARG;
    if (n == 0) return KPA_OK;
    if (n > ((int64_t)1 << 40)) return KPA_ERR_UNSUPPORTED;
    const int64_t pairs = (n + 1) / 2;
    const unsigned blocks = (unsigned)((pairs + 255) / 256);
    kpa::exp2_poly_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(x, y, n);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        kpa::record_cuda_error(e);
        return KPA_ERR_CUDA;
    }
    return KPA_OK;
}
