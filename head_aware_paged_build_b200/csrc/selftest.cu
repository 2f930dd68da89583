// segpaged_eval_exp2_fma: the FMA-pipe 2^x of the bf16 prefill kernel, run on
// its own so that its error bound can be checked on the device that uses it.
#include <string>

#include "device_common.cuh"
#include "kernels.h"

namespace sp {
namespace {

__global__ void eval_exp2_fma_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = 2 * (int64_t(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
  float e0, e1;
  exp2_poly_pair(f2_pack(x0, x1), e0, e1);
  y[i] = e0;
  if (i + 1 < n) y[i + 1] = e1;
}

}  // namespace
}  // namespace sp

extern "C" sp_status segpaged_eval_exp2_fma(const float* d_x, float* d_y, int64_t n, void* stream) {
  using namespace sp;
  if (n < 0) return fail(SP_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return SP_OK;
  if (!d_x || !d_y || (reinterpret_cast<uintptr_t>(d_x) & 3) || (reinterpret_cast<uintptr_t>(d_y) & 3))
    return fail(SP_ERR_INVALID_ARG, "d_x and d_y must be 4-byte aligned device pointers");
  if (n > (int64_t(1) << 40)) return fail(SP_ERR_INVALID_ARG, "n above 2^40");
  const int64_t pairs = (n + 1) / 2;
  const unsigned blocks = unsigned((pairs + 255) / 256);
  eval_exp2_fma_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(d_x, d_y, n);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SP_OK : fail(SP_ERR_CUDA, std::string("eval_exp2_fma launch: ") + cudaGetErrorString(e));
}
