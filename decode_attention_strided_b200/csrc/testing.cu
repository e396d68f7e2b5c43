// testing.cu -- test support: the device implementations of the codec
// nonlinearity, run on caller-chosen inputs (include/deltakv_testing.h).
//
// The tensor-core kernels evaluate GELU with fast forms of their own
// (common.cuh); a host test holds each form to its stated error bound by
// running exactly these device functions over a dense grid and edge values.
#include "common.cuh"
#include "deltakv_testing.h"

namespace dkv {
namespace {

__global__ void act_forms_kernel(int form, const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const bool two = i + 1 < n;
  const float a = x[i], b = two ? x[i + 1] : 0.f;
  float ya = 0.f, yb = 0.f;
  switch (form) {
    case DELTAKV_TEST_ACT_GELU_ERFF:
      ya = act_eval(DELTAKV_ACT_GELU_ERF, a);
      yb = act_eval(DELTAKV_ACT_GELU_ERF, b);
      break;
    case DELTAKV_TEST_ACT_GELU_FAST:
      ya = gelu_fast(a);
      yb = gelu_fast(b);
      break;
    case DELTAKV_TEST_ACT_GELU_FAST2: {
      const float2 r = gelu_fast2(a, b);
      ya = r.x;
      yb = r.y;
      break;
    }
    case DELTAKV_TEST_ACT_GELU_TANHFIT2: {
      const float2 r = gelu_tanhfit2(a, b);
      ya = r.x;
      yb = r.y;
      break;
    }
    default:  // DELTAKV_TEST_ACT_GELU_TANH
      ya = act_eval(DELTAKV_ACT_GELU_TANH, a);
      yb = act_eval(DELTAKV_ACT_GELU_TANH, b);
      break;
  }
  y[i] = ya;
  if (two) y[i + 1] = yb;
}

}  // namespace
}  // namespace dkv

extern "C" deltakv_status deltakv_test_activation(int32_t form, const float* x, float* y, int64_t n,
                                                  deltakv_stream_t stream) {
  if (form < DELTAKV_TEST_ACT_GELU_ERFF || form > DELTAKV_TEST_ACT_GELU_TANHFIT2 || n < 0)
    return DELTAKV_ERR_INVALID_ARG;
  if (n == 0) return DELTAKV_OK;
  if (!x || !y) return DELTAKV_ERR_INVALID_ARG;
  const int64_t pairs = (n + 1) / 2;
  const int threads = 256;
  const int64_t blocks = (pairs + threads - 1) / threads;
  if (blocks > 0x7fffffff) return DELTAKV_ERR_INVALID_ARG;
  dkv::act_forms_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(form, x, y, n);
  return cudaGetLastError() == cudaSuccess ? DELTAKV_OK : DELTAKV_ERR_CUDA;
}
