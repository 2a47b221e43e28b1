// Element-wise evaluation of the device math helpers that the fused kernels
// use inside their epilogues and softmax, so that each approximation can be
// checked on its own against its stated error bound over its whole input
// range (the whole-model tests only see them through the logits):
//   fn 0  exp2_affine_f16x2:      2^(c x + b) as fp16, exponent unit (f16x2)
//   fn 1  exp2_affine_poly_f16x2: the same on the FMA/ALU pipes (cubic)
//   fn 2  gelu_tanh2:             tanh-GELU of a pair, fp16x2 exponent
//   fn 3  gelu_tanh:              tanh-GELU, fp32 with the hardware tanh
//   fn 4  gelu_erf:               exact GELU through erff
//   fn 5  exp2f(c x + b):         CUDA's own exp2f, for comparison
// The pair forms take elements 2i and 2i+1 together (n must be even).
#include "ptx.cuh"
#include "w2v.h"
#include "w2v_internal.h"
#include "w2v_ops.h"

namespace w2v {

__global__ void pointwise_kernel(int fn, const float* __restrict__ x, int n, float c, float b, float* __restrict__ y) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (fn <= 2) {
    const int p = i;  // pair index
    if (2 * p + 1 >= n) return;
    const float x0 = x[2 * p], x1 = x[2 * p + 1];
    float2 r;
    if (fn == 0 || fn == 1) {
      const uint32_t h = fn == 0 ? exp2_affine_f16x2(x0, x1, c, b) : exp2_affine_poly_f16x2(x0, x1, c, b);
      r = __half22float2(*reinterpret_cast<const __half2*>(&h));
    } else {
      r = gelu_tanh2(make_float2(x0, x1));
    }
    y[2 * p] = r.x;
    y[2 * p + 1] = r.y;
    return;
  }
  if (i >= n) return;
  const float v = x[i];
  float r = 0.f;
  if (fn == 3) r = gelu_tanh(v);
  else if (fn == 4) r = gelu_erf(v);
  else r = exp2f(fmaf(v, c, b));
  y[i] = r;
}

}  // namespace w2v

extern "C" int w2v_op_pointwise(int fn, const float* x_dev, int n, float c, float b, float* y_dev, void* stream) {
  if (!x_dev || !y_dev) return W2V_EINVAL;
  if (fn < 0 || fn > 5) return W2V_EINVAL;
  if (n < 0 || (fn <= 2 && n % 2 != 0)) return W2V_ESHAPE;
  if (n == 0) return W2V_OK;
  const int threads = 256;
  const int work = fn <= 2 ? n / 2 : n;
  w2v::pointwise_kernel<<<(work + threads - 1) / threads, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      fn, x_dev, n, c, b, y_dev);
  return cudaGetLastError() == cudaSuccess ? W2V_OK : W2V_ECUDA;
}
