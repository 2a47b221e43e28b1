// The raw-PCM front door: a long clip cut into fixed windows for the forward
// pass.  The pages run the encoder over a fixed window and zero-pad a short
// clip to it, decoding only its valid frames; a clip longer than the window
// becomes consecutive windows the same way.  Each window is normalised over
// its own valid samples to zero mean and unit variance,
// (x - mean) / sqrt(var + 1e-7) with the biased variance, and only then
// zero-padded, as a short clip is normalised before its padding.
//
// One CTA per window (grid = windows): two passes over the valid samples for
// the mean and the variance about it, each reduced in a fixed order (per
// thread strided sums, then a shared-memory tree), then one pass that writes
// the normalised samples and the zeros.
#include "w2v.h"
#include "w2v_internal.h"

namespace w2v {
namespace {

constexpr int kWinThreads = 256;

__device__ float block_sum(float v, float* red) {
  const int t = threadIdx.x;
  red[t] = v;
  __syncthreads();
#pragma unroll
  for (int s = kWinThreads / 2; s > 0; s >>= 1) {
    if (t < s) red[t] += red[t + s];
    __syncthreads();
  }
  const float r = red[0];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kWinThreads)
window_pcm_kernel(const float* pcm, int64_t n, int window, float* out) {
  __shared__ float red[kWinThreads];
  const int64_t w = blockIdx.x;
  const int64_t start = w * window;
  const int64_t left = n - start;
  const int valid = left < window ? static_cast<int>(left) : window;  // >= 1: grid = ceil(n / window)
  const float* x = pcm + start;
  float* y = out + w * static_cast<int64_t>(window);
  float s = 0.f;
  for (int i = threadIdx.x; i < valid; i += kWinThreads) s += x[i];
  const float mean = block_sum(s, red) / static_cast<float>(valid);
  float q = 0.f;
  for (int i = threadIdx.x; i < valid; i += kWinThreads) {
    const float d = x[i] - mean;
    q = fmaf(d, d, q);
  }
  const float var = block_sum(q, red) / static_cast<float>(valid);
  const float rstd = rsqrtf(var + 1e-7f);
  for (int i = threadIdx.x; i < valid; i += kWinThreads) y[i] = (x[i] - mean) * rstd;
  for (int i = valid + threadIdx.x; i < window; i += kWinThreads) y[i] = 0.f;
}

}  // namespace
}  // namespace w2v

extern "C" int w2v_num_windows(int n_samples, int window) {
  if (n_samples <= 0 || window <= 0) return 0;
  return static_cast<int>((static_cast<int64_t>(n_samples) + window - 1) / window);
}

extern "C" int w2v_window_pcm(const float* pcm_dev, int n_samples, int window, float* out_dev, void* stream) {
  if (!pcm_dev || !out_dev) return W2V_EINVAL;
  if (n_samples < 1 || window < 1) return W2V_ESHAPE;
  const int nw = w2v_num_windows(n_samples, window);
  w2v::window_pcm_kernel<<<nw, w2v::kWinThreads, 0, static_cast<cudaStream_t>(stream)>>>(pcm_dev, n_samples, window,
                                                                                          out_dev);
  return cudaGetLastError() == cudaSuccess ? W2V_OK : W2V_ECUDA;
}
