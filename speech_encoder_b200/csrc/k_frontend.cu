// Feature-encoder layer 0 and the row LayerNorm.
//
// Conv layer 0 is Conv1d(1 -> 512, kernel 10, stride 5) on the PCM.  With the
// "group" layout it is followed by GroupNorm(512 groups, 512 channels): each
// channel normalised with its mean and variance over every frame of the clip
// (the TensorRT wav2vec2 README's kernel-time paragraph: "a group norm over
// every time step of the clip").  Because conv 0 is linear in the PCM, those
// statistics follow exactly from the mean vector m and covariance S of the
// 10-sample input windows:  mean_c = w_c . m  and  var_c = w_c^T S w_c.  So
// instead of materialising the 512-channel output to reduce it (the largest
// kernel in the pages' TensorRT profile), one pass over the PCM accumulates the
// 10 + 55 window moments, and the conv-0 kernel applies the normalisation as
// it computes each output.  With the "layer" layout conv 0 has a bias and a
// per-frame LayerNorm over the 512 channels, computed in the same kernel.
#include "ptx.cuh"
#include "w2v_internal.h"

namespace w2v {

constexpr int kC = 512;
constexpr int kK0 = 10;
constexpr int kS0 = 5;
constexpr int kMom = kK0 + kK0 * (kK0 + 1) / 2;  // 65

// Moments of the conv-0 input windows of one clip: grid (nblocks, batch).
// Every block writes its 65 partial sums; the last block of a clip to finish
// (atomic ticket) adds the partials in block order (deterministic), turns them
// into per-channel GroupNorm scale/shift (fp64) and re-arms the ticket.
__global__ void __launch_bounds__(256)
gn_moments_kernel(const float* __restrict__ pcm, int n, int t0, const float* __restrict__ w0,
                  const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                  double* __restrict__ partial, unsigned* __restrict__ ticket, float2* __restrict__ scale_shift) {
  if (threadIdx.x == 0) pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.y;
  const float* x = pcm + static_cast<int64_t>(b) * n;
  float s[kMom];
#pragma unroll
  for (int i = 0; i < kMom; ++i) s[i] = 0.f;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < t0; t += gridDim.x * blockDim.x) {
    float w[kK0];
#pragma unroll
    for (int j = 0; j < kK0; ++j) w[j] = __ldg(x + kS0 * t + j);
    int idx = kK0;
#pragma unroll
    for (int j = 0; j < kK0; ++j) {
      s[j] += w[j];
#pragma unroll
      for (int jj = j; jj < kK0; ++jj) s[idx++] += w[j] * w[jj];
    }
  }
  __shared__ float red[8][kMom];
  __shared__ double mom[kMom];
  __shared__ unsigned last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < kMom; ++i) {
    float v = s[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][i] = v;
  }
  __syncthreads();
  double* mine = partial + (static_cast<int64_t>(b) * gridDim.x + blockIdx.x) * kMom;
  if (threadIdx.x < kMom) {
    double sum = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) sum += red[w][threadIdx.x];
    mine[threadIdx.x] = sum;
    __threadfence();
  }
  __syncthreads();
  if (threadIdx.x == 0) last = (atomicAdd(ticket + b, 1u) == gridDim.x - 1) ? 1u : 0u;
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (threadIdx.x < kMom) {
    const volatile double* pb = partial + static_cast<int64_t>(b) * gridDim.x * kMom;
    double sum = 0.0;
    for (unsigned k = 0; k < gridDim.x; ++k) sum += pb[k * kMom + threadIdx.x];
    mom[threadIdx.x] = sum;
  }
  __syncthreads();
  if (threadIdx.x == 0) ticket[b] = 0u;
  const double inv = 1.0 / static_cast<double>(t0);
  for (int c = threadIdx.x; c < kC; c += blockDim.x) {
    double w[kK0], m[kK0];
#pragma unroll
    for (int j = 0; j < kK0; ++j) {
      w[j] = w0[c * kK0 + j];
      m[j] = mom[j] * inv;
    }
    double mean = 0.0, var = 0.0;
    int idx = kK0;
#pragma unroll
    for (int j = 0; j < kK0; ++j) {
      mean += w[j] * m[j];
#pragma unroll
      for (int jj = j; jj < kK0; ++jj) {
        const double cov = mom[idx++] * inv - m[j] * m[jj];
        var += (jj == j ? 1.0 : 2.0) * w[j] * w[jj] * cov;
      }
    }
    if (var < 0.0) var = 0.0;
    const double scale = static_cast<double>(gamma[c]) / sqrt(var + static_cast<double>(eps));
    // a conv bias cancels inside the normalisation, so it never appears here
    scale_shift[b * kC + c] = make_float2(static_cast<float>(scale),
                                          static_cast<float>(static_cast<double>(beta[c]) - mean * scale));
  }
}

int gn_moment_blocks(int t0) {
  int nb = (t0 + 256 * 8 - 1) / (256 * 8);
  if (nb > 296) nb = 296;
  if (nb < 1) nb = 1;
  return nb;
}

cudaError_t launch_gn_moments(const float* pcm, int n, int batch, int t0, const float* w0, const float* gamma,
                              const float* beta, float eps, double* partial, unsigned* ticket, float2* scale_shift,
                              cudaStream_t st) {
  return launch_pdl(gn_moments_kernel, dim3(gn_moment_blocks(t0), batch), dim3(256), 0, st, pcm, n, t0, w0, gamma,
                    beta, eps, partial, ticket, scale_shift);
}

// One warp per output frame; lane l owns channel pairs (2l + 64i, 2l + 64i + 1),
// i = 0..7, so each half2 store instruction of a warp writes 128 contiguous bytes.
// group layout: y*scale + shift from the clip's GroupNorm statistics;
// layer layout: bias, then LayerNorm over the 512 channels of the frame.
__global__ void __launch_bounds__(256, 2)
conv0_kernel(const float* __restrict__ pcm, int n, int t0, int clip_rows, const float* __restrict__ w0,
             const float* __restrict__ b0, const float* __restrict__ gamma, const float* __restrict__ beta,
             const float2* __restrict__ scale_shift, int layer_norm, float eps, int act, __half* __restrict__ out) {
  __shared__ __align__(16) float sw[kK0][kC];
  __shared__ __align__(16) float sa[kC];  // group: scale;  layer: gamma
  __shared__ __align__(16) float sb[kC];  // group: shift;  layer: beta
  __shared__ __align__(16) float sbias[kC];
  if (threadIdx.x == 0) pdl_launch_dependents();
  const int b = blockIdx.y;
  for (int i = threadIdx.x; i < kC * kK0; i += blockDim.x) sw[i % kK0][i / kK0] = w0[i];
  if (layer_norm) {
    for (int c = threadIdx.x; c < kC; c += blockDim.x) {
      sa[c] = gamma[c];
      sb[c] = beta[c];
      sbias[c] = b0 ? b0[c] : 0.f;
    }
  }
  pdl_wait();
  if (!layer_norm) {
    for (int c = threadIdx.x; c < kC; c += blockDim.x) {
      const float2 v = scale_shift[b * kC + c];
      sa[c] = v.x;
      sb[c] = v.y;
    }
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const float* x = pcm + static_cast<int64_t>(b) * n;
  __half* ob = out + static_cast<int64_t>(b) * clip_rows * kC;
  for (int t = blockIdx.x * wpb + warp; t < t0; t += gridDim.x * wpb) {
    float xw[kK0];
#pragma unroll
    for (int j = 0; j < kK0; ++j) xw[j] = __ldg(x + kS0 * t + j);
    float y[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = 2 * lane + 64 * i;
      float y0 = 0.f, y1 = 0.f;
#pragma unroll
      for (int j = 0; j < kK0; ++j) {
        const float2 w = *reinterpret_cast<const float2*>(&sw[j][c]);
        y0 = fmaf(w.x, xw[j], y0);
        y1 = fmaf(w.y, xw[j], y1);
      }
      y[2 * i] = y0;
      y[2 * i + 1] = y1;
    }
    if (layer_norm) {
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int c = 2 * lane + 64 * i;
        y[2 * i] += sbias[c];
        y[2 * i + 1] += sbias[c + 1];
        sum += y[2 * i] + y[2 * i + 1];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float mean = sum * (1.0f / kC);
      float sq = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float dlt = y[i] - mean;
        sq += dlt * dlt;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
      const float rstd = rsqrtf(sq * (1.0f / kC) + eps);
#pragma unroll
      for (int i = 0; i < 16; ++i) y[i] = (y[i] - mean) * rstd;
    }
    __half* orow = ob + static_cast<int64_t>(t) * kC;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = 2 * lane + 64 * i;
      const float a0 = fmaf(y[2 * i], sa[c], sb[c]);
      const float a1 = fmaf(y[2 * i + 1], sa[c + 1], sb[c + 1]);
      *reinterpret_cast<__half2*>(orow + c) = __floats2half2_rn(apply_act(a0, act), apply_act(a1, act));
    }
  }
}

cudaError_t launch_conv0(const float* pcm, int n, int batch, int t0, int clip_rows, const float* w0, const float* b0,
                         const float* gamma, const float* beta, const float2* scale_shift, int layer_norm, float eps,
                         int act, __half* out, cudaStream_t st) {
  int nbx = (t0 + 8 * 8 - 1) / (8 * 8);  // ~8 frames per warp
  if (nbx > 148 * 4) nbx = 148 * 4;
  if (nbx < 1) nbx = 1;
  return launch_pdl(conv0_kernel, dim3(nbx, batch), dim3(256), 0, st, pcm, n, t0, clip_rows, w0, b0, gamma, beta,
                    scale_shift, layer_norm, eps, act, out);
}

// ------------------------------------------------------------------ LayerNorm
// One warp per row.  fp16 input: lane owns 8-element chunks (lane + 32 i);
// fp32 input: 4-element chunks.  Two passes over registers (mean, then the
// centred sum of squares), fp32 throughout, fp16 output.
template <int COLS, bool F32IN>
__global__ void __launch_bounds__(256)
layernorm_kernel(const void* __restrict__ xin, __half* __restrict__ y, int rows, const float* __restrict__ gamma,
                 const float* __restrict__ beta, float eps, int act) {
  constexpr int VEC = F32IN ? 4 : 8;
  constexpr int NCH = COLS / (32 * VEC);
  constexpr int NPL = COLS / 32;
  if (threadIdx.x == 0) pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  float v[NPL];
  if (F32IN) {
    const float* xr = static_cast<const float*>(xin) + static_cast<int64_t>(row) * COLS;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const float4 f = *reinterpret_cast<const float4*>(xr + (lane + 32 * i) * 4);
      v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
  } else {
    const __half* xr = static_cast<const __half*>(xin) + static_cast<int64_t>(row) * COLS;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const uint4 u = *reinterpret_cast<const uint4*>(xr + (lane + 32 * i) * 8);
      const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(h[j]);
        v[8 * i + 2 * j] = f.x;
        v[8 * i + 2 * j + 1] = f.y;
      }
    }
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NPL; ++i) s += v[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s * (1.0f / COLS);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const float d = v[i] - mean;
    q += d * d;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q * (1.0f / COLS) + eps);
  __half* yr = y + static_cast<int64_t>(row) * COLS;
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c0 = (lane + 32 * i) * VEC;
    __align__(16) __half2 hv[VEC / 2];
#pragma unroll
    for (int j = 0; j < VEC; j += 2) {
      const float a0 = (v[VEC * i + j] - mean) * rstd * __ldg(gamma + c0 + j) + __ldg(beta + c0 + j);
      const float a1 = (v[VEC * i + j + 1] - mean) * rstd * __ldg(gamma + c0 + j + 1) + __ldg(beta + c0 + j + 1);
      hv[j / 2] = __floats2half2_rn(apply_act(a0, act), apply_act(a1, act));
    }
    if (VEC == 8)
      *reinterpret_cast<uint4*>(yr + c0) = *reinterpret_cast<const uint4*>(hv);
    else
      *reinterpret_cast<uint2*>(yr + c0) = *reinterpret_cast<const uint2*>(hv);
  }
}

template <int COLS>
static void ln_dispatch(const void* x, int in_f32, __half* y, int rows, const float* g, const float* b, float eps,
                        int act, cudaStream_t st) {
  const int blocks = (rows + 7) / 8;
  if (in_f32)
    launch_pdl(layernorm_kernel<COLS, true>, dim3(blocks), dim3(256), 0, st, x, y, rows, g, b, eps, act);
  else
    launch_pdl(layernorm_kernel<COLS, false>, dim3(blocks), dim3(256), 0, st, x, y, rows, g, b, eps, act);
}

cudaError_t launch_layernorm(const void* x, int in_f32, __half* y, int rows, int cols, const float* gamma,
                             const float* beta, float eps, int act, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  switch (cols) {
    case 512: ln_dispatch<512>(x, in_f32, y, rows, gamma, beta, eps, act, st); break;
    case 768: ln_dispatch<768>(x, in_f32, y, rows, gamma, beta, eps, act, st); break;
    case 1024: ln_dispatch<1024>(x, in_f32, y, rows, gamma, beta, eps, act, st); break;
    case 256: ln_dispatch<256>(x, in_f32, y, rows, gamma, beta, eps, act, st); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace w2v
