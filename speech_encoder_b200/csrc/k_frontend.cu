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
gn_moments_kernel(const float* pcm, int n, int t0, const float* __restrict__ w0,
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
    for (int j = 0; j < kK0; ++j) w[j] = x[kS0 * t + j];
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
  {
    // All 256 threads add the per-block partials (L2-coherent loads, which
    // pipeline) in four fixed groups, then the groups combine in order.
    __shared__ double part[4][kMom];
    const double* pb = partial + static_cast<int64_t>(b) * gridDim.x * kMom;
    const int mi = threadIdx.x % kMom, grp = threadIdx.x / kMom;  // 260 slots > 256 threads: grp 3 has 61
    if (grp < 4) {
      // loads issued eight at a time (independent L2 reads), added in block order
      double sum = 0.0;
      for (unsigned k0 = grp; k0 < gridDim.x; k0 += 32) {
        double v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const unsigned k = k0 + 4u * u;
          v[u] = k < gridDim.x ? __ldcg(pb + k * kMom + mi) : 0.0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) sum += v[u];
      }
      part[grp][mi] = sum;
    }
    __syncthreads();
    if (threadIdx.x < kMom) {
      // threads 195..255 cover moments 0..60 of group 3; moments 61..64 of
      // group 3 were not visited: add their blocks here.
      double s3 = threadIdx.x < 256 - 3 * kMom ? part[3][threadIdx.x] : 0.0;
      if (threadIdx.x >= 256 - 3 * kMom) {
        for (unsigned k0 = 3; k0 < gridDim.x; k0 += 32) {
          double v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const unsigned k = k0 + 4u * u;
            v[u] = k < gridDim.x ? __ldcg(pb + k * kMom + threadIdx.x) : 0.0;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) s3 += v[u];
        }
      }
      mom[threadIdx.x] = ((part[0][threadIdx.x] + part[1][threadIdx.x]) + part[2][threadIdx.x]) + s3;
    }
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
  int nb = (t0 + 256 * 2 - 1) / (256 * 2);
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

// ------------------------------------------------------------------ LayerNorm
// One warp per row, two rows per 64-thread CTA (many small CTAs spread a
// ~800-row activation over every SM).  fp16 input: lane owns 8-element chunks
// (lane + 32 i); fp32 input: 4-element chunks.  The row, gamma and beta are
// all requested before any arithmetic (one memory round trip); two passes over
// registers (mean, then the centred sum of squares), fp32 throughout, fp16 out.
template <int COLS, bool F32IN>
__global__ void __launch_bounds__(64)
layernorm_kernel(const void* xin, __half* __restrict__ y, int rows, const float* __restrict__ gamma,
                 const float* __restrict__ beta, float eps, int act) {
  // xin is the previous kernel's output: plain loads after pdl_wait().
  constexpr int VEC = F32IN ? 4 : 8;
  constexpr int NCH = COLS / (32 * VEC);
  constexpr int NPL = COLS / 32;
  if (threadIdx.x == 0) pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 2 + warp;
  float g[NPL], bt[NPL];
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c0 = (lane + 32 * i) * VEC;
#pragma unroll
    for (int k = 0; k < VEC; k += 4) {
      const float4 gv = __ldg(reinterpret_cast<const float4*>(gamma + c0 + k));
      const float4 bv = __ldg(reinterpret_cast<const float4*>(beta + c0 + k));
      g[VEC * i + k] = gv.x; g[VEC * i + k + 1] = gv.y; g[VEC * i + k + 2] = gv.z; g[VEC * i + k + 3] = gv.w;
      bt[VEC * i + k] = bv.x; bt[VEC * i + k + 1] = bv.y; bt[VEC * i + k + 2] = bv.z; bt[VEC * i + k + 3] = bv.w;
    }
  }
  pdl_wait();
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
    uint32_t hv[VEC / 2];
#pragma unroll
    for (int j = 0; j < VEC; j += 2) {
      const float a0 = fmaf((v[VEC * i + j] - mean) * rstd, g[VEC * i + j], bt[VEC * i + j]);
      const float a1 = fmaf((v[VEC * i + j + 1] - mean) * rstd, g[VEC * i + j + 1], bt[VEC * i + j + 1]);
      __half2 h2 = __floats2half2_rn(apply_act(a0, act), apply_act(a1, act));
      hv[j / 2] = *reinterpret_cast<uint32_t*>(&h2);
    }
    if (VEC == 8)
      *reinterpret_cast<uint4*>(yr + c0) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    else
      *reinterpret_cast<uint2*>(yr + c0) = make_uint2(hv[0], hv[1]);
  }
}

template <int COLS>
static void ln_dispatch(const void* x, int in_f32, __half* y, int rows, const float* g, const float* b, float eps,
                        int act, cudaStream_t st) {
  const int blocks = (rows + 1) / 2;
  if (in_f32)
    launch_pdl(layernorm_kernel<COLS, true>, dim3(blocks), dim3(64), 0, st, x, y, rows, g, b, eps, act);
  else
    launch_pdl(layernorm_kernel<COLS, false>, dim3(blocks), dim3(64), 0, st, x, y, rows, g, b, eps, act);
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
