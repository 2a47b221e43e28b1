// Per-frame argmax over the CTC head logits and greedy CTC collapse (merge
// repeated ids, then drop blank), the decoding the TensorRT wav2vec2 README's
// "CTC ids" exact-match check refers to.
#include "ptx.cuh"
#include "w2v_internal.h"

namespace w2v {

// One warp per frame.  Ties resolve to the lowest index; the comparison is an
// fp32 compare on the stored logits, the same values the caller reads back.
__global__ void __launch_bounds__(256)
argmax_kernel(const float* logits, int rows, int V, int32_t* __restrict__ ids) {
  // logits come from the previous kernel: plain loads after pdl_wait().
  if (threadIdx.x == 0) pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  const float* z = logits + static_cast<int64_t>(row) * V;
  float best = -INFINITY;
  int bi = 0x7fffffff;
  for (int v = lane; v < V; v += 32) {
    const float x = z[v];
    if (x > best) {  // strictly greater: keeps the first (lowest) index per lane
      best = x;
      bi = v;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ob > best || (ob == best && oi < bi)) {
      best = ob;
      bi = oi;
    }
  }
  if (lane == 0) ids[row] = (bi == 0x7fffffff) ? 0 : bi;
}

cudaError_t launch_argmax(const float* logits, int rows, int V, int32_t* ids, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  return launch_pdl(argmax_kernel, dim3((rows + 7) / 8), dim3(256), 0, st, logits, rows, V, ids);
}

// One CTA of 1024 threads per clip; frames in chunks of 1024 with a block-wide
// exclusive scan of the keep flags (keep a_t iff a_t != blank and
// (t == 0 or a_t != a_{t-1})).
__global__ void __launch_bounds__(1024)
ctc_collapse_kernel(const int32_t* ids, int T, int t_valid, int blank, int32_t* __restrict__ tokens,
                    int32_t* __restrict__ n_tokens) {
  __shared__ int warp_sums[32];
  __shared__ int total_s;
  if (threadIdx.x == 0) pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x;
  const int32_t* a = ids + static_cast<int64_t>(b) * T;
  int32_t* out = tokens + static_cast<int64_t>(b) * t_valid;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int count = 0;
  for (int base = 0; base < t_valid; base += blockDim.x) {
    const int t = base + threadIdx.x;
    int keep = 0, v = 0;
    if (t < t_valid) {
      v = a[t];
      keep = (v != blank) && (t == 0 || v != a[t - 1]);
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    const int in_warp = __popc(bal & ((1u << lane) - 1u));
    if (lane == 0) warp_sums[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x >> 5;
      int s = lane < nw ? warp_sums[lane] : 0;
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane < nw) warp_sums[lane] = incl - s;  // exclusive
      if (lane == 31) total_s = incl;
    }
    __syncthreads();
    if (keep) out[count + warp_sums[warp] + in_warp] = v;
    count += total_s;
    __syncthreads();
  }
  if (threadIdx.x == 0) n_tokens[b] = count;
}

cudaError_t launch_ctc_collapse(const int32_t* ids, int batch, int T, int t_valid, int blank, int32_t* tokens,
                                int32_t* n_tokens, cudaStream_t st) {
  if (batch <= 0) return cudaSuccess;
  return launch_pdl(ctc_collapse_kernel, dim3(batch), dim3(1024), 0, st, ids, T, t_valid, blank, tokens, n_tokens);
}

// -------------------------------------------------------- bounded-wait probe
__global__ void wait_timeout_probe_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing arrives on this barrier: the wait must give up and report.
    if (!mbar_wait(&bar, 0, limit_ns)) atomicOr(err, kErrTest);
  }
}

// Holds the stream for `ns` nanoseconds (one thread sleeping in 1 us steps):
// lets a host queue many launches before the device starts on them, so that
// event timings between them measure device time only.
__global__ void stream_gate_kernel(uint64_t ns) {
  const uint64_t t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < ns) __nanosleep(1000);
}

cudaError_t launch_stream_gate(uint64_t ns, cudaStream_t st) {
  if (ns > 100000000ull) ns = 100000000ull;  // at most 0.1 s
  stream_gate_kernel<<<1, 1, 0, st>>>(ns);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_probe(int* err, uint64_t limit_ns, cudaStream_t st) {
  wait_timeout_probe_kernel<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace w2v
