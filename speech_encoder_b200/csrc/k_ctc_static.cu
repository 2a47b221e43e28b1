// Greedy CTC decode that allocates nothing: the same argmax and collapse
// kernels as w2v_ctc_greedy, but the per-frame argmax ids (the only scratch
// the decode needs) live in a fixed-size array in this library's device
// memory instead of a workspace obtained with cudaMalloc.
//
// Who needs this: callers that must not allocate device memory while they
// run — for example code that queues work from a real-time audio callback
// (cudaMalloc can block on the whole device), programs whose GPU memory is
// owned by their own allocator and budgeted up front, or plugins whose host
// application forbids allocations after start-up.  They pass the logits and
// the output buffers; the library supplies the scratch.
//
// The array is a file-scope __device__ variable.  CUDA loads a library's
// device code lazily by default (CUDA_MODULE_LOADING=LAZY), so the array is
// placed on a GPU when its module is first used there: by the first call of
// this entry point on that device.  That first call may therefore allocate
// and block like any module load; make it at start-up, before any stream
// capture.  From then on the GPU holds W2V_CTC_STATIC_MAX_ROWS int32 values
// (4 MiB) until the process exits.  On the host the array's name is only a
// stand-in for the symbol, not a device address: every call looks the address
// up with cudaGetSymbolAddress, with the caller's device current (after the
// module is loaded this allocates nothing), so a device reset or a new primary
// context never leaves a stale address behind.
#include "w2v.h"
#include "w2v_internal.h"

namespace w2v {

static __device__ __align__(256) int32_t g_ctc_static_ids[W2V_CTC_STATIC_MAX_ROWS];

namespace {

// Device address of g_ctc_static_ids on the current device.
cudaError_t static_ids_address(int32_t** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_ctc_static_ids);
  if (e != cudaSuccess) return e;
  *out = static_cast<int32_t*>(p);
  return cudaSuccess;
}

}  // namespace
}  // namespace w2v

extern "C" int w2v_ctc_greedy_static(const float* logits_dev, int batch, int T, int vocab, int t_valid,
                                     int blank_id, int32_t* tokens_dev, int32_t* n_tokens_dev, void* stream) {
  if (!logits_dev || !tokens_dev || !n_tokens_dev) return W2V_EINVAL;
  if ((reinterpret_cast<uintptr_t>(logits_dev) | reinterpret_cast<uintptr_t>(tokens_dev) |
       reinterpret_cast<uintptr_t>(n_tokens_dev)) & 15u)
    return W2V_EINVAL;
  if (batch < 1 || T < 0 || vocab < 1 || t_valid < 0 || t_valid > T) return W2V_ESHAPE;
  if (blank_id < 0 || blank_id >= vocab) return W2V_EINVAL;
  if (static_cast<int64_t>(batch) * T > W2V_CTC_STATIC_MAX_ROWS) return W2V_ESHAPE;
  int32_t* ids = nullptr;
  if (w2v::static_ids_address(&ids) != cudaSuccess) return W2V_ECUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The argmax writes every id the collapse reads (frames [0, t_valid) of each
  // clip), so nothing left in the array by an earlier call is ever used.
  if (w2v::launch_argmax(logits_dev, batch * T, vocab, ids, st) != cudaSuccess) return W2V_ECUDA;
  if (w2v::launch_ctc_collapse(ids, batch, T, t_valid, blank_id, tokens_dev, n_tokens_dev, st) != cudaSuccess)
    return W2V_ECUDA;
  return W2V_OK;
}
