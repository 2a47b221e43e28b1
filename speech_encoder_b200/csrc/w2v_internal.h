// Host-side declarations shared by the kernel launchers and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace w2v {

// Launches a kernel with programmatic dependent launch enabled: it may begin
// (set-up, weight prefetch) while the previous kernel on the stream drains,
// and waits in-kernel (griddepcontrol.wait) before reading that kernel's
// outputs.  Recorded as programmatic edges when captured into a CUDA graph.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- tensor maps
// Encodes a tiled TMA descriptor for a row-major fp16 tensor with up to 3
// dimensions (dims[0] innermost).  strides_bytes[i] is the stride of dims[i+1].
// Returns cudaSuccess or an error (bad alignment, driver entry point missing).
cudaError_t make_tmap_f16(CUtensorMap* out, const void* base, int rank, const uint64_t* dims,
                          const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128);
// Same for fp16 (elem_bytes 2) or fp32 (4) with a 0/32/64/128-byte swizzle.
cudaError_t make_tmap(CUtensorMap* out, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                      const uint32_t* box, int elem_bytes, int swizzle_bytes);

// ----------------------------------------------------------------------- GEMM
// D = A * B^T over fp16 operands with fp32 accumulation on tcgen05 and a fused
// epilogue.  A is read through a 3-D tensor map {K-ish cols, rows, batch}: the
// K block starting at k is fetched from column (k % a_kwrap) of row
// (m0 + k / a_kwrap) — a_kwrap = K for an ordinary matrix, or the width of a
// pair of frames for the stride-2 conv layers (implicit GEMM).
// The kernel's own copy of the epilogue arguments.  Its size is capped: the
// GEMM kernel's by-value parameter block (5 tensor maps, GemmDims, this struct
// and 16 bytes more) measured the same speed up to 808 bytes and 30-50 %
// slower launches from 816 bytes on (direct TMA-store epilogues), so this
// struct stays at or below 128 bytes (static_assert in k_gemm.cu) and
// host-only additions go into GemmEpilogue below.
struct GemmEpiArgs {
  const float* bias = nullptr;     // [N] or null
  const void* residual = nullptr;  // [rows, ldr], fp16 or fp32 per res_f32, or null
  int res_f32 = 0;
  int ldr = 0;
  int64_t res_batch_stride = 0;    // elements between batch items
  void* out = nullptr;             // [rows, ldo], fp16 or fp32 per out_f32
  int out_f32 = 0;
  int ldo = 0;
  int64_t out_batch_stride = 0;
  int act = 0;                     // 0 none, 1 exact GELU, 2 tanh GELU
  // QKV split: when qkv_d > 0 the N = 3*qkv_d columns go to three places:
  // [0, d) -> out (Q, row-major, ldo), [d, 2d) -> out_k (K, row-major, ldo),
  // [2d, 3d) -> vt laid out [batch][head][64][t_pad] (V transposed per head).
  int qkv_d = 0;
  void* out_k = nullptr;
  void* vt = nullptr;
  int t_pad = 0;
  int n_heads = 0;
  int t_len = 0;                   // frames per clip (rows are clip-major)
  // LayerNorm folded into the GEMMs (post-norm encoder blocks).  Row
  // statistics travel as partial sums: a GEMM with ln_out set stores, for each
  // output row and each 32-column group p (ceil(N / 32) partials, whatever the
  // tile width or split form), the sum and the sum of squares of its final
  // values at ln_out[p * M + row].  A GEMM
  // reading such rows gets (ln_cfg >> 8) partials per row at ln_in and
  //  ln_mode 1 (ln_cfg & 255): A holds the un-normalised rows x and B holds
  //    W diag(gamma); the epilogue turns the accumulator into LN(x) W^T + bias
  //    as rstd * (acc - mean * ln_vec[n]) + bias[n], with ln_vec = the column
  //    sums of the scaled weight and bias = the original bias + W beta;
  //  ln_mode 2: the fp16 residual is un-normalised; the epilogue adds
  //    LN(residual) = (res - mean) * rstd * gamma[n] + beta[n], with
  //    gamma = ln_vec[n], beta = ln_vec[N + n].
  int ln_cfg = 0;
  const float* ln_vec = nullptr;
  const float2* ln_in = nullptr;
  float2* ln_out = nullptr;
  float ln_eps = 0.f;
};

struct GemmEpilogue : GemmEpiArgs {
  // Split-K scratch for GemmShape::split_l2: fp32 [splits][ws_rows][ws_ld],
  // ws_rows >= the row tiles' extent (128 * ceil(M / 128)), ws_ld >= N.  The
  // kernel reaches it through a tensor map only.
  float* part_ws = nullptr;
  int64_t ws_rows = 0;
  int64_t ws_ld = 0;
  // one arrival counter per output tile for the same form, zero before the
  // first launch (each launch leaves them zero); ticket_cap counters
  int* split_tickets = nullptr;
  int64_t ticket_cap = 0;
};

// Streaming multiprocessors of a B200: the grid of the persistent kernels.
constexpr int kNumSMs = 148;

// The kernel's copy of the problem shape (see GemmEpiArgs on its size).
struct GemmDims {
  int M = 0;        // valid rows per batch item
  int N = 0;        // valid output columns
  int K = 0;        // multiple of 64
  int a_kwrap = 0;  // see above
  int batch = 1;
  int splits = 1;   // split-K factor (batch must be 1 when > 1): the splits of
                    // one output tile form a thread-block cluster and reduce
                    // their fp32 partials through distributed shared memory,
};

struct GemmShape : GemmDims {
  bool split_l2 = false;  // or, with splits 2..4, through the L2 scratch of
                          // GemmEpilogue (TMA stores and loads of fp32 boxes,
                          // the last split to arrive finishing the tile)
  bool pair = false;      // CTA pairs on 256-row tiles (2-CTA tensor-core
                          // instructions); then tmB's box is {64, bn/2}, no split
  bool persist = false;   // persistent CTAs (one per SM) walking the output tiles
                          // with double-buffered TMEM accumulators; no split,
                          // pair or QKV split, 16-byte aligned rows
};

// Chooses the N tile width (returned) and the split-K factor (s->splits) for
// this shape.  bn_divides > 0 restricts the width to divisors of it (the fused
// QKV projection needs tiles that do not straddle Q/K/V).
// tmA: {cols, rows, batch}, box {64,128,1}; tmB: {K, N}, box {64, bn}.
int gemm_pick(GemmShape* s, int bn_divides);
// Whether the split-K-through-L2 form fits tile width bn with `splits` splits.
bool gemm_l2_split_fits(int bn, int splits);
// Whether a GEMM of this form can stage its fp16 residual tile in shared memory.
bool gemm_res_stage_fits(int bn, bool pair, int mode, int splits);
// Raise the dynamic shared-memory limits of the tcgen05 kernels (idempotent;
// called before any launch or stream capture).
cudaError_t gemm_prepare();
cudaError_t posconv_prepare();
cudaError_t attention_prepare();
cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmShape& s, int bn,
                        const GemmEpilogue& e, int* err, cudaStream_t st);

// ------------------------------------------------------------------ frontend
// Group layout: GroupNorm statistics of conv layer 0 from the moments of its
// 10-sample input windows.  Writes scale_shift[b][512] = (gamma/sigma,
// beta - mean*gamma/sigma).  partial: [batch][gn_moment_blocks(t0)][65] fp64
// scratch; ticket: [batch] counters that must be zero before the first call
// (the kernel leaves them zero).
int gn_moment_blocks(int t0);
cudaError_t launch_gn_moments(const float* pcm, int n, int batch, int t0, const float* w0, const float* gamma,
                              const float* beta, float eps, double* partial, unsigned* ticket, float2* scale_shift,
                              cudaStream_t st);
// conv0 + norm + GELU on the tensor core -> fp16 [batch][clip_rows][512]
// (rows >= t0 untouched).  wpack: fp16 taps [2][512][8] (tap j of channel c
// at [j/8][c][j%8], taps 10..15 zero).
//   group layout: per-channel scale/shift from launch_gn_moments,
//   layer layout: conv bias, per-frame LayerNorm over the 512 channels.
cudaError_t conv0_prepare();
cudaError_t launch_conv0_tc(const float* pcm, int n, int batch, int t0, int clip_rows, const __half* wpack,
                            const float* b0, const float* gamma, const float* beta, const float2* scale_shift,
                            int layer_norm, float eps, int act, __half* out, int* err, cudaStream_t st);
// Row LayerNorm over `cols` channels (512, 768 or 1024), fp16 or fp32 input,
// fp16 output, optional GELU after the affine.
cudaError_t launch_layernorm(const void* x, int in_f32, __half* y, int rows, int cols, const float* gamma,
                             const float* beta, float eps, int act, cudaStream_t st);

// ----------------------------------------------------------- positional conv
// h[t, c] (fp32) = x[t, c] + GELU(bias[c] + sum_{j, i} x[t + j - 64, g*m + i] * W[c, i, j]),
// grouped conv over 16 groups of m = d/16 channels, kernel 128.  x is read
// through tmX {d, T, batch}, box {8, 256, 1}, no swizzle.  wpack holds the
// weights pre-arranged per (group, tap) in the no-swizzle K-major core-matrix
// layout that the tensor core reads directly.
cudaError_t launch_posconv(const CUtensorMap& tmX, const __half* x, const __half* wpack, const float* bias, int T,
                           int batch, int d, int act, float* h, int* err, cudaStream_t st);

// ----------------------------------------------------------------- attention
// O = softmax(Q K^T / 8) V per (clip, head), no mask, head dim 64.
// tmQ/tmK: {d, T, batch} box {64,128,1} SW128; tmVt: {T, batch*H*64} box {64,64} SW128.
cudaError_t launch_attention(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmVt, int T,
                             int batch, int H, __half* out, int* err, cudaStream_t st);
// Clips of different lengths in one launch: clip c has len[c] frames at rows
// row0[c] (a multiple of 128) of the packed Q/K/out matrices and columns
// row0[c] of V^T; its query tiles are qt0[c] .. qt0[c+1]-1 of the grid.
// tmQ/tmK: {d, rows, 1} box {64,128,1}; tmVt: {rows, H*64} box {64,64}.
constexpr int kMaxVarlenClips = 64;
struct AttnClips {
  int n = 0;
  int row0[kMaxVarlenClips] = {};
  int len[kMaxVarlenClips] = {};
  int qt0[kMaxVarlenClips + 1] = {};
};
cudaError_t launch_attention_varlen(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmVt,
                                    const AttnClips& clips, int H, __half* out, int* err, cudaStream_t st);

// ----------------------------------------------------------------------- CTC
cudaError_t launch_argmax(const float* logits, int rows, int V, int32_t* ids, cudaStream_t st);
cudaError_t launch_ctc_collapse(const int32_t* ids, int batch, int T, int t_valid, int blank, int32_t* tokens,
                                int32_t* n_tokens, cudaStream_t st);

// Holds the stream for `ns` nanoseconds (<= 0.1 s).
cudaError_t launch_stream_gate(uint64_t ns, cudaStream_t st);

// A kernel whose bounded wait runs out on purpose (nothing ever arrives on its
// barrier); it records kErrTest in *err and returns.
cudaError_t launch_wait_timeout_probe(int* err, uint64_t limit_ns, cudaStream_t st);

}  // namespace w2v
