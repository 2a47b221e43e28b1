/*
 * w2v_ops.h — single-kernel entry points of the same library, for kernel-level
 * parity tests on shapes the whole model does not reach (odd M, N tails,
 * varying K) and for the bounded-wait error path.  Same conventions as w2v.h:
 * plain device pointers owned by the caller, cudaStream_t as void*, int status
 * return, asynchronous on the stream.  `err_dev` is a caller-owned device int
 * that a kernel ORs a nonzero code into when one of its bounded waits gives up.
 */
#ifndef W2V_OPS_H
#define W2V_OPS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* out[M][N] = act(A[M][K] * B[N][K]^T + bias) + residual  on the tcgen05 GEMM.
 * A, B: fp16 row-major (B in the PyTorch Linear layout [out, in]); K a multiple
 * of 64; bias fp32 [N] or NULL; residual [M][N] fp16 (res_f32 = 0) or fp32
 * (res_f32 = 1) or NULL; out [M][N] fp16 or fp32 (out_f32); act 0 none,
 * 1 exact GELU, 2 tanh GELU.  This is the contraction of every projection in
 * the encoder blocks (README "Recipe" table: q/k/v/out projections,
 * intermediate_dense, output_dense) and of the CTC head.  bn = 0 picks the
 * tile width and split-K factor; otherwise bn (32/64/128/192/256) and splits
 * are forced: splits 1..8 (<= K/64) divides the K blocks among a cluster of
 * `splits` CTAs whose partial sums are reduced in distributed shared memory;
 * splits -2, -3 or -4 (bn >= 64, as far as the last arrival's staging fits:
 * bn 64 up to 4 splits, 128 up to 3, 192 up to 2) reduces the splits through
 * an fp32 scratch in L2 without a cluster: each split TMA-stores its partial,
 * takes a ticket, and the last to arrive loads the others and finishes the
 * tile, adding the partials in split order (the call allocates and frees
 * the scratch on the stream); splits 0 (bn >= 64) runs CTA pairs: clusters of
 * two CTAs on 256-row tiles with the 2-CTA tensor-core instructions, each CTA
 * loading its 128 rows of A and half of the tile's B columns (needs a
 * 16-byte-aligned output row pitch: the direct TMA-store epilogue); splits 9
 * (bn >= 64) runs the persistent form: one CTA per SM walking the output
 * tiles, two TMEM accumulators so that each tile's epilogue overlaps the next
 * tile's mainloop (needs 16-byte-aligned output and residual row pitches).
 * With splits 2..8 and bn / splits a multiple of 64 each cluster CTA
 * finishes a group of the tile's columns, otherwise a band of its rows.
 * Invalid combinations return W2V_EINVAL. */
int w2v_op_gemm(const void* A, const void* B, int M, int N, int K, const float* bias, const void* residual,
                int res_f32, void* out, int out_f32, int act, int bn, int splits, int* err_dev, void* stream);

/* O = softmax(Q K^T / 8) V per (clip, head) with no mask (plain SDPA, LiteRT
 * discussion fourth rewrite), head dim 64.  q, k: fp16 [batch][T][H*64];
 * vt: fp16 [batch][H][64][t_pad] (V transposed per head, t_pad >= T, a multiple
 * of 8); out: fp16 [batch][T][H*64]. */
int w2v_op_attention(const void* q, const void* k, const void* vt, void* out, int batch, int T, int H, int t_pad,
                     int* err_dev, void* stream);

/* y = act(LN(x) * gamma + beta) per row over `cols` (256, 512, 768 or 1024)
 * channels, biased variance, fp32 statistics.  x fp16 (in_f32 = 0) or fp32;
 * y fp16. */
int w2v_op_layernorm(const void* x, int in_f32, void* y, int rows, int cols, const float* gamma, const float* beta,
                     float eps, int act, void* stream);

/* Launches a kernel whose mbarrier wait can never complete; the bounded wait
 * gives up after limit_ns and ORs a nonzero code into *err_dev.  Used to test
 * that the timeout path reports instead of hanging. */
int w2v_op_wait_probe(int* err_dev, uint64_t limit_ns, void* stream);

/* Element-wise evaluation of the library's device math helpers, so that each
 * hand-written approximation can be checked against its stated error bound on
 * its own (inside the model they only show through the logits).  x_dev, y_dev:
 * float [n] on the device.  fn:
 *   0  y = 2^(c x + b) through fp16x2 rounding of the argument and the fp16x2
 *      exponent instruction (the softmax's exponent-unit path);
 *   1  the same through the cubic on the FMA/ALU pipes (the softmax's
 *      polynomial path; argument clamped to [-15, 8], results below 2^-15
 *      flush to zero);
 *   2  tanh-GELU of a pair with the fp16x2 exponent (conv/FFN epilogues);
 *   3  tanh-GELU in fp32 with the hardware tanh (the GEMM epilogues);
 *   4  exact GELU (erff);
 *   5  CUDA's exp2f(c x + b), the comparison point for 0 and 1.
 * Forms 0-2 take elements 2i and 2i+1 as one pair: n must be even.  The
 * softmax is the LiteRT discussion's plain SDPA and the tanh-GELU its first GPU
 * rewrite.  Errors: W2V_EINVAL (null pointer, unknown fn), W2V_ESHAPE (n < 0,
 * or odd for a pair form), W2V_ECUDA (launch failure). */
int w2v_op_pointwise(int fn, const float* x_dev, int n, float c, float b, float* y_dev, void* stream);

/* Host only: the weights of LayerNorm(x) -> Linear(W, bias) folded so that
 * the GEMM runs on the un-normalised x (the post-norm LayerNorm fold of
 * w2v_create).  W: float [N][K] (PyTorch Linear layout), bias: float [N] or
 * NULL, gamma / beta: float [K].  Outputs (caller-owned host arrays):
 * w_fp16 [N][K] = fp16 bits of W[n][k] * gamma[k] (product in float32, rounded
 * to nearest even); bias_out [N] = bias[n] + sum_k W[n][k] beta[k] and
 * colsum_out [N] = sum_k fp16 value of w_fp16[n][k], both accumulated in
 * float64.  Then LN(x) W^T + bias = rstd (x W''^T - mean * colsum) + bias_out
 * for every row x with mean and rstd = 1 / sqrt(var + eps), up to the fp16
 * rounding of W''.  Errors: W2V_EINVAL (null pointer), W2V_ESHAPE (N or K < 1). */
int w2v_fold_layernorm_linear(const float* W, int N, int K, const float* bias, const float* gamma, const float* beta,
                              uint16_t* w_fp16, float* bias_out, float* colsum_out);

#ifdef __cplusplus
}
#endif

#endif /* W2V_OPS_H */
