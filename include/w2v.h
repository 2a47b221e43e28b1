/*
 * w2v.h — C ABI of the wav2vec2-style CTC forward pass on NVIDIA B200 (sm_100a).
 *
 * The library computes, on one GPU, raw 16 kHz PCM -> conv feature encoder ->
 * feature projection -> grouped positional conv -> N transformer blocks ->
 * CTC head logits, and the greedy CTC token sequence from those logits.
 *
 * Passages that define the operations (pages on the subject):
 *  - TensorRT-Model-Connect wav2vec2 README, section "Wav2Vec2 CTC layouts":
 *    group-normalised or per-frame layer-normalised conv feature encoders, with
 *    or without conv bias; post-norm or stable pre-norm blocks; the encoder-level
 *    normalisation after the blocks for stable checkpoints; width 1024, 24
 *    blocks, 2341-token CTC head for the large layout; true-length PCM input
 *    with no resampling and no padded-batch attention mask.
 *  - Same README, section "FP8 quantization study": fp16 convolutions,
 *    projections and attention with every normalisation in fp32; the first
 *    feature-encoder norm is a group norm over every time step of the clip;
 *    "CTC ids" as the exact-match output.
 *  - LiteRT wav2vec2 discussion, "Rewrites for the GPU": tanh-GELU as the
 *    replacement of exact GELU; the positional conv's weight-norm folded into a
 *    static weight; attention as plain SDPA with no mask; short clips zero-padded
 *    to a fixed window and decoded over their valid frames.
 *
 * Conventions for every entry point:
 *  - Return value: W2V_OK (0) or one of the W2V_E* codes below.  On error a
 *    message is kept in the model (w2v_last_error).  No partial-output
 *    guarantee on error.
 *  - Device pointers are plain CUDA device addresses owned by the caller (for
 *    example torch tensors' data_ptr()).  They must stay valid until the work
 *    queued on `stream` has finished.  Float/int32 buffers must be 16-byte
 *    aligned.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *    stream.  Calls are asynchronous: they queue kernels and return; nothing
 *    in w2v_forward or w2v_ctc_greedy synchronises with the host.
 *  - Errors found by the device (a bounded wait inside a kernel that gave up)
 *    are latched in a device word and reported by w2v_sync.
 *  - A model handle may be used from one host thread at a time.
 */
#ifndef W2V_H
#define W2V_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct w2v_model w2v_model; /* opaque: owns device weights and workspace */

enum {
  W2V_OK = 0,
  W2V_EINVAL = 1,   /* bad argument: null pointer, bad config value, misaligned pointer */
  W2V_ESHAPE = 2,   /* size out of range: n_samples < 400, n_samples > max_samples, batch > max_batch, ... */
  W2V_ENOMEM = 3,   /* device allocation failed */
  W2V_ECUDA = 4,    /* a CUDA runtime/driver call or kernel launch failed */
  W2V_EDEVICE = 5,  /* no usable sm_100 device */
  W2V_ETIMEOUT = 6  /* a kernel's bounded wait gave up (reported by w2v_sync) */
};

/* Model configuration (the checkpoint config fields the LiteRT discussion says
 * are read from the config, plus workspace sizing). */
typedef struct {
  int d_model;           /* 768 (base) | 1024 (large); multiple of 256, <= 1024 */
  int n_layers;          /* 12 | 24; >= 0 */
  int n_heads;           /* 12 | 16; d_model / n_heads must be 64 */
  int d_ffn;             /* 3072 | 4096; multiple of 64 */
  int vocab;             /* CTC head width: 32 | 2341 */
  int blank_id;          /* CTC blank token id, 0 */
  int conv_norm;         /* 0 = group (GroupNorm(512,512) on conv layer 0), 1 = layer (per-frame LN on every conv layer) */
  int conv_bias;         /* 0/1: bias on all 7 conv layers */
  int stable_layer_norm; /* 0 = post-norm blocks, encoder LN before them; 1 = pre-norm blocks, encoder LN after them */
  int gelu_tanh;         /* 0 = exact (erf) GELU, 1 = tanh-GELU, for every GELU of the model */
  int max_samples;       /* largest n_samples per clip a forward call may pass (workspace sizing), >= 400 */
  int max_batch;         /* largest batch a forward call may pass (workspace sizing), >= 1 */
  float ln_eps;          /* epsilon of every LayerNorm / GroupNorm, 1e-5 */
  int use_cuda_graph;    /* 1: record each (n_samples, batch, pcm, logits) launch sequence once as a CUDA graph and replay it */
} w2v_config;

/* Frames produced by the 7-layer conv encoder for a clip of n_samples:
 * floor((n - 400) / 320) + 1 for n >= 400, else 0 (receptive field 400, hop 320). */
int w2v_num_frames(int n_samples);

/* Weight blob layout.  The blob is float32, tensors concatenated in manifest
 * order, PyTorch layouts: Conv1d weight [C_out, C_in/groups, k], Linear weight
 * [out, in].  The positional-conv weight is the folded static weight g*v/||v||.
 * Names: conv{i}.weight, conv{i}.bias (conv_bias), conv{i}.norm.{weight,bias}
 * (i = 0 for group, every i for layer), fp.norm.*, fp.proj.*, pos_conv.*,
 * enc.norm.*, layers.{l}.attn.{q,k,v,out}.{weight,bias},
 * layers.{l}.attn_norm.*, layers.{l}.ffn.{in,out}.{weight,bias},
 * layers.{l}.ffn_norm.*, lm_head.{weight,bias}. */
size_t w2v_weight_count(const w2v_config* cfg); /* total floats; 0 if cfg is invalid */
int w2v_weight_num_entries(const w2v_config* cfg);
/* Entry `index` of the manifest: name (NUL-terminated, truncated to name_len),
 * ndim (1..3), shape, and float offset into the blob. */
int w2v_weight_entry(const w2v_config* cfg, int index, char* name, size_t name_len, int* ndim, int64_t shape[3],
                     size_t* offset);

/* Raw PCM to forward-pass windows (the fixed-window form of the pages: a clip
 * zero-padded to the window and decoded over its valid frames).  pcm_dev:
 * float32 [n_samples] on the device, one clip at the model's sample rate.
 * It is cut into w2v_num_windows(n_samples, window) = ceil(n_samples / window)
 * consecutive windows; window w holds samples [w*window, w*window + valid_w),
 * valid_w = min(window, n_samples - w*window), normalised over those valid
 * samples to (x - mean) / sqrt(var + 1e-7) (biased variance), then zeros up
 * to `window`.  out_dev: float32 [num_windows][window] on the device, owned by
 * the caller, ready for w2v_forward(batch = num_windows, n_samples = window);
 * decode window w over w2v_num_frames(valid_w) frames.  Asynchronous on
 * `stream`.  Errors: W2V_EINVAL (null pointer), W2V_ESHAPE (n_samples or
 * window < 1), W2V_ECUDA (launch failure). */
int w2v_num_windows(int n_samples, int window);
int w2v_window_pcm(const float* pcm_dev, int n_samples, int window, float* out_dev, void* stream);

/* Packs a single-file safetensors checkpoint into the float32 weight blob
 * (blob: host float[n_floats], n_floats == w2v_weight_count(cfg); owned by the
 * caller).  Host only, no device work.  Format: 8-byte little-endian header
 * length, JSON header {name: {dtype, shape, data_offsets}}, raw data; dtypes
 * F32, F16, BF16, F64 (converted to float32).  Each manifest entry is looked
 * up under its own name, then under the checkpoint module path, with or
 * without a "wav2vec2." prefix:
 *   conv{i}.weight/.bias    feature_extractor.conv_layers.{i}.conv.weight/.bias
 *   conv{i}.norm.*          feature_extractor.conv_layers.{i}.layer_norm.*
 *   fp.norm.* / fp.proj.*   feature_projection.layer_norm.* / .projection.*
 *   pos_conv.*              encoder.pos_conv_embed.conv.*
 *   enc.norm.*              encoder.layer_norm.*
 *   layers.{l}.attn.{q,k,v,out}.*  encoder.layers.{l}.attention.{q,k,v,out}_proj.*
 *   layers.{l}.attn_norm.*  encoder.layers.{l}.layer_norm.*
 *   layers.{l}.ffn.in.* / ffn.out.*  encoder.layers.{l}.feed_forward.
 *                           intermediate_dense.* / output_dense.*
 *   layers.{l}.ffn_norm.*   encoder.layers.{l}.final_layer_norm.*
 *   lm_head.*               lm_head.*
 * The positional conv weight may be stored weight-normalised, as weight_g /
 * weight_v or parametrizations.weight.original0 / original1 (g, v): it is
 * folded to g * v / ||v||, the norm (float64) taken over the axes where g has
 * extent 1 (the pages' "pos_conv weight-norm folded into a static weight").
 * Errors: W2V_EINVAL (unreadable or malformed file, missing tensor,
 * unsupported dtype, bad config), W2V_ESHAPE (a tensor's shape differs from
 * the manifest, or n_floats is wrong); err (err_len bytes, may be NULL)
 * receives a message naming the tensor. */
int w2v_pack_safetensors(const char* path, const w2v_config* cfg, float* blob, size_t n_floats, char* err,
                         size_t err_len);
/* w2v_pack_safetensors then w2v_create; *out is NULL on error. */
int w2v_create_from_safetensors(const char* path, const w2v_config* cfg, w2v_model** out, char* err,
                                size_t err_len);

/* Creates a model on the current CUDA device: validates cfg, converts the host
 * float32 blob (n_floats == w2v_weight_count(cfg)) to the device layouts (fp16
 * matrices, repacked conv and positional-conv weights, fp32 vectors) and
 * allocates the workspace for max_batch clips of max_samples.  The host blob is
 * not retained.  *out receives the handle (NULL on error). */
int w2v_create(const w2v_config* cfg, const float* host_weights, size_t n_floats, w2v_model** out);

/* Forward pass of `batch` clips of n_samples each, packed contiguously in
 * pcm_dev (float32 [batch][n_samples], already normalised).  Writes
 * logits_dev (float32 [batch][T][vocab], T = w2v_num_frames(n_samples)).
 * The first call for a given (n_samples, batch) builds that shape's launch
 * plan: it times the tile and split-K candidates of every GEMM on the device,
 * then re-chooses the per-layer GEMMs by timing the whole forward with each
 * candidate (a few hundred milliseconds, synchronous; W2V_AUTOTUNE=0 in the
 * environment uses a cost model instead, W2V_TUNE_LOG=1 prints the choices),
 * so make that first call outside any stream capture.  With W2V_PLAN_FILE set
 * to a path, a plan tuned for this model shape, n_samples and batch is
 * appended to that text file, and a later process that finds its line there
 * launches exactly those GEMM configurations without timing anything (the
 * same kernels, hence bit-identical logits, across processes); a line whose
 * choices do not fit the shapes makes the call fail with W2V_EINVAL.
 * Post-norm models (stable_layer_norm = 0) with encoder layers run the two
 * LayerNorms of every block inside the neighbouring GEMMs (gamma folded into
 * the next weights at w2v_create, row statistics as partial sums written by
 * the GEMM that produces the rows); W2V_LN_FOLD=0 in the environment at
 * w2v_create keeps them as separate kernels.
 * Errors: W2V_ESHAPE if n_samples < 400 or > max_samples or batch outside
 * [1, max_batch]; W2V_EINVAL for null/misaligned pointers. */
int w2v_forward(w2v_model* m, const float* pcm_dev, int n_samples, int batch, float* logits_dev, void* stream);

/* Greedy CTC decode of logits (float32 [batch][T][vocab]) over frames
 * [0, t_valid): per-frame argmax (lowest index on ties), merge repeats, drop
 * blank_id.  tokens_dev: int32 [batch][t_valid], clip b's tokens first;
 * n_tokens_dev: int32 [batch].  0 <= t_valid <= T <= w2v_num_frames(max_samples). */
int w2v_ctc_greedy(w2v_model* m, const float* logits_dev, int batch, int T, int t_valid, int32_t* tokens_dev,
                   int32_t* n_tokens_dev, void* stream);

/* Varlen batched forward: `batch` clips of different lengths, each at its
 * own true length (no padding, no attention mask across clips), in one
 * launch set.  TensorRT-Model-Connect wav2vec2 README, "Wav2Vec2 CTC layouts"
 * (true-length PCM input, no padded-batch attention mask) and "FP8
 * quantization study -> When to revisit" (batches of clips give the GEMMs a
 * larger share of the time).
 *  - pcm_dev: float32, the clips packed back to back: clip c's n_samples[c]
 *    samples (already normalised) start at sample offset
 *    n_samples[0] + ... + n_samples[c-1].  n_samples: HOST int array [batch],
 *    each in [400, max_samples].  1 <= batch <= min(max_batch, 64).
 *  - logits_dev: float32 [T_0 + ... + T_{batch-1}][vocab], T_c =
 *    w2v_num_frames(n_samples[c]); clip c's rows start at T_0 + ... + T_{c-1}.
 *  - Each clip's conv feature encoder and positional conv run per clip; the
 *    projection, encoder GEMMs and CTC head run once over all clips' frames
 *    (packed on 128-row boundaries inside the model's workspace); attention
 *    runs in one launch in which every query tile attends to its own clip's
 *    keys only.  Results equal w2v_forward of each clip alone up to the GEMMs'
 *    summation order.
 *  - The first call whose packed frame count falls in a new bucket of 512
 *    rows times the encoder GEMM tile candidates once (synchronous; make it
 *    outside any stream capture); conv tiles come from a cost model, so a new
 *    clip length never times anything.  Not recorded as a CUDA graph.
 * Errors: W2V_EINVAL (null or misaligned pointer), W2V_ESHAPE (batch or a
 * length out of range). */
int w2v_forward_varlen(w2v_model* m, const float* pcm_dev, const int* n_samples, int batch, float* logits_dev,
                       void* stream);

/* Greedy CTC decode of packed clips of different lengths (the output of
 * w2v_forward_varlen): logits_dev float32 [frames[0] + ... ][vocab], frames:
 * HOST int array [batch] (frames decoded per clip, all of them).  tokens_dev:
 * int32 [frames[0] + ...], clip c's tokens from offset frames[0] + ... +
 * frames[c-1]; n_tokens_dev: int32 [batch].  Same decoding as
 * w2v_ctc_greedy. */
int w2v_ctc_greedy_varlen(w2v_model* m, const float* logits_dev, const int* frames, int batch, int32_t* tokens_dev,
                          int32_t* n_tokens_dev, void* stream);

/* Greedy CTC decode that allocates no memory and needs no model handle.  The
 * pages have no counterpart of this entry point: it exists for callers that
 * cannot allocate device memory when they decode — code driven from a
 * real-time audio callback (cudaMalloc may block on the whole device), programs
 * whose GPU memory belongs to their own allocator, or plugins whose host
 * forbids allocations after start-up.
 *
 * Same result as w2v_ctc_greedy: logits_dev float32 [batch][T][vocab], frames
 * [0, t_valid) of each clip, argmax with the lowest index on ties, repeats
 * merged, blank_id dropped; tokens_dev int32 [batch][t_valid] (clip b's
 * tokens first), n_tokens_dev int32 [batch].  The caller owns logits and
 * outputs; the per-frame argmax scratch is a fixed array of
 * W2V_CTC_STATIC_MAX_ROWS int32 (4 MiB) in the library's device memory.
 *  - batch * T must not exceed W2V_CTC_STATIC_MAX_ROWS (1048576 frames, e.g.
 *    16 clips of 30 s): larger requests return W2V_ESHAPE and launch nothing.
 *  - CUDA loads device code lazily by default, so the array is placed on a
 *    GPU by the first call of this entry point on that device: that first
 *    call may allocate device memory and block like any module load.  Make
 *    it at start-up (a call with t_valid = 0 is enough), before any stream
 *    capture; the GPU then holds the 4 MiB until the process exits.  Every
 *    call looks the array's address up for the current device, which
 *    allocates nothing once the array is loaded.
 *  - All calls share the one array, so calls whose work overlaps on the GPU
 *    (on different streams, or from different threads) race and may return
 *    wrong tokens; serialise them.  Nothing in the array needs clearing: each
 *    call writes every entry it reads.
 *  - W2V_EINVAL for null or misaligned (not 16-byte) pointers or a bad
 *    blank_id; W2V_ECUDA if the lookup or a launch fails. */
#define W2V_CTC_STATIC_MAX_ROWS (1 << 20)
int w2v_ctc_greedy_static(const float* logits_dev, int batch, int T, int vocab, int t_valid, int blank_id,
                          int32_t* tokens_dev, int32_t* n_tokens_dev, void* stream);

/* Waits for `stream`, then reports device-side errors latched since the last
 * call (W2V_ETIMEOUT) or a CUDA error; clears the latch. */
int w2v_sync(w2v_model* m, void* stream);

/* Copies an internal activation left by the last forward into dst_dev (up to
 * dst_bytes; *bytes receives the size).  which: 0 = conv encoder output fp16
 * [rows][512], 1 = projection output fp16 [rows][d], 2 = residual stream fp32
 * [rows][d] (posconv output when n_layers == 0), 3 = encoder output fed to the
 * CTC head, fp16 [rows][d].  rows = batch * T.  Debug / test aid. */
int w2v_debug_read(w2v_model* m, int which, void* dst_dev, size_t dst_bytes, size_t* bytes, void* stream);

/* End to end from host memory: copies pcm_host (float32 [batch][n_samples],
 * ideally pinned) to the device, runs w2v_forward and w2v_ctc_greedy over
 * frames [0, t_valid), copies the tokens (int32 [batch][t_valid]) and counts
 * (int32 [batch]) back to host memory, and waits for `stream`.  Device
 * staging buffers are allocated on the first call (so make that first call
 * outside any stream capture).  Returns like w2v_sync. */
int w2v_transcribe(w2v_model* m, const float* pcm_host, int n_samples, int batch, int t_valid, int32_t* tokens_host,
                   int32_t* n_tokens_host, void* stream);

/* Number of kernel launches of the last w2v_forward / w2v_profile_forward. */
int w2v_last_launch_count(w2v_model* m);

/* Kernel classes reported by the profiler. */
enum {
  W2V_K_GN_MOMENTS = 0, W2V_K_CONV0, W2V_K_CONV_GEMM, W2V_K_CONV_LN, W2V_K_FP_LN, W2V_K_PROJ_GEMM, W2V_K_POSCONV,
  W2V_K_ENC_LN, W2V_K_QKV_GEMM, W2V_K_ATTENTION, W2V_K_OUT_GEMM, W2V_K_FFN1_GEMM, W2V_K_FFN2_GEMM, W2V_K_LM_HEAD,
  W2V_K_ARGMAX, W2V_K_CTC_COLLAPSE, W2V_K_NUM_CLASSES
};

typedef struct {
  int klass;     /* W2V_K_* */
  float ms;      /* device time between CUDA events recorded just before and after the launch */
  double flops;  /* algorithmic floating-point operations of the launch (2 per multiply-add) */
  double bytes;  /* algorithmic bytes: each input read once, each output written once */
} w2v_kernel_time;

const char* w2v_kernel_class_name(int klass);

/* Runs one forward (direct launches, no graph) plus the argmax/collapse over
 * all frames, with a CUDA event pair around every kernel launch, waits for the
 * stream and fills out[0 .. *n_out) in launch order.  The launches are queued
 * behind a 20 ms device-side gate, so the events measure device time and not
 * the host's launch rate.  Used for per-kernel timing and roofline reporting. */
int w2v_profile_forward(w2v_model* m, const float* pcm_dev, int n_samples, int batch, float* logits_dev, void* stream,
                        w2v_kernel_time* out, int max_out, int* n_out);

/* Per-launch device time of one kernel class: records `reps` passes of only
 * that class's launches of a forward of this shape (inputs as the buffers
 * hold them) as one CUDA graph, replays it once to warm up, times one replay
 * with CUDA events on `stream` and divides by the number of launches.  Also
 * returns the launches per forward and the algorithmic FLOPs and bytes per
 * launch.  Synchronises the stream. */
int w2v_time_class(w2v_model* m, const float* pcm_dev, int n_samples, int batch, float* logits_dev, int klass,
                   int reps, float* us_per_launch, int* launches, double* flops_per_launch, double* bytes_per_launch,
                   void* stream);

/* Copies the last error message into buf (NUL-terminated). */
int w2v_last_error(w2v_model* m, char* buf, size_t len);

/* Frees the model's device memory and graphs. */
void w2v_destroy(w2v_model* m);

#ifdef __cplusplus
}
#endif

#endif /* W2V_H */
