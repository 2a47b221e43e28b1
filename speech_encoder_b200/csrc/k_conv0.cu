// Conv layer 0 of the feature encoder on the tensor core: Conv1d(1 -> 512,
// kernel 10, stride 5) is a GEMM with K = 10 taps (zero-padded to the MMA's
// K = 16): A[t, j] = pcm[5 t + j], B[c, j] = w0[c, j].  A tile is 128 output
// frames of one clip x all 512 channels: two tcgen05 MMAs (M = 128, N = 256,
// K = 16) into 512 TMEM columns; the epilogue applies the norm and GELU and
// stores through TMA:
//   group layout: GroupNorm with per-channel statistics over every frame of
//     the clip (the TensorRT wav2vec2 README's "group norm over every time
//     step"), precomputed as scale/shift by the moments kernel;
//   layer layout: conv bias, then LayerNorm over the 512 channels of each
//     frame (the four warps that share a row combine their partial sums).
// Persistent: one CTA per SM walks the tiles (stride gridDim.x), so the
// weights, TMEM and barriers are set up once; warp 0 builds the next tile's
// window matrix while the epilogue of the current one runs (two A buffers),
// and issues its MMAs as soon as the epilogue has read the accumulator.
// 576 threads: warp 0 stages A and issues the MMAs, warp 1 owns TMEM, warps
// 2-17 run the epilogue (four warps per TMEM lane quarter, one per 128-channel
// slice).  The PCM is rounded to fp16 for the MMA, the same rounding every
// inter-layer activation of this path gets.
#include "ptx.cuh"
#include "w2v_internal.h"

namespace w2v {

namespace {
constexpr int kC0 = 512;
constexpr int kTaps = 10;
constexpr int kHop = 5;
constexpr int A_OFF = 0;                   // [2 buffers][2 k-chunks][128 rows][8] fp16, 2 x 4 KB
constexpr int B_OFF = 8192;                // [2 k-chunks][512 rows][8] fp16, 16 KB
constexpr int PA_OFF = B_OFF + 16384;      // float[512]: GroupNorm scale, or LayerNorm gamma
constexpr int PB_OFF = PA_OFF + 2048;      // float[512]: GroupNorm shift, or LayerNorm beta
constexpr int BIAS_OFF = PB_OFF + 2048;    // float bias[512]
constexpr int kEpiWarps = 16;              // 4 per TMEM lane quarter, 128 channels each
constexpr int kCols = 512 / (kEpiWarps / 4);
constexpr int RED_OFF = BIAS_OFF + 2048;   // float red[4 slices][128 rows]
constexpr int STG_OFF = RED_OFF + 2048;    // staging: 16 warps x 4 boxes x 2 KB
constexpr int BAR_OFF = STG_OFF + kEpiWarps * (kCols / 32) * 2048;
constexpr int SMEM = BAR_OFF + 64 + 1024;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kEpiThreads = 32 * kEpiWarps;
}  // namespace

template <int ACT, bool LN>
__global__ void __launch_bounds__(kThreads, 1)
conv0_tc_kernel(const __grid_constant__ CUtensorMap tmOut, const float* pcm, int n, int t0, int tiles_per_clip,
                int ntiles, const __half* __restrict__ wpack, const float* __restrict__ b0,
                const float* __restrict__ gamma, const float* __restrict__ beta, const float2* scale_shift,
                float eps, int* err) {
  constexpr bool layer_norm = LN;
  // pcm and scale_shift may be written by the previous kernel (programmatic
  // dependent launch): plain coherent loads after pdl_wait() only.
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* pa = reinterpret_cast<float*>(smem + PA_OFF);
  float* pb = reinterpret_cast<float*>(smem + PB_OFF);
  float* bias = reinterpret_cast<float*>(smem + BIAS_OFF);
  float* red = reinterpret_cast<float*>(smem + RED_OFF);
  uint64_t* w_full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* accf = w_full + 1;         // MMA of a tile done (one completion per tile)
  uint64_t* tmem_empty = w_full + 2;   // epilogue has read the accumulator (16 warp arrivals)
  uint64_t* a_free = w_full + 3;       // [2] MMA done reading A buffer b
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(w_full + 5);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(w_full, 1);
    mbar_init(accf, 1);
    mbar_init(tmem_empty, kEpiWarps);
    mbar_init(&a_free[0], 1);
    mbar_init(&a_free[1], 1);
    fence_mbar_init();
    pdl_launch_dependents();
    // The packed weights do not depend on the previous kernel.
    mbar_arrive_expect_tx(w_full, 16384);
    bulk_load(smem + B_OFF, wpack, 16384, w_full);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (layer_norm) {
    for (int c = threadIdx.x; c < kC0; c += kThreads) {
      pa[c] = gamma[c];
      pb[c] = beta[c];
      bias[c] = b0 ? b0[c] : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------ A builder + MMA issuer
    bool ok = true;
    int i = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
      const int b = tile / tiles_per_clip;
      const int f0 = (tile - b * tiles_per_clip) * 128;
      // A buffer i & 1 was last read by the MMA of tile i - 2.
      if (i >= 2 && ok) ok = __all_sync(0xffffffffu, mbar_wait(&a_free[i & 1], ((i >> 1) - 1) & 1));
      // row t of A holds pcm[5 (f0 + t) + j], j < 10, then zeros; 16-byte chunk
      // (row, k-chunk) at k-chunk * 2048 + row * 16 (no-swizzle core matrices)
      uint8_t* abuf = smem + A_OFF + (i & 1) * 4096;
      const float* x = pcm + static_cast<int64_t>(b) * n;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int idx = u * 32 + lane;
        const int row = idx >> 1, kc = idx & 1;
        const int t = f0 + row;
        const float* xr = x + static_cast<int64_t>(kHop) * t;
        uint32_t hv[4];
#pragma unroll
        for (int e2 = 0; e2 < 8; e2 += 2) {
          const int j = kc * 8 + e2;
          const float v0 = (t < t0 && j < kTaps) ? xr[j] : 0.f;
          const float v1 = (t < t0 && j + 1 < kTaps) ? xr[j + 1] : 0.f;
          __half2 h = __floats2half2_rn(v0, v1);
          hv[e2 / 2] = *reinterpret_cast<uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(abuf + kc * 2048 + row * 16) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        // the accumulator is free once the epilogue of tile i - 1 has read it
        if (ok && i == 0) ok = mbar_wait(w_full, 0);
        if (ok && i >= 1) ok = mbar_wait(tmem_empty, (i - 1) & 1);
        if (ok) {
          tc_fence_after();
          constexpr uint32_t idesc = idesc_f16_f32(128, 256);
          const uint32_t sa = smem_u32(abuf);
          const uint32_t sb = smem_u32(smem + B_OFF);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            umma_f16(tmem + h * 256, smem_desc(sa, 2048, 128, kSwizzleNone),
                     smem_desc(sb + h * 256 * 16, 8192, 128, kSwizzleNone), idesc, 0u);
          umma_commit(accf);
          umma_commit(&a_free[i & 1]);
        } else {
          atomicOr(err, kErrWaitMma);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lane quarter
    const int sl = (warp - 2) >> 2;      // channel slice [kCols sl, kCols sl + kCols)
    const int r = q * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16) + sl * kCols;
    uint8_t* stage = smem + STG_OFF + (warp - 2) * (kCols / 32) * 2048;
    bool ok = true;
    int cur_b = -1;
    int i = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
      const int b = tile / tiles_per_clip;
      const int f0 = (tile - b * tiles_per_clip) * 128;
      if (!layer_norm && b != cur_b) {
        // GroupNorm scale/shift of this clip (every epilogue warp walks the
        // same tiles, so all of them take this branch together)
        named_barrier_sync(2, kEpiThreads);
        for (int c = threadIdx.x - 64; c < kC0; c += kEpiThreads) {
          const float2 ss = scale_shift[b * kC0 + c];
          pa[c] = ss.x;
          pb[c] = ss.y;
        }
        named_barrier_sync(2, kEpiThreads);
        cur_b = b;
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(accf, i & 1));
      if (!ok && lane == 0) atomicOr(err, kErrWaitEpilogue);
      tc_fence_after();
      float mean = 0.f, rstd = 1.f;
      if (layer_norm) {
        // Per-frame LayerNorm statistics over all 512 channels (two passes; the
        // four slices of a row meet in shared memory).
        float s1 = 0.f;
        if (ok) {
#pragma unroll 1
          for (int c = 0; c < kCols; c += 32) {
            float v[32];
            tmem_ld32(trow + c, v);
#pragma unroll
            for (int k = 0; k < 32; ++k) s1 += v[k] + bias[sl * kCols + c + k];
          }
        }
        red[sl * 128 + r] = s1;
        named_barrier_sync(1, kEpiThreads);
        mean = ((red[r] + red[128 + r]) + (red[256 + r] + red[384 + r])) * (1.0f / kC0);
        named_barrier_sync(1, kEpiThreads);
        float s2 = 0.f;
        if (ok) {
#pragma unroll 1
          for (int c = 0; c < kCols; c += 32) {
            float v[32];
            tmem_ld32(trow + c, v);
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const float d = v[k] + bias[sl * kCols + c + k] - mean;
              s2 += d * d;
            }
          }
        }
        red[sl * 128 + r] = s2;
        named_barrier_sync(1, kEpiThreads);
        rstd = rsqrtf(((red[r] + red[128 + r]) + (red[256 + r] + red[384 + r])) * (1.0f / kC0) + eps);
        named_barrier_sync(1, kEpiThreads);  // red is rewritten by the next tile
      }
      // this warp's staging boxes: the previous tile's stores have read them
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      // 8 chunks of 16 columns; the TMEM load of chunk k + 1 is in flight
      // while chunk k is processed (two register buffers, alternating).
      auto process = [&](uint32_t(&cur)[16], int k16) {
        const int cb = k16 >> 1, hh = k16 & 1;
        const int ch = sl * kCols + cb * 32;
        uint32_t hv[8];
#pragma unroll
        for (int k = 0; k < 16; k += 4) {
          const int cc = ch + hh * 16 + k;
          const float v0 = __uint_as_float(cur[k]), v1 = __uint_as_float(cur[k + 1]);
          const float v2 = __uint_as_float(cur[k + 2]), v3 = __uint_as_float(cur[k + 3]);
          // Warp-uniform addresses: broadcast loads of 4 channels' parameters.
          const float4 A4 = *reinterpret_cast<const float4*>(pa + cc);
          const float4 B4 = *reinterpret_cast<const float4*>(pb + cc);
          float2 a01, a23;
          if (layer_norm) {
            const float4 c4 = *reinterpret_cast<const float4*>(bias + cc);
            // ((v + bias) - mean) * rstd * gamma + beta
            const float2 m2 = make_float2(-mean, -mean), r2 = make_float2(rstd, rstd);
            a01 = fmul2(fadd2(fadd2(make_float2(v0, v1), make_float2(c4.x, c4.y)), m2), r2);
            a23 = fmul2(fadd2(fadd2(make_float2(v2, v3), make_float2(c4.z, c4.w)), m2), r2);
            a01 = ffma2(a01, make_float2(A4.x, A4.y), make_float2(B4.x, B4.y));
            a23 = ffma2(a23, make_float2(A4.z, A4.w), make_float2(B4.z, B4.w));
          } else {
            a01 = ffma2(make_float2(v0, v1), make_float2(A4.x, A4.y), make_float2(B4.x, B4.y));
            a23 = ffma2(make_float2(v2, v3), make_float2(A4.z, A4.w), make_float2(B4.z, B4.w));
          }
          if (ACT == 2) {
            a01 = gelu_tanh2(a01);
            a23 = gelu_tanh2(a23);
          } else if (ACT == 1) {
            a01 = make_float2(gelu_erf(a01.x), gelu_erf(a01.y));
            a23 = make_float2(gelu_erf(a23.x), gelu_erf(a23.y));
          }
          __half2 h01 = __floats2half2_rn(a01.x, a01.y), h23 = __floats2half2_rn(a23.x, a23.y);
          hv[k / 2] = *reinterpret_cast<uint32_t*>(&h01);
          hv[k / 2 + 1] = *reinterpret_cast<uint32_t*>(&h23);
        }
        // 32 rows x 32 channels box, 64-byte rows, 64-byte swizzle: this half
        // fills the row's 16-byte chunks 2 hh and 2 hh + 1.
        uint8_t* box = stage + cb * 2048;
#pragma unroll
        for (int k = 0; k < 2; ++k)
          *reinterpret_cast<uint4*>(box + lane * 64 + (((2 * hh + k) ^ ((lane >> 1) & 3)) << 4)) =
              make_uint4(hv[4 * k], hv[4 * k + 1], hv[4 * k + 2], hv[4 * k + 3]);
        if (hh == 1) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && ok) tma_store_3d(&tmOut, box, ch, f0 + q * 32, b);
        }
      };
      uint32_t b0[16], b1[16];
      if (!(ACT == 1 && LN)) {
        if (ok) tmem_ld16_issue(trow, b0);
#pragma unroll 1
        for (int k16 = 0; k16 < kCols / 16; k16 += 2) {
          if (ok) {
            tmem_wait16(b0);
            tmem_ld16_issue(trow + (k16 + 1) * 16, b1);
          }
          process(b0, k16);
          if (ok) {
            tmem_wait16(b1);
            if (k16 + 2 < kCols / 16) tmem_ld16_issue(trow + (k16 + 2) * 16, b0);
          }
          if (k16 + 2 == kCols / 16) {
            // last accumulator read of this tile: hand TMEM to the next MMA
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tmem_empty);
          }
          process(b1, k16 + 1);
        }
      } else {
        // The erf + LayerNorm variant has no registers to spare for a second
        // buffer at this thread count: one load at a time.
#pragma unroll 1
        for (int k16 = 0; k16 < kCols / 16; ++k16) {
          if (ok) {
            tmem_ld16_issue(trow + k16 * 16, b0);
            tmem_wait16(b0);
          }
          if (k16 + 1 == kCols / 16) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tmem_empty);
          }
          process(b0, k16);
        }
      }
      if (lane == 0) bulk_commit_group();
    }
    // the staging boxes must outlive the stores' reads of them; the grid
    // boundary makes the global writes visible to the next kernel
    if (lane == 0) bulk_wait_read_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int ACT, bool LN>
static cudaError_t prepare_one() {
  return cudaFuncSetAttribute(conv0_tc_kernel<ACT, LN>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
}

cudaError_t conv0_prepare() {
  cudaError_t r = prepare_one<0, false>();
  if (r == cudaSuccess) r = prepare_one<1, false>();
  if (r == cudaSuccess) r = prepare_one<2, false>();
  if (r == cudaSuccess) r = prepare_one<0, true>();
  if (r == cudaSuccess) r = prepare_one<1, true>();
  if (r == cudaSuccess) r = prepare_one<2, true>();
  return r;
}

cudaError_t launch_conv0_tc(const float* pcm, int n, int batch, int t0, int clip_rows, const __half* wpack,
                            const float* b0, const float* gamma, const float* beta, const float2* scale_shift,
                            int layer_norm, float eps, int act, __half* out, int* err, cudaStream_t st) {
  if (t0 <= 0 || batch <= 0) return cudaSuccess;
  CUtensorMap tm;
  const uint64_t dims[3] = {static_cast<uint64_t>(kC0), static_cast<uint64_t>(t0), static_cast<uint64_t>(batch)};
  const uint64_t str[2] = {static_cast<uint64_t>(kC0) * 2, static_cast<uint64_t>(clip_rows) * kC0 * 2};
  const uint32_t box[3] = {32, 32, 1};
  cudaError_t r = make_tmap(&tm, out, 3, dims, str, box, 2, 64);
  if (r != cudaSuccess) return r;
  const int tiles_per_clip = (t0 + 127) / 128;
  const int ntiles = tiles_per_clip * batch;
  const int grid = ntiles < kNumSMs ? ntiles : kNumSMs;
  auto k = layer_norm ? (act == 2 ? conv0_tc_kernel<2, true> : (act == 1 ? conv0_tc_kernel<1, true> : conv0_tc_kernel<0, true>))
                      : (act == 2 ? conv0_tc_kernel<2, false>
                                  : (act == 1 ? conv0_tc_kernel<1, false> : conv0_tc_kernel<0, false>));
  return launch_pdl(k, dim3(grid), dim3(kThreads), SMEM, st, tm, pcm, n, t0, tiles_per_clip, ntiles, wpack, b0, gamma,
                    beta, scale_shift, eps, err);
}

}  // namespace w2v
