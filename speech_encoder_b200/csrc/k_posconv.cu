// Positional convolution of the wav2vec2 encoder as a grouped implicit GEMM on
// tcgen05.  Conv1d(d -> d, kernel 128, 16 groups, 64 zeros of padding on each
// side, last output frame dropped), bias, GELU, then the residual add
// h = x + pos(x).  The weight-norm of the checkpoint is already folded into a
// static weight (the LiteRT wav2vec2 discussion's third GPU rewrite).
//
// Per CTA: 128 output frames x one group (m = d/16 channels).  The input
// window x[t0-64, t0+192) x (m channels of the group) is loaded once into
// shared memory in the no-swizzle K-major core-matrix layout, in which rows
// sit 16 bytes apart inside each 8-channel column block.  Tap j of the conv is
// then the MMA  acc += X[t0+j-64 .. t0+j+63, :] * W_j^T  whose A descriptor
// simply starts j rows (16*j bytes) into the window: 128 taps, m/16 MMAs each,
// one resident window, no re-loads.  Rows outside [0, T) are zero-filled by
// the TMA unit, which gives the conv's zero padding for free.  Weights stream
// through a ring of per-tap [m x m] blocks pre-arranged on the host in the
// same core-matrix layout, one bulk copy per stage.
#include "ptx.cuh"
#include "w2v_internal.h"

namespace w2v {

constexpr int kPosK = 128;
constexpr int kWin = 256;  // window rows held in shared memory (>= 128 + 127)

template <int MG>
struct PosCfg {
  static constexpr int KCH = MG / 8;                   // 16-byte column blocks per row
  static constexpr int A_BYTES = KCH * kWin * 16;
  static constexpr int TAP_BYTES = MG * MG * 2;
  static constexpr int TAPS = (MG <= 32) ? 16 : (MG == 48 ? 8 : 4);
  static constexpr int STAGE = TAPS * TAP_BYTES;
  static constexpr int STAGES = 4;
  static constexpr int ITERS = kPosK / TAPS;
  static constexpr int TMEM_COLS = MG <= 32 ? 32 : 64;
  static constexpr int SMEM = A_BYTES + STAGES * STAGE + 1024 + 256;
};

template <int MG>
__global__ void __launch_bounds__(192, 1)
posconv_kernel(const __grid_constant__ CUtensorMap tmX, const __half* x, const __half* __restrict__ wpack,
               const float* __restrict__ bias, int T, int d, int act, float* __restrict__ h, int* err) {
  using C = PosCfg<MG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::STAGES * C::STAGE);
  uint64_t* empty = full + C::STAGES;
  uint64_t* a_full = empty + C::STAGES;
  uint64_t* accf = a_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * 128;
  const int g = blockIdx.y;
  const int b = blockIdx.z;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(a_full, 1);
    mbar_init(accf, 1);
    fence_mbar_init();
    pdl_launch_dependents();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmX);
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint8_t* wg = reinterpret_cast<const uint8_t*>(wpack) + static_cast<int64_t>(g) * kPosK * C::TAP_BYTES;
      // Weights first (independent of the previous kernel), then the window.
      const int pre = C::ITERS < C::STAGES ? C::ITERS : C::STAGES;
      for (int it = 0; it < pre; ++it) {
        mbar_arrive_expect_tx(&full[it], C::STAGE);
        bulk_load(sB + it * C::STAGE, wg + static_cast<int64_t>(it) * C::STAGE, C::STAGE, &full[it]);
      }
      pdl_wait();
      mbar_arrive_expect_tx(a_full, C::A_BYTES);
#pragma unroll
      for (int c = 0; c < C::KCH; ++c) tma_load_3d(sA + c * kWin * 16, &tmX, a_full, g * MG + 8 * c, t0 - 64, b);
      int issued = pre;
      bool ok = true;
      for (int it = pre; it < C::ITERS; ++it) {
        const int st = it % C::STAGES;
        if (!mbar_wait(&empty[st], ((it / C::STAGES) & 1) ^ 1)) {
          atomicOr(err, kErrWaitProducer);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[st], C::STAGE);
        bulk_load(sB + st * C::STAGE, wg + static_cast<int64_t>(it) * C::STAGE, C::STAGE, &full[st]);
        issued = it + 1;
      }
      if (!ok) {
        mbar_wait(a_full, 0);
        for (int it = (issued > C::STAGES ? issued - C::STAGES : 0); it < issued; ++it)
          mbar_wait(&full[it % C::STAGES], (it / C::STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, MG);
      bool ok = mbar_wait(a_full, 0);
      if (!ok) atomicOr(err, kErrWaitMma);
      // Descriptors built once; a tap or stage step only moves the 14-bit
      // start-address field (16-byte units; addresses stay below 256 KB).
      const uint64_t dA0 = smem_desc(smem_u32(sA), kWin * 16, 128, kSwizzleNone);
      const uint64_t dB0 = smem_desc(smem_u32(sB), MG * 16, 128, kSwizzleNone);
      for (int it = 0; ok && it < C::ITERS; ++it) {
        const int st = it % C::STAGES;
        if (!mbar_wait(&full[st], (it / C::STAGES) & 1)) {
          atomicOr(err, kErrWaitMma);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bst = dB0 + static_cast<uint64_t>(st * (C::STAGE >> 4));
#pragma unroll 4
        for (int tt = 0; tt < C::TAPS; ++tt) {
          const int j = it * C::TAPS + tt;
          const uint64_t ad = dA0 + static_cast<uint64_t>(j);                        // window row j
          const uint64_t bd = bst + static_cast<uint64_t>(tt * (C::TAP_BYTES >> 4));  // tap tt's block
#pragma unroll
          for (int kk = 0; kk < MG / 16; ++kk)
            umma_f16(tmem, ad + kk * 2 * kWin, bd + kk * 2 * MG, idesc, (j | kk) != 0 ? 1u : 0u);
        }
        umma_commit(&empty[st]);
      }
      if (ok) umma_commit(accf);
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;
    bool ok = mbar_wait(accf, 0);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) atomicOr(err, kErrWaitEpilogue);
    tc_fence_after();
    if (ok) {
      const int t = t0 + r;
      const bool row_ok = t < T;
      const int64_t rowoff = (static_cast<int64_t>(b) * T + t) * d + g * MG;
#pragma unroll 1
      for (int c = 0; c < MG; c += 16) {
        float v[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + c, v);
        if (!row_ok) continue;
        const uint4* xr = reinterpret_cast<const uint4*>(x + rowoff + c);
        uint4 u[2] = {xr[0], xr[1]};
        const __half2* hx = reinterpret_cast<const __half2*>(u);
        float out[16];
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          const float2 xf = __half22float2(hx[i / 2]);
          out[i] = xf.x + apply_act(v[i] + __ldg(bias + g * MG + c + i), act);
          out[i + 1] = xf.y + apply_act(v[i + 1] + __ldg(bias + g * MG + c + i + 1), act);
        }
        float4* hr = reinterpret_cast<float4*>(h + rowoff + c);
#pragma unroll
        for (int i = 0; i < 4; ++i) hr[i] = make_float4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int MG>
static cudaError_t prepare_mg() {
  return cudaFuncSetAttribute(posconv_kernel<MG>, cudaFuncAttributeMaxDynamicSharedMemorySize, PosCfg<MG>::SMEM);
}

cudaError_t posconv_prepare() {
  cudaError_t r;
  if ((r = prepare_mg<16>()) != cudaSuccess) return r;
  if ((r = prepare_mg<32>()) != cudaSuccess) return r;
  if ((r = prepare_mg<48>()) != cudaSuccess) return r;
  return prepare_mg<64>();
}

template <int MG>
static cudaError_t launch_mg(const CUtensorMap& tmX, const __half* x, const __half* wpack, const float* bias, int T,
                             int batch, int d, int act, float* h, int* err, cudaStream_t st) {
  using C = PosCfg<MG>;
  dim3 grid((T + 127) / 128, 16, batch);
  return launch_pdl(posconv_kernel<MG>, grid, dim3(192), C::SMEM, st, tmX, x, wpack, bias, T, d, act, h, err);
}

cudaError_t launch_posconv(const CUtensorMap& tmX, const __half* x, const __half* wpack, const float* bias, int T,
                           int batch, int d, int act, float* h, int* err, cudaStream_t st) {
  if (T <= 0 || batch <= 0) return cudaSuccess;
  switch (d / 16) {
    case 16: return launch_mg<16>(tmX, x, wpack, bias, T, batch, d, act, h, err, st);
    case 32: return launch_mg<32>(tmX, x, wpack, bias, T, batch, d, act, h, err, st);
    case 48: return launch_mg<48>(tmX, x, wpack, bias, T, batch, d, act, h, err, st);
    case 64: return launch_mg<64>(tmX, x, wpack, bias, T, batch, d, act, h, err, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace w2v
