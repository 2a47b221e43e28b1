// Multi-head self-attention with no mask (plain SDPA over every frame of the
// window, as the LiteRT wav2vec2 discussion's fourth GPU rewrite leaves it),
// head dim 64, scale 1/8, fused flash-style on tcgen05.
//
// One CTA per (128-query tile, head, clip), 576 threads:
//   warp 0      TMA: the Q tile once, then K and V^T tiles of 128 keys into a
//               2-deep ring
//   warp 1      TMEM owner; one thread issues S_j = Q K_j^T (M=128, N=128,
//               K=64) into one of two TMEM score buffers and, once P_j is in
//               shared memory, O_j = P_j V_j (M=128, N=64, K=128).  S_{j+1} is
//               issued before waiting for P_j, so the next scores are computed
//               while the softmax of the current tile runs.
//   warps 2-17  softmax: four warps per TMEM lane quarter, each owning 32 of
//               the 128 key columns (and 16 of the 64 output columns) of its
//               32 query rows.  Row maxima and sums are combined through shared
//               memory with a 128-thread named barrier per quarter.  fp32 online
//               softmax with exp2 (1/8 scale folded in), P rounded to fp16
//               into the 128-byte-swizzled K-major layout the MMA reads, O
//               accumulated in registers with the running rescale.
// V arrives transposed ([clip][head][64][T], written by the QKV projection's
// epilogue) so both MMAs read K-major operands.  Keys past T are zero-filled by
// TMA and masked before the exponent.
#include "ptx.cuh"
#include "w2v_internal.h"

namespace w2v {

struct AttnSmem {
  static constexpr int Q = 0;
  static constexpr int K0 = 16384;
  static constexpr int V0 = K0 + 2 * 16384;
  static constexpr int P = V0 + 2 * 16384;
  static constexpr int RED = P + 32768;       // float red_max[2][4][128], red_sum[4][128]
  static constexpr int BAR = RED + 6144;
  static constexpr int TOTAL = BAR + 256 + 1024;
};

constexpr int kSoftWarps = 16;
constexpr int kAttnThreads = 64 + 32 * kSoftWarps;
constexpr int kSubs = kSoftWarps / 4;    // warps per TMEM lane quarter
constexpr int kSCols = 128 / kSubs;      // score columns per warp
constexpr int kOCols = 64 / kSubs;       // output columns per warp

__device__ __forceinline__ void quarter_barrier(int q) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "r"(32 * kSubs) : "memory");
}

__global__ void __launch_bounds__(kAttnThreads, 1)
attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmVt, int T, int H, __half* __restrict__ out, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* red_max = reinterpret_cast<float*>(smem + AttnSmem::RED);  // [slot][sub][row]
  float* red_sum = red_max + 2 * kSubs * 128;                       // [sub][row]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* p_full = bars + 7;
  uint64_t* o_full = bars + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nkv = (T + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(&kv_full[0], 1);
    mbar_init(&kv_full[1], 1);
    mbar_init(&kv_empty[0], 1);
    mbar_init(&kv_empty[1], 1);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, 32 * kSoftWarps);
    mbar_init(o_full, 1);
    fence_mbar_init();
    pdl_launch_dependents();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmVt);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem + 256;

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();
      mbar_arrive_expect_tx(q_full, 16384);
      tma_load_3d(smem + AttnSmem::Q, &tmQ, q_full, h * 64, qt * 128, b);
      const int vrow = (b * H + h) * 64;
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait(&kv_empty[st], ((j >> 1) & 1) ^ 1)) {
          atomicOr(err, kErrWaitProducer);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&kv_full[st], 32768);
        tma_load_3d(smem + AttnSmem::K0 + st * 16384, &tmK, &kv_full[st], h * 64, j * 128, b);
        tma_load_2d(smem + AttnSmem::V0 + st * 16384, &tmVt, &kv_full[st], j * 128, vrow);
        tma_load_2d(smem + AttnSmem::V0 + st * 16384 + 8192, &tmVt, &kv_full[st], j * 128 + 64, vrow);
        issued = j + 1;
      }
      if (!ok) {
        mbar_wait(q_full, 0);
        for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j) mbar_wait(&kv_full[j & 1], (j >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16_f32(128, 128);
      constexpr uint32_t idO = idesc_f16_f32(128, 64);
      const uint32_t sQ = smem_u32(smem + AttnSmem::Q);
      const uint32_t sP = smem_u32(smem + AttnSmem::P);
      auto issue_s = [&](int j) {
        const uint32_t sK = smem_u32(smem + AttnSmem::K0 + (j & 1) * 16384);
        const uint32_t tS = tmem + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_f16(tS, desc_sw128(sQ + kk * 32), desc_sw128(sK + kk * 32), idS, kk);
        umma_commit(&s_full[j & 1]);
      };
      bool ok = mbar_wait(q_full, 0) && mbar_wait(&kv_full[0], 0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        if (j + 1 < nkv) {
          if (!mbar_wait(&kv_full[(j + 1) & 1], ((j + 1) >> 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(j + 1);
        }
        if (!mbar_wait(p_full, j & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sV = smem_u32(smem + AttnSmem::V0 + (j & 1) * 16384);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = sP + (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t bv = sV + (kk >> 2) * 8192 + (kk & 3) * 32;
          umma_f16(tO, desc_sw128(a), desc_sw128(bv), idO, kk);
        }
        umma_commit(o_full);
        umma_commit(&kv_empty[j & 1]);
      }
      if (!ok) atomicOr(err, kErrWaitMma);
    }
  } else {
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;  // score columns [32 sub, 32 sub + 32), output columns [16 sub, 16 sub + 16)
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const float c = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
    float o[kOCols];
#pragma unroll
    for (int i = 0; i < kOCols; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f;
    // This warp's 32 keys are half of the 64-key swizzle atom (sub >> 1).
    uint8_t* prow = smem + AttnSmem::P + (sub >> 1) * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
    const int ch0 = (sub & 1) * 4;
    bool ok = true;
    // Every iteration runs the quarter barrier and the p_full arrival even
    // after a failed wait (the work is skipped), so no thread is left waiting
    // on a barrier that another warp of its quarter will never reach.
    for (int j = 0; j < nkv; ++j) {
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&s_full[j & 1], (j >> 1) & 1));
      float s[kSCols];
      const int nvalid = min(128, T - j * 128) - sub * kSCols;  // valid columns of this warp
      float mx = -INFINITY;
      if (ok) {
        tc_fence_after();
        tmem_ld32(tmem + (j & 1) * 128 + sub * kSCols + lane_base, s);
#pragma unroll
        for (int i = 0; i < kSCols; ++i)
          if (i < nvalid) mx = fmaxf(mx, s[i]);
      }
      float* slot = red_max + (j & 1) * (kSubs * 128);
      slot[sub * 128 + r] = mx;
      quarter_barrier(q);
#pragma unroll
      for (int k = 0; k < kSubs; ++k) mx = fmaxf(mx, slot[k * 128 + r]);
      const float m_new = fmaxf(m, mx * c);
      const float alpha = ex2_approx(m - m_new);
      float rs = 0.f;
      uint32_t pk[kSCols / 2];
#pragma unroll
      for (int i = 0; i < kSCols; i += 2) {
        const float p0 = (i < nvalid) ? ex2_approx(fmaf(s[i], c, -m_new)) : 0.f;
        const float p1 = (i + 1 < nvalid) ? ex2_approx(fmaf(s[i + 1], c, -m_new)) : 0.f;
        __half2 hp = __floats2half2_rn(p0, p1);
        rs += p0 + p1;  // fp32 row sum (the conversion unit is the scarce pipe here)
        pk[i / 2] = *reinterpret_cast<uint32_t*>(&hp);
      }
      if (j > 0 && ok) {
        ok = __all_sync(0xffffffffu, mbar_wait(o_full, (j - 1) & 1));
        if (ok) {
          tc_fence_after();
          float v[16];
          tmem_ld16(tO + lane_base + sub * kOCols, v);
#pragma unroll
          for (int i = 0; i < kOCols; ++i) o[i] = (o[i] + v[i]) * alpha;
        }
      }
      l = l * alpha + rs;
      m = m_new;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        *reinterpret_cast<uint4*>(prow + (((ch0 + ch) ^ (r & 7)) << 4)) =
            make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_full, (nkv - 1) & 1));
    if (ok) {
      tc_fence_after();
      float v[16];
      tmem_ld16(tO + lane_base + sub * kOCols, v);
#pragma unroll
      for (int i = 0; i < kOCols; ++i) o[i] += v[i];
    } else if (lane == 0) {
      atomicOr(err, kErrWaitSoftmax);
    }
    red_sum[sub * 128 + r] = l;
    quarter_barrier(q);
    float ltot = 0.f;
#pragma unroll
    for (int k = 0; k < kSubs; ++k) ltot += red_sum[k * 128 + r];
    const int t = qt * 128 + r;
    if (ok && t < T) {
      const float inv = 1.0f / ltot;
      __half* dst = out + (static_cast<int64_t>(b) * T + t) * (H * 64) + h * 64 + sub * kOCols;
#pragma unroll
      for (int i = 0; i < kOCols; i += 8) {
        __half2 h0 = __floats2half2_rn(o[i] * inv, o[i + 1] * inv);
        __half2 h1 = __floats2half2_rn(o[i + 2] * inv, o[i + 3] * inv);
        __half2 h2 = __floats2half2_rn(o[i + 4] * inv, o[i + 5] * inv);
        __half2 h3 = __floats2half2_rn(o[i + 6] * inv, o[i + 7] * inv);
        *reinterpret_cast<uint4*>(dst + i) =
            make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                       *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t attention_prepare() {
  return cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnSmem::TOTAL);
}

cudaError_t launch_attention(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmVt, int T,
                             int batch, int H, __half* out, int* err, cudaStream_t st) {
  if (T <= 0 || batch <= 0) return cudaSuccess;
  dim3 grid((T + 127) / 128, H, batch);
  return launch_pdl(attention_kernel, grid, dim3(kAttnThreads), AttnSmem::TOTAL, st, tmQ, tmK, tmVt, T, H, out, err);
}

}  // namespace w2v
