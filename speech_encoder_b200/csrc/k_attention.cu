// Multi-head self-attention with no mask (plain SDPA over every frame of the
// window, as the LiteRT wav2vec2 discussion's fourth GPU rewrite leaves it),
// head dim 64, scale 1/8, fused flash-style on tcgen05.
//
// One CTA per (128-query tile, head, clip).  Warp roles:
//   warp 0      TMA: the Q tile once, then K and V^T tiles of 128 keys into a
//               2-deep ring
//   warp 1      TMEM owner; one thread issues S = Q K^T (M=128, N=128, K=64)
//               into TMEM columns [0,128) and, once P is in shared memory,
//               O_j = P V_j (M=128, N=64, K=128) into columns [128,192)
//   warps 2-5   one thread per query row: read its S row from TMEM, online
//               softmax in fp32 (exp2 with the 1/8 scale folded in), write P
//               (fp16) into the 128-byte-swizzled K-major layout the MMA reads,
//               and accumulate O_j into registers with the running rescale.
// V arrives transposed ([clip][head][64][T], written by the QKV projection's
// epilogue) so both MMAs read K-major operands.  Keys past T are zero-filled by
// TMA and masked to -inf before the exponent.
#include "ptx.cuh"
#include "w2v_internal.h"

namespace w2v {

struct AttnSmem {
  static constexpr int Q = 0;
  static constexpr int K0 = 16384;
  static constexpr int V0 = K0 + 2 * 16384;
  static constexpr int P = V0 + 2 * 16384;
  static constexpr int BAR = P + 32768;
  static constexpr int TOTAL = BAR + 256 + 1024;
};

__global__ void __launch_bounds__(192, 1)
attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmVt, int T, int H, __half* __restrict__ out, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* o_full = bars + 7;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nkv = (T + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(&kv_full[0], 1);
    mbar_init(&kv_full[1], 1);
    mbar_init(&kv_empty[0], 1);
    mbar_init(&kv_empty[1], 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_full, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmVt);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;
  const uint32_t tO = tmem + 128;

  if (warp == 0) {
    if (lane == 0) {
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
      bool ok = mbar_wait(q_full, 0);
      const uint32_t sQ = smem_u32(smem + AttnSmem::Q);
      const uint32_t sP = smem_u32(smem + AttnSmem::P);
      for (int j = 0; ok && j < nkv; ++j) {
        const int st = j & 1;
        if (!mbar_wait(&kv_full[st], (j >> 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + AttnSmem::K0 + st * 16384);
        const uint32_t sV = smem_u32(smem + AttnSmem::V0 + st * 16384);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_f16(tS, desc_sw128(sQ + kk * 32), desc_sw128(sK + kk * 32), idS, kk);
        umma_commit(s_full);
        if (!mbar_wait(p_full, j & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = sP + (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t bv = sV + (kk >> 2) * 8192 + (kk & 3) * 32;
          umma_f16(tO, desc_sw128(a), desc_sw128(bv), idO, kk);
        }
        umma_commit(o_full);
        umma_commit(&kv_empty[st]);
      }
      if (!ok) atomicOr(err, kErrWaitMma);
    }
  } else {
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const float c = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
    float o[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f;
    uint8_t* prow = smem + AttnSmem::P + (r >> 3) * 1024 + (r & 7) * 128;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      ok = mbar_wait(s_full, j & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float s[128];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        tmem_ld32(tS + lane_base + cc * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[cc * 32 + i] = v[i];
      }
      const int nvalid = min(128, T - j * 128);
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; ++i)
        if (i < nvalid) mx = fmaxf(mx, s[i]);
      const float m_new = fmaxf(m, mx * c);
      const float alpha = ex2_approx(m - m_new);
      float rs = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 128; i += 2) {
        const float p0 = (i < nvalid) ? ex2_approx(fmaf(s[i], c, -m_new)) : 0.f;
        const float p1 = (i + 1 < nvalid) ? ex2_approx(fmaf(s[i + 1], c, -m_new)) : 0.f;
        __half2 hp = __floats2half2_rn(p0, p1);
        const float2 back = __half22float2(hp);
        rs += back.x + back.y;
        pk[i / 2] = *reinterpret_cast<uint32_t*>(&hp);
      }
      if (j > 0) {
        ok = mbar_wait(o_full, (j - 1) & 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float v[32];
          tmem_ld32(tO + lane_base + cc * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[cc * 32 + i] = (o[cc * 32 + i] + v[i]) * alpha;
        }
      }
      l = l * alpha + rs;
      m = m_new;
      // P row r -> two 128-byte swizzle atoms (keys 0-63, 64-127).
#pragma unroll
      for (int a = 0; a < 2; ++a) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 u = make_uint4(pk[a * 32 + ch * 4], pk[a * 32 + ch * 4 + 1], pk[a * 32 + ch * 4 + 2],
                                     pk[a * 32 + ch * 4 + 3]);
          *reinterpret_cast<uint4*>(prow + a * 16384 + ((ch ^ (r & 7)) << 4)) = u;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok) {
      ok = mbar_wait(o_full, (nkv - 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (!ok) {
      if (lane == 0) atomicOr(err, kErrWaitSoftmax);
    } else {
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float v[32];
        tmem_ld32(tO + lane_base + cc * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[cc * 32 + i] += v[i];
      }
      const int t = qt * 128 + r;
      if (t < T) {
        const float inv = 1.0f / l;
        __half* dst = out + (static_cast<int64_t>(b) * T + t) * (H * 64) + h * 64;
#pragma unroll
        for (int i = 0; i < 64; i += 8) {
          __half2 h0 = __floats2half2_rn(o[i] * inv, o[i + 1] * inv);
          __half2 h1 = __floats2half2_rn(o[i + 2] * inv, o[i + 3] * inv);
          __half2 h2 = __floats2half2_rn(o[i + 4] * inv, o[i + 5] * inv);
          __half2 h3 = __floats2half2_rn(o[i + 6] * inv, o[i + 7] * inv);
          uint4 u;
          u.x = *reinterpret_cast<uint32_t*>(&h0);
          u.y = *reinterpret_cast<uint32_t*>(&h1);
          u.z = *reinterpret_cast<uint32_t*>(&h2);
          u.w = *reinterpret_cast<uint32_t*>(&h3);
          *reinterpret_cast<uint4*>(dst + i) = u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

cudaError_t attention_prepare() {
  return cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnSmem::TOTAL);
}

cudaError_t launch_attention(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmVt, int T,
                             int batch, int H, __half* out, int* err, cudaStream_t st) {
  if (T <= 0 || batch <= 0) return cudaSuccess;
  dim3 grid((T + 127) / 128, H, batch);
  attention_kernel<<<grid, 192, AttnSmem::TOTAL, st>>>(tmQ, tmK, tmVt, T, H, out, err);
  return cudaGetLastError();
}

}  // namespace w2v
