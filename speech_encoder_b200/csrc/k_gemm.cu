// tcgen05 GEMM with fused epilogues: every dense contraction of the forward
// pass (conv layers 1-6 as implicit GEMM, the feature projection, QKV, the
// attention output projection, both FFN layers and the CTC head) runs here.
//
// One CTA computes a 128 x BN output tile.  Warp roles:
//   warp 0      TMA producer: A and B K-blocks (64 fp16 = one 128-byte swizzle
//               atom wide) into a STAGES-deep shared-memory ring
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN,
//               K=16) into an fp32 accumulator in TMEM and frees ring slots
//               with tcgen05.commit
//   warps 2-5   epilogue: tcgen05.ld of their 32-lane quarter of the
//               accumulator, bias, GELU, residual add, fp16/fp32 stores (or
//               the Q / K / V^T split of the fused QKV projection)
#include <stdio.h>

#include "ptx.cuh"
#include "w2v_internal.h"

namespace w2v {

template <int BN>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN >= 256) ? 4 : (BN >= 128 ? 6 : 8);
  static constexpr int TMEM_COLS = BN;
  static constexpr int SMEM = STAGES * STAGE + 1024 + 256;
};

__device__ __forceinline__ void store_chunk_f16(__half* dst, const float (&v)[32], int nvalid, bool vec) {
  if (vec && nvalid >= 32) {
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
      uint4 u;
      __half2 h0 = __floats2half2_rn(v[i + 0], v[i + 1]);
      __half2 h1 = __floats2half2_rn(v[i + 2], v[i + 3]);
      __half2 h2 = __floats2half2_rn(v[i + 4], v[i + 5]);
      __half2 h3 = __floats2half2_rn(v[i + 6], v[i + 7]);
      u.x = *reinterpret_cast<uint32_t*>(&h0);
      u.y = *reinterpret_cast<uint32_t*>(&h1);
      u.z = *reinterpret_cast<uint32_t*>(&h2);
      u.w = *reinterpret_cast<uint32_t*>(&h3);
      *reinterpret_cast<uint4*>(dst + i) = u;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < nvalid) dst[i] = __float2half_rn(v[i]);
  }
}

__device__ __forceinline__ void store_chunk_f32(float* dst, const float (&v)[32], int nvalid, bool vec) {
  if (vec && nvalid >= 32) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < nvalid) dst[i] = v[i];
  }
}

__device__ __forceinline__ void add_residual(float (&v)[32], const void* res, int res_f32, int nvalid, bool vec) {
  if (res_f32) {
    const float* r = static_cast<const float*>(res);
    if (vec && nvalid >= 32) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 f = *reinterpret_cast<const float4*>(r + i);
        v[i] += f.x; v[i + 1] += f.y; v[i + 2] += f.z; v[i + 3] += f.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nvalid) v[i] += r[i];
    }
  } else {
    const __half* r = static_cast<const __half*>(res);
    if (vec && nvalid >= 32) {
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        uint4 u = *reinterpret_cast<const uint4*>(r + i);
        const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 f = __half22float2(h[j]);
          v[i + 2 * j] += f.x;
          v[i + 2 * j + 1] += f.y;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nvalid) v[i] += __half2float(r[i]);
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(192, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmShape s,
               GemmEpilogue e, int vec_ok, int* err) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * C::BM;
  const int n0 = blockIdx.y * BN;
  const int bz = blockIdx.z;
  const int nk = s.K / C::BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(accf, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
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
      int issued = 0;
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % C::STAGES;
        const uint32_t ph = (kb / C::STAGES) & 1;
        if (kb >= C::STAGES && !mbar_wait(&empty[st], ph ^ 1)) {
          atomicOr(err, kErrWaitProducer);
          ok = false;
          break;
        }
        uint8_t* sa = smem + st * C::STAGE;
        mbar_arrive_expect_tx(&full[st], C::STAGE);
        const int k = kb * C::BK;
        tma_load_3d(sa, &tmA, &full[st], k % s.a_kwrap, m0 + k / s.a_kwrap, bz);
        tma_load_2d(sa + C::A_BYTES, &tmB, &full[st], k, n0);
        issued = kb + 1;
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA exits.
        for (int kb = (issued > C::STAGES ? issued - C::STAGES : 0); kb < issued; ++kb)
          mbar_wait(&full[kb % C::STAGES], (kb / C::STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, BN);
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        const int st = kb % C::STAGES;
        if (!mbar_wait(&full[st], (kb / C::STAGES) & 1)) {
          atomicOr(err, kErrWaitMma);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + st * C::STAGE);
        const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16(tmem, desc_sw128(sa + kk * 32), desc_sw128(sb + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
        umma_commit(&empty[st]);
      }
      if (ok) umma_commit(accf);
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    bool ok = mbar_wait(accf, 0);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) atomicOr(err, kErrWaitEpilogue);
    tc_fence_after();
    if (ok) {
      const int row = m0 + r;
      const bool row_ok = row < s.M;
      const int64_t orow = static_cast<int64_t>(bz) * e.out_batch_stride + static_cast<int64_t>(row) * e.ldo;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + c, v);
        const int nc = n0 + c;
        if (nc >= s.N || !row_ok) continue;
        const int nvalid = min(32, s.N - nc);
        if (e.bias) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nvalid) v[i] += __ldg(e.bias + nc + i);
        }
        if (e.act) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = apply_act(v[i], e.act);
        }
        if (e.residual) {
          const int64_t roff = static_cast<int64_t>(bz) * e.res_batch_stride + static_cast<int64_t>(row) * e.ldr + nc;
          const void* rp = e.res_f32 ? static_cast<const void*>(static_cast<const float*>(e.residual) + roff)
                                     : static_cast<const void*>(static_cast<const __half*>(e.residual) + roff);
          add_residual(v, rp, e.res_f32, nvalid, vec_ok != 0);
        }
        if (e.qkv_d > 0) {
          const int region = nc / e.qkv_d;
          const int cc = nc - region * e.qkv_d;
          if (region == 0) {
            store_chunk_f16(static_cast<__half*>(e.out) + orow + cc, v, nvalid, vec_ok != 0);
          } else if (region == 1) {
            store_chunk_f16(static_cast<__half*>(e.out_k) + orow + cc, v, nvalid, vec_ok != 0);
          } else {
            // rows are clip-major: row = clip * t_len + t
            const int clip = row / e.t_len;
            const int t = row - clip * e.t_len;
            const int h = cc >> 6;
            const int dd0 = cc & 63;
            __half* dst = static_cast<__half*>(e.vt) +
                          (static_cast<int64_t>(clip * e.n_heads + h) * 64 + dd0) * e.t_pad + t;
#pragma unroll
            for (int i = 0; i < 32; ++i) dst[static_cast<int64_t>(i) * e.t_pad] = __float2half_rn(v[i]);
          }
        } else if (e.out_f32) {
          store_chunk_f32(static_cast<float*>(e.out) + orow + nc, v, nvalid, vec_ok != 0);
        } else {
          store_chunk_f16(static_cast<__half*>(e.out) + orow + nc, v, nvalid, vec_ok != 0);
        }
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

int gemm_pick_bn(const GemmShape& s) {
  if (s.N <= 32) return 32;
  if (s.N <= 64) return 64;
  const long mt = static_cast<long>((s.M + 127) / 128) * s.batch;
  if (mt * ((s.N + 255) / 256) >= 148) return 256;
  if (mt * ((s.N + 127) / 128) >= 100) return 128;
  return 64;
}

template <int BN>
static cudaError_t prepare_bn() {
  return cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, GemmCfg<BN>::SMEM);
}

cudaError_t gemm_prepare() {
  cudaError_t r;
  if ((r = prepare_bn<32>()) != cudaSuccess) return r;
  if ((r = prepare_bn<64>()) != cudaSuccess) return r;
  if ((r = prepare_bn<128>()) != cudaSuccess) return r;
  return prepare_bn<256>();
}

template <int BN>
static cudaError_t launch_bn(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmShape& s,
                             const GemmEpilogue& e, int vec_ok, int* err, cudaStream_t st) {
  using C = GemmCfg<BN>;
  dim3 grid((s.M + 127) / 128, (s.N + BN - 1) / BN, s.batch);
  gemm_tc_kernel<BN><<<grid, 192, C::SMEM, st>>>(tmA, tmB, s, e, vec_ok, err);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmShape& s, int bn,
                        const GemmEpilogue& e, int* err, cudaStream_t st) {
  if (s.M <= 0 || s.N <= 0 || s.batch <= 0) return cudaSuccess;
  if (s.K <= 0 || s.K % 64 != 0 || s.a_kwrap <= 0 || s.a_kwrap % 64 != 0) return cudaErrorInvalidValue;
  // Vector loads/stores need 16-byte aligned rows and column offsets.
  const int esz_out = e.out_f32 ? 4 : 2;
  const int esz_res = e.res_f32 ? 4 : 2;
  bool vec = (reinterpret_cast<uintptr_t>(e.out) % 16 == 0) && ((e.ldo * esz_out) % 16 == 0) &&
             ((e.out_batch_stride * esz_out) % 16 == 0);
  if (e.residual)
    vec = vec && (reinterpret_cast<uintptr_t>(e.residual) % 16 == 0) && ((e.ldr * esz_res) % 16 == 0) &&
          ((e.res_batch_stride * esz_res) % 16 == 0);
  if (e.qkv_d > 0) vec = vec && (reinterpret_cast<uintptr_t>(e.out_k) % 16 == 0);
  switch (bn) {
    case 32: return launch_bn<32>(tmA, tmB, s, e, vec, err, st);
    case 64: return launch_bn<64>(tmA, tmB, s, e, vec, err, st);
    case 128: return launch_bn<128>(tmA, tmB, s, e, vec, err, st);
    case 256: return launch_bn<256>(tmA, tmB, s, e, vec, err, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace w2v
