// Multi-head self-attention with no mask (plain SDPA over every frame of the
// window, as the LiteRT wav2vec2 discussion's fourth GPU rewrite leaves it),
// head dim 64, scale 1/8, fused flash-style on tcgen05.
//
// One CTA per (128-query tile, head, clip), 576 threads:
//   warp 0      TMA: the Q tile once, then K and V^T tiles of 128 keys into a
//               3-deep ring
//   warp 1      TMEM owner; one thread issues S_j = Q K_j^T (M=128, N=128,
//               K=64) into one of three TMEM score buffers and, once P_j is
//               written, O += P_j [V_j | 1] (M=128, N=80, K=128) into a TMEM
//               accumulator that lives across all key tiles.  P_j is the A
//               operand straight from tensor memory (it overwrites the first
//               half of each warp's own columns of S_j), so only V crosses the
//               shared-memory port for P V.  The scores run up to two tiles
//               ahead (S_{j+2} is issued as soon as its K/V tile lands and
//               P_{j-1} V_{j-1}, the last reader of its buffer, has completed;
//               polled together with P_j), so the softmax rarely waits for its
//               scores.
//   warps 2-17  softmax: four warps per TMEM lane quarter, each owning 32 of
//               the 128 key columns (and 16 of the 64 output columns) of its
//               32 query rows; a 128-thread named barrier per quarter
//               tells whether any row's reference must move (an OR-reduced
//               predicate), and only then are the row maxima combined
//               through shared memory.
// Online softmax with a lazily moved reference: a row's reference maximum m
// (log2 units, 1/8 scale folded in) moves only when the tile's maximum exceeds
// it by more than 8, so P = 2^(s/8 log2 e - m) stays <= 256 and the rescale of
// the TMEM accumulator (wait for the previous P V, load, scale, store) is rare;
// otherwise no softmax step waits for the tensor core.  P is formed as packed
// fp16 pairs (packed fp32 FMA, rounding, then the fp16x2 exponent instruction
// or, for a share of the pairs, a cubic on the FMA pipe) and stored to tensor
// memory in the layout of a K-major A operand (lane = query row, one 32-bit
// column per two keys).  The row sum
// is not accumulated by the threads: V^T carries a 65th row of ones, so column
// 64 of the accumulator is sum_k P[r][k] computed from the same fp16 P that
// multiplies V.
// V arrives transposed ([clip][head][64][T], written by the QKV projection's
// epilogue) so both MMAs read K-major operands.  Keys past T are zero-filled by
// TMA and masked to -inf before the exponent.
#include "ptx.cuh"
#include "w2v_internal.h"

namespace w2v {

constexpr int kKvStages = 3;

struct AttnSmem {
  static constexpr int Q = 0;
  static constexpr int K0 = 16384;                        // [stages] 128 keys x 64 dims, SW128
  static constexpr int kVHalf = 10240;                    // 80 rows (64 dims + ones + zeros) x 64 keys
  static constexpr int V0 = K0 + kKvStages * 16384;       // [stages][2 key halves] kVHalf
  static constexpr int RED = V0 + kKvStages * 2 * kVHalf;  // float red_max[2][4][128]
  static constexpr int BAR = RED + 4096;
  static constexpr int TOTAL = BAR + 256 + 1024;
};

constexpr int kSoftWarps = 16;
constexpr int kAttnThreads = 64 + 32 * kSoftWarps;
constexpr int kSubs = kSoftWarps / 4;    // warps per TMEM lane quarter
constexpr int kSCols = 128 / kSubs;      // score columns per warp
constexpr int kOCols = 64 / kSubs;       // output columns per warp
constexpr float kLazyLimit = 8.0f;       // log2 of the largest P value allowed (256)
constexpr int kPolyPairs = 6 * (kSCols / 32);  // exponential pairs per warp and tile computed by polynomial

__device__ __forceinline__ void quarter_barrier(int q) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "r"(32 * kSubs) : "memory");
}

// The same barrier, returning whether any thread of the quarter passed true.
__device__ __forceinline__ bool quarter_barrier_any(int q, bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"(v ? 1u : 0u), "r"(1 + q), "r"(32 * kSubs)
      : "memory");
  return out != 0;
}

// One CTA's work: query tile qt (local rows qt*128 ..) of one clip of T frames
// and head h.  The clip's queries start at row qrow of the Q map (batch
// coordinate bz), its keys at row krow0 of the K map and column krow0 of the V^T
// map (V^T row block vrow .. vrow+63 for this head), its outputs at row
// out_row0 of `out`.
__device__ __forceinline__ void attention_body(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmVt,
                                               int T, int H, __half* __restrict__ out, int* err, int qt, int h,
                                               int qrow, int krow0, int bz, int vrow, int64_t out_row0) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* red_max = reinterpret_cast<float*>(smem + AttnSmem::RED);  // [slot][sub][row]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [3]
  uint64_t* kv_empty = bars + 4;  // [3]
  uint64_t* s_full = bars + 7;    // [3]
  uint64_t* p_full = bars + 10;   // [2]
  uint64_t* pv_done = bars + 12;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkv = (T + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kKvStages; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], kSoftWarps);  // one arrival per softmax warp
      mbar_init(&pv_done[i], 1);
    }
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
  // Rows 64..79 of every V^T half-tile: row 64 all ones (fp16 1.0), the rest
  // zero.  They sit in the last two 1 KB swizzle atoms of each half-tile; a row
  // of identical 16-byte chunks is unchanged by the swizzle.
  for (int i = threadIdx.x; i < kKvStages * 2 * 2048 / 16; i += kAttnThreads) {
    const int half = i / 128, off = (i % 128) * 16;
    const uint32_t v = off < 128 ? 0x3C003C00u : 0u;
    *reinterpret_cast<uint4*>(smem + AttnSmem::V0 + half * AttnSmem::kVHalf + 8192 + off) = make_uint4(v, v, v, v);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem + 384;   // 80 columns: O (64) | row sum | zeros; scores at 0, 128, 256

  if (warp == 0) {
    if (lane == 0) {
      pdl_wait();
      mbar_arrive_expect_tx(q_full, 16384);
      tma_load_3d(smem + AttnSmem::Q, &tmQ, q_full, h * 64, qrow, bz);
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % kKvStages;
        if (j >= kKvStages && !mbar_wait(&kv_empty[st], ((j / kKvStages) & 1) ^ 1)) {
          atomicOr(err, kErrWaitProducer);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&kv_full[st], 32768);
        uint8_t* vs = smem + AttnSmem::V0 + st * 2 * AttnSmem::kVHalf;
        tma_load_3d(smem + AttnSmem::K0 + st * 16384, &tmK, &kv_full[st], h * 64, krow0 + j * 128, bz);
        tma_load_2d(vs, &tmVt, &kv_full[st], krow0 + j * 128, vrow);
        tma_load_2d(vs + AttnSmem::kVHalf, &tmVt, &kv_full[st], krow0 + j * 128 + 64, vrow);
        issued = j + 1;
      }
      if (!ok) {
        mbar_wait(q_full, 0);
        for (int j = (issued > kKvStages ? issued - kKvStages : 0); j < issued; ++j)
          mbar_wait(&kv_full[j % kKvStages], (j / kKvStages) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16_f32(128, 128);
      constexpr uint32_t idO = idesc_f16_f32(128, 80);
      // Descriptors built once; a buffer or K step only moves the 14-bit
      // start-address field (16-byte units; addresses stay below 256 KB).
      const uint64_t dQ = desc_sw128(smem_u32(smem + AttnSmem::Q));
      const uint64_t dK0 = desc_sw128(smem_u32(smem + AttnSmem::K0));
      const uint64_t dV0 = desc_sw128(smem_u32(smem + AttnSmem::V0));
      auto issue_s = [&](int j) {
        const int b = j % kKvStages;
        const uint64_t dK = dK0 + static_cast<uint64_t>(b * (16384 >> 4));
        const uint32_t tS = tmem + b * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) umma_f16(tS, dQ + 2 * kk, dK + 2 * kk, idS, kk);
        umma_commit(&s_full[b]);
      };
      bool ok = mbar_wait(q_full, 0) && mbar_wait(&kv_full[0], 0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        if (nkv > 1) {
          ok = mbar_wait(&kv_full[1], 0);
          if (ok) {
            tc_fence_after();
            issue_s(1);
          }
        }
      }
      // S_m may be issued once its K/V stage has landed and P_{m-3} V_{m-3},
      // the last reader of its score buffer (P_{m-3} lives there), has
      // completed; m <= j + 2 while waiting for P_j.  Completed P V products
      // are confirmed strictly in order (pv_seen), and P_j V_j is issued only
      // after P_{j-2} V_{j-2} was confirmed, so the phase tested on a pv_done
      // barrier is always the latest one it can have reached: a parity test
      // would otherwise pass or fail wrongly once the barrier had moved two
      // phases on.  The thread polls everything with test_wait (a try_wait on
      // an open phase may suspend it and delay the other barriers), so P_j V_j
      // never waits behind a K/V tile that is still in flight (that tile's
      // stage is only refilled after an earlier P V completes).
      int next_s = nkv > 1 ? 2 : 1;
      int pv_seen = 0;  // P V products known complete
      for (int j = 0; ok && j < nkv; ++j) {
        bool have_p = false, ready = false;
        uint64_t t0 = globaltimer_ns();
        for (uint32_t it = 1;; ++it) {
          while (pv_seen < j && mbar_test_wait(&pv_done[pv_seen & 1], (pv_seen >> 1) & 1)) ++pv_seen;
          if (next_s < nkv && next_s <= j + 2 && (next_s < 3 || pv_seen >= next_s - 2) &&
              mbar_test_wait(&kv_full[next_s % kKvStages], (next_s / kKvStages) & 1)) {
            tc_fence_after();
            issue_s(next_s);
            ++next_s;
            t0 = globaltimer_ns();
          }
          if (!have_p) have_p = mbar_test_wait(&p_full[j & 1], (j >> 1) & 1);
          if (have_p && (j < 2 || pv_seen >= j - 1)) {
            ready = true;
            break;
          }
          if ((it & 255u) == 0 && globaltimer_ns() - t0 > W2V_WAIT_LIMIT_NS) break;
        }
        if (!ready) {
          ok = false;
          break;
        }
        tc_fence_after();
        // P_j: keys kSCols w .. kSCols (w + 1) - 1 (softmax warp w of a lane
        // quarter) at columns kSCols w .. kSCols w + kSCols / 2 - 1 of score
        // buffer j % 3, so K step kk (16 keys) starts at column
        // kSCols (16 kk / kSCols) + 8 (kk % (kSCols / 16)).
        const uint32_t tP = tmem + static_cast<uint32_t>((j % kKvStages) * 128);
        const uint64_t dV = dV0 + static_cast<uint64_t>((j % kKvStages) * (2 * AttnSmem::kVHalf >> 4));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = tP + static_cast<uint32_t>(kSCols * (16 * kk / kSCols) + 8 * (kk % (kSCols / 16)));
          const uint64_t bv = dV + static_cast<uint64_t>((kk >> 2) * (AttnSmem::kVHalf >> 4) + (kk & 3) * 2);
          umma_f16_ts(tO, a, bv, idO, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&pv_done[j & 1]);
        umma_commit(&kv_empty[j % kKvStages]);
      }
      if (!ok) atomicOr(err, kErrWaitMma);
    }
  } else {
    const int q = warp & 3;
    const int sub = (warp - 2) >> 2;  // score columns [kSCols sub, +kSCols), output columns [kOCols sub, +kOCols)
    const int r = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const float c = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
    float m_ref = -INFINITY;                        // reference maximum, log2 units
    bool ok = true;
    // Every iteration runs the quarter barrier and the p_full arrival even
    // after a failed wait (the work is skipped), so no thread is left waiting
    // on a barrier that another warp of its quarter will never reach.
    for (int j = 0; j < nkv; ++j) {
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&s_full[j % kKvStages], (j / kKvStages) & 1));
      float s[kSCols];
      const int nvalid = min(128, T - j * 128) - sub * kSCols;  // valid columns of this warp
      float mx = -INFINITY;
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int h32 = 0; h32 < kSCols; h32 += 32)
          tmem_ld32(tmem + (j % kKvStages) * 128 + sub * kSCols + h32 + lane_base,
                    *reinterpret_cast<float(*)[32]>(s + h32));
        if (nvalid < kSCols) {
#pragma unroll
          for (int i = 0; i < kSCols; ++i)
            if (i >= nvalid) s[i] = -INFINITY;
        }
        float m0 = fmax3(s[0], s[1], s[2]), m1 = fmax3(s[3], s[4], s[5]);
#pragma unroll
        for (int i = 6; i + 3 < kSCols; i += 4) {
          m0 = fmax3(m0, s[i], s[i + 1]);
          m1 = fmax3(m1, s[i + 2], s[i + 3]);
        }
        mx = fmax3(m0, m1, s[kSCols - 2]);
        mx = fmaxf(mx, s[kSCols - 1]);
      }
      // Move a row's reference when the tile's maximum is more than 2^8 above
      // it.  Usually no row of the lane quarter moves: one barrier whose
      // predicate reduction says so replaces the exchange of the row maxima
      // (exact: a row's maximum exceeds the limit only if one of its warps'
      // column maxima does).  Otherwise the maxima are combined through shared
      // memory and the warps of a row see the same mt and m_ref and decide
      // alike.
      bool move = false;
      float mt = 0.f;
      if (quarter_barrier_any(q, mx * c > m_ref + kLazyLimit)) {
        float* slot = red_max + (j & 1) * (kSubs * 128);
        slot[sub * 128 + r] = mx;
        quarter_barrier(q);
        mx = slot[r];
#pragma unroll
        for (int k = 1; k < kSubs; ++k) mx = fmaxf(mx, slot[k * 128 + r]);
        mt = mx * c;  // finite: every key tile has a valid column
        move = mt > m_ref + kLazyLimit;
      }
      if (__any_sync(0xffffffffu, move)) {
        const float m_new = move ? mt : m_ref;
        if (j > 0 && ok) {
          // Rescale this warp's accumulator columns (and, for sub 0, the row
          // sum column) once the previous P V has landed.
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1));
          if (ok) {
            tc_fence_after();
            const float alpha = ex2_approx(m_ref - m_new);
            float v[16];
#pragma unroll
            for (int h16 = 0; h16 < kOCols; h16 += 16) {
              tmem_ld16(tO + lane_base + sub * kOCols + h16, v);
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] *= alpha;
              tmem_st16(tO + lane_base + sub * kOCols + h16, v);
            }
            if (sub == 0) {
              tmem_ld16(tO + lane_base + 64, v);
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] *= alpha;
              tmem_st16(tO + lane_base + 64, v);
            }
          }
        }
        m_ref = m_new;
      }
      uint32_t pk[kSCols / 2];
      const float nb = -m_ref;
      // The first kPolyPairs pairs on the FMA/ALU pipes, the rest on the
      // exponent unit (16 results per clock per SM), so both pipes share the load.
#pragma unroll
      for (int i = 0; i < kSCols; i += 2)
        pk[i / 2] = (i / 2 < kPolyPairs) ? exp2_affine_poly_f16x2(s[i], s[i + 1], c, nb)
                                         : exp2_affine_f16x2(s[i], s[i + 1], c, nb);
      // This warp's arrival for P_j goes to the barrier that carried P_{j-2}:
      // that phase must be complete first, which P_{j-2} V_{j-2} having run
      // shows (no warp of another lane quarter may still owe it an arrival).
      if (j >= 2 && ok) ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[j & 1], ((j - 2) >> 1) & 1));
      // P over the first half of this warp's own score columns (read above):
      // packed key pairs, the A operand layout of P V.
      if (ok) {
#pragma unroll
        for (int h16 = 0; h16 < kSCols / 2; h16 += 16)
          tmem_st16_u32(tmem + (j % kKvStages) * 128 + sub * kSCols + h16 + lane_base,
                        *reinterpret_cast<const uint32_t(*)[16]>(pk + h16));
      }
      tc_fence_before();
      // one arrival per warp: 512 arrivals on one barrier word serialise
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[j & 1]);
    }
    // The last product (P_{last-2} V_{last-2}, the previous phase of its
    // barrier, was waited for above, so the parity is unambiguous).
    const int last = nkv - 1;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[last & 1], (last >> 1) & 1));
    const int t = qt * 128 + r;
    if (ok) {
      tc_fence_after();
      float o[kOCols];
#pragma unroll
      for (int h16 = 0; h16 < kOCols; h16 += 16)
        tmem_ld16(tO + lane_base + sub * kOCols + h16, *reinterpret_cast<float(*)[16]>(o + h16));
      const float l = tmem_ld1(tO + lane_base + 64);
      if (t < T) {
        const float inv = 1.0f / l;
        __half* dst = out + (out_row0 + t) * (H * 64) + h * 64 + sub * kOCols;
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
    } else if (lane == 0) {
      atomicOr(err, kErrWaitSoftmax);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

__global__ void __launch_bounds__(kAttnThreads, 1)
attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmVt, int T, int H, __half* __restrict__ out, int* err) {
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  attention_body(tmQ, tmK, tmVt, T, H, out, err, qt, h, qt * 128, 0, b, (b * H + h) * 64,
                 static_cast<int64_t>(b) * T);
}

// Clips of different lengths packed along the rows of one [rows][H*64]
// Q/K/output matrix (V^T [H*64][rows]), each clip's rows starting on a
// 128-row boundary, so that no query or key tile holds two clips.  Query
// tiles are numbered clip after clip; each attends to its own clip's keys.
__global__ void __launch_bounds__(kAttnThreads, 1)
attention_varlen_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmVt, int H, __half* __restrict__ out, int* err,
                        const AttnClips clips) {
  int c = 0;
  while (c + 1 < clips.n && clips.qt0[c + 1] <= static_cast<int>(blockIdx.x)) ++c;
  const int qt = static_cast<int>(blockIdx.x) - clips.qt0[c], h = blockIdx.y;
  const int row0 = clips.row0[c];
  attention_body(tmQ, tmK, tmVt, clips.len[c], H, out, err, qt, h, row0 + qt * 128, row0, 0, h * 64, row0);
}

cudaError_t attention_prepare() {
  cudaError_t r = cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnSmem::TOTAL);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(attention_varlen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnSmem::TOTAL);
  return r;
}

cudaError_t launch_attention(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmVt, int T,
                             int batch, int H, __half* out, int* err, cudaStream_t st) {
  if (T <= 0 || batch <= 0) return cudaSuccess;
  dim3 grid((T + 127) / 128, H, batch);
  return launch_pdl(attention_kernel, grid, dim3(kAttnThreads), AttnSmem::TOTAL, st, tmQ, tmK, tmVt, T, H, out, err);
}

cudaError_t launch_attention_varlen(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmVt,
                                    const AttnClips& clips, int H, __half* out, int* err, cudaStream_t st) {
  if (clips.n <= 0 || clips.n > kMaxVarlenClips) return cudaErrorInvalidValue;
  for (int c = 0; c < clips.n; ++c)
    if (clips.row0[c] % 128 != 0 || clips.len[c] <= 0 || clips.qt0[c + 1] - clips.qt0[c] != (clips.len[c] + 127) / 128)
      return cudaErrorInvalidValue;
  dim3 grid(clips.qt0[clips.n], H, 1);
  return launch_pdl(attention_varlen_kernel, grid, dim3(kAttnThreads), AttnSmem::TOTAL, st, tmQ, tmK, tmVt, H, out,
                    err, clips);
}

}  // namespace w2v
