// tcgen05 GEMM with fused epilogues: every dense contraction of the forward
// pass (conv layers 1-6 as implicit GEMM, the feature projection, QKV, the
// attention output projection, both FFN layers and the CTC head) runs here.
//
// One CTA computes a 128 x BN output tile (or a K-range of it, see split-K),
// 320 threads:
//   warp 0      TMA producer: A and B K-blocks (64 fp16 = one 128-byte swizzle
//               atom wide) into a STAGES-deep shared-memory ring.  Weight (B)
//               blocks of the first ring fill are issued before waiting on the
//               previous kernel (programmatic dependent launch).
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN,
//               K=16) into an fp32 accumulator in TMEM and frees ring slots
//               with tcgen05.commit
//   warps 2-9   epilogue.  Two warps per TMEM lane quarter (32 rows) split the
//               columns.  Three forms:
//     direct    (one CTA per tile, TMA-storable output): each thread takes its
//               row's 32-column chunks from TMEM, adds bias and residual,
//               applies GELU, writes the chunk in the output type into a
//               swizzled staging box in the drained operand ring, and one lane
//               per warp issues a TMA tensor store of the 32 x 32 box.
//     split-K   (s.splits = S > 1): the S CTAs of a tile form a thread-block
//               cluster, each reducing a contiguous range of K blocks.  After a
//               cluster barrier (all rings drained) every thread pushes its fp32
//               partial row chunks straight into the shared memory of the CTA
//               that owns those rows (remote st.shared::cluster, fire and
//               forget); after a second barrier each CTA sums the S received
//               copies of its 128/S rows in rank order (deterministic) and
//               stores coalesced rows.  Small-M projections thereby use wide,
//               L2-friendly tiles, still fill the SMs, and split the epilogue.
//     generic   (V part of the fused QKV projection, unaligned outputs): the
//               fp32 tile is parked in shared memory and walked row by row
//               (column by column for V, which is stored transposed per head)
//               with coalesced stores.
#include <cstring>

#include "ptx.cuh"
#include "w2v_internal.h"

namespace w2v {

// PAIR: a CTA pair computes a 256 x BN tile (cta_group::2), each CTA holding
// 128 rows of A and BN/2 rows of B per stage.
template <int BN, bool PAIR = false>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = (PAIR ? BN / 2 : BN) * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int RING_MAX = 200 * 1024;
  static constexpr int STAGES = (RING_MAX / STAGE) > 8 ? 8 : (RING_MAX / STAGE);
  static constexpr int RING = STAGES * STAGE;
  static constexpr int TMEM_COLS = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  static constexpr int CHUNK = BN >= 64 ? 32 : 16;  // TMEM columns per load
  static constexpr int ROW_CHUNKS = BN / 4;         // 16-byte fp32 chunks per row
  static constexpr int BIAS_OFF = RING;
  static constexpr int VEC_OFF = BIAS_OFF + BN * 4;   // LN column vectors, 2 x BN floats
  static constexpr int ROWLN_OFF = VEC_OFF + 2 * BN * 4;  // per-row LN factors, 128 float2
  static constexpr int BAR_OFF = ROWLN_OFF + 128 * 8;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  // Row LayerNorm over a cluster of column tiles (ln_mode 3): per row the two
  // half-tile (count, mean, M2) and one slot per cluster CTA (up to 8),
  // outside the ring so that peers may write before this CTA's ring drains.
  // Only those launches request it (a larger request shrinks the SM's L1).
  static constexpr int LN3_OFF = BAR_OFF + 256;
  static constexpr int LN3_BYTES = (2 + 8) * 128 * 16;
  static constexpr int SMEM_LN3 = SMEM + LN3_BYTES;
  static_assert(SMEM_LN3 <= 227 * 1024, "a CTA's dynamic shared memory is at most 227 KB");
  // An fp16 residual tile (128 rows x BN) staged by TMA during the mainloop
  // takes the ring's last RES_STAGES stages.
  static constexpr int RES_BYTES = BM * BN * 2;
  static constexpr int RES_STAGES = (RES_BYTES + STAGE - 1) / STAGE;
  static_assert(BM * BN * 4 <= RING, "parked tile must fit in the operand ring");
  static_assert(ROW_CHUNKS >= 8, "row swizzle needs >= 8 chunks");
};

constexpr int kGemmThreads = 320;
constexpr int kEpiThreads = 256;
// Flag in the kernel's mode word: the fp16 residual tile is staged in shared
// memory by TMA (its map in tmO2's slot, which only the QKV split uses).
constexpr int kModeResTma = 16;
static_assert(sizeof(GemmEpiArgs) <= 128, "the GEMM kernel's parameter block must stay within 808 bytes");

// fp32 tile rows of `row_chunks` 16-byte chunks; chunk j of row r lives at
// chunk (j ^ (r & 7)) so that 8 consecutive rows hit 8 different bank groups.
__device__ __forceinline__ uint32_t swz_off(int row_chunks, int r, int j) {
  return static_cast<uint32_t>((r * row_chunks + (j ^ (r & 7))) * 16);
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Epilogue chunk helpers.  Each tests its uniform condition once, outside the
// unrolled loop over the chunk, so that the code a launch executes is one
// compact straight run (it runs once per CTA, from a cold instruction cache).
// v += bias (tile columns lcol..lcol+N-1, 16-byte aligned in shared memory)
template <int N>
__device__ __forceinline__ void add_cols(float (&v)[N], const float* col_s) {
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    const float4 b = *reinterpret_cast<const float4*>(col_s + i);
    v[i] += b.x;
    v[i + 1] += b.y;
    v[i + 2] += b.z;
    v[i + 3] += b.w;
  }
}

// Folded LayerNorm of the A rows (ln_mode 1): v = rstd * v - mean * rstd * colsum
template <int N>
__device__ __forceinline__ void ln1_cols(float (&v)[N], const float* cs_s, float2 lnr) {
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    const float4 cs = *reinterpret_cast<const float4*>(cs_s + i);
    v[i] = fmaf(lnr.x, v[i], lnr.y * cs.x);
    v[i + 1] = fmaf(lnr.x, v[i + 1], lnr.y * cs.y);
    v[i + 2] = fmaf(lnr.x, v[i + 2], lnr.y * cs.z);
    v[i + 3] = fmaf(lnr.x, v[i + 3], lnr.y * cs.w);
  }
}

template <int N>
__device__ __forceinline__ void act_inplace(float (&v)[N], int act) {
  if (act == 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = gelu_erf(v[i]);
  } else if (act == 2) {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = gelu_tanh(v[i]);
  }
}

// v += residual f, normalised first when ln_mode == 2:
// (f * rstd - mean * rstd) * gamma + beta (gamma at g_s, beta at g_s + bn)
template <int N>
__device__ __forceinline__ void add_residual(float (&v)[N], const float (&f)[N], int ln_mode, const float* g_s,
                                             int bn, float2 lnr) {
  if (ln_mode == 2) {
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      const float4 g = *reinterpret_cast<const float4*>(g_s + i);
      const float4 b = *reinterpret_cast<const float4*>(g_s + bn + i);
      v[i] += fmaf(fmaf(f[i], lnr.x, lnr.y), g.x, b.x);
      v[i + 1] += fmaf(fmaf(f[i + 1], lnr.x, lnr.y), g.y, b.y);
      v[i + 2] += fmaf(fmaf(f[i + 2], lnr.x, lnr.y), g.z, b.z);
      v[i + 3] += fmaf(fmaf(f[i + 3], lnr.x, lnr.y), g.w, b.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] += f[i];
  }
}

// Final epilogue for 4 consecutive columns [col, col+4) of row grow: bias
// (from shared memory), GELU, residual, store.  `vec` selects 16-/8-byte
// accesses (row starts and pointers 16-byte aligned, full 4-vector in range).
// lnr: the row's LayerNorm factors (rstd, -mean * rstd) when e.ln_mode != 0;
// vec_s: the LN column vectors of this tile (ln_mode 1: column sums; 2: gamma,
// then beta at vec_s + BN).
// res_s: the staged fp16 residual tile (boxes of 32 columns x 128 rows,
// 64-byte rows, 64-byte swizzle; zeros outside the matrix) or null to read
// the residual from global memory; lrow: the tile row.
__device__ __forceinline__ void finish4(float (&x)[4], const float* bias_s, const float* vec_s, int bn, float2 lnr,
                                        int lcol, int grow, int col, int nv, int bzb, const GemmEpiArgs& e,
                                        void* outp, int ocol0, bool vec, const uint8_t* res_s = nullptr,
                                        int lrow = 0) {
  const int ln_mode = e.ln_cfg & 255;
  if (ln_mode == 1) ln1_cols<4>(x, vec_s + lcol, lnr);
  add_cols<4>(x, bias_s + lcol);
  act_inplace<4>(x, e.act);
  if (e.residual) {
    const int64_t roff = static_cast<int64_t>(bzb) * e.res_batch_stride + static_cast<int64_t>(grow) * e.ldr + col;
    float rv[4] = {0.f, 0.f, 0.f, 0.f};
    if (res_s) {
      const int cc = lcol & 31;
      const uint2 u = *reinterpret_cast<const uint2*>(res_s + (lcol >> 5) * 8192 + lrow * 64 +
                                                      (((cc >> 3) ^ ((lrow >> 1) & 3)) << 4) + (cc & 7) * 2);
      const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
      const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
      rv[0] = a.x; rv[1] = a.y; rv[2] = b.x; rv[3] = b.y;
    } else if (e.res_f32) {
      const float* rp = static_cast<const float*>(e.residual) + roff;
      if (vec && nv == 4) {
        const float4 t = *reinterpret_cast<const float4*>(rp);
        rv[0] = t.x; rv[1] = t.y; rv[2] = t.z; rv[3] = t.w;
      } else {
        for (int i = 0; i < nv; ++i) rv[i] = rp[i];
      }
    } else {
      const __half* rp = static_cast<const __half*>(e.residual) + roff;
      if (vec && nv == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(rp);
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        rv[0] = a.x; rv[1] = a.y; rv[2] = b.x; rv[3] = b.y;
      } else {
        for (int i = 0; i < nv; ++i) rv[i] = __half2float(rp[i]);
      }
    }
    add_residual<4>(x, rv, ln_mode, vec_s + lcol, bn, lnr);
  }
  const int64_t ooff = static_cast<int64_t>(bzb) * e.out_batch_stride + static_cast<int64_t>(grow) * e.ldo + (col - ocol0);
  if (e.out_f32) {
    float* op = static_cast<float*>(outp) + ooff;
    if (vec && nv == 4)
      *reinterpret_cast<float4*>(op) = make_float4(x[0], x[1], x[2], x[3]);
    else
      for (int i = 0; i < nv; ++i) op[i] = x[i];
  } else {
    __half* op = static_cast<__half*>(outp) + ooff;
    if (vec && nv == 4)
      *reinterpret_cast<uint2*>(op) = make_uint2(pack_h2(x[0], x[1]), pack_h2(x[2], x[3]));
    else
      for (int i = 0; i < nv; ++i) op[i] = __float2half_rn(x[i]);
  }
}

// mode: 0 generic, 1 direct (TMA store), 2 split-K through distributed shared
// memory (each cluster CTA finishing a band of rows), 3 split-K through an L2
// scratch, 4 split-K through distributed shared memory (each cluster CTA
// finishing a group of columns); 3 and 4 with the direct stores.
// SPLIT: the instantiation with cluster code, for split-K launches (modes
// 2-4) and the row-LayerNorm epilogue (mode 1, ln_mode 3); the other one runs
// modes 0 and 1 only.
// PAIR: CTA pairs (clusters of 2 along M) on 256-row tiles with the 2-CTA
// tensor-core instructions, mode 1 only.  The pair halves the B operand bytes
// each SM takes in per output, which bounds the mainloop (an SM receives
// about 72 bytes per clock from L2).  Each CTA still owns 128 accumulator rows
// (m0 = blockIdx.x * 128) and runs the same epilogue on them.
template <int BN, bool SPLIT, bool PAIR>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO2,
               const __grid_constant__ CUtensorMap tmV, GemmDims s, GemmEpiArgs e, int vec_ok, int mode_word,
               int* err) {
  static_assert(!(SPLIT && PAIR), "pairs do not split K");
  using C = GemmCfg<BN, PAIR>;
  const int mode = mode_word & 15;
  const bool res_tma = (mode_word & kModeResTma) != 0;
  // ring stages in use (the staged residual takes the last ones)
  const int nst = res_tma ? C::STAGES - C::RES_STAGES : C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* bias_s = reinterpret_cast<float*>(smem + C::BIAS_OFF);
  float* vec_s = reinterpret_cast<float*>(smem + C::VEC_OFF);
  float2* rowln_s = reinterpret_cast<float2*>(smem + C::ROWLN_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::STAGES;
  uint64_t* accf = empty + C::STAGES;
  uint64_t* peer_bar = accf + 1;  // [8] mode 3: one per epilogue warp
  uint64_t* res_bar = peer_bar + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(res_bar + 1);
  const uint8_t* res_s = smem + nst * C::STAGE;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * C::BM;
  const int n0 = blockIdx.y * BN;
  const int nk = s.K / C::BK;
  const int S = s.splits;
  const int split = S > 1 ? static_cast<int>(blockIdx.z) : 0;
  const int bzb = S > 1 ? 0 : static_cast<int>(blockIdx.z);  // batch index
  const int kb0 = split * nk / S;
  const int nkl = (split + 1) * nk / S - kb0;  // K blocks of this CTA (>= 1)
  const int pre = nkl < nst ? nkl : nst;
  // pair rank (0: the CTA that issues the MMAs), cluster rank of that CTA,
  // the first B row this CTA loads, and the pair's CTA mask
  const uint32_t crank = PAIR ? cluster_ctarank() : 0u;
  const uint32_t prank = crank & 1u;
  const uint32_t lead = crank & ~1u;
  const int nb0 = PAIR ? n0 + static_cast<int>(prank) * (BN / 2) : n0;
  const uint16_t pmask = static_cast<uint16_t>(3u << lead);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(accf, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&peer_bar[i], 1);
    mbar_init(res_bar, 1);
    fence_mbar_init();
    pdl_launch_dependents();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    // Weights do not depend on the previous kernel: start them right away
    // (pairs: after the cluster barrier below, since they complete on the
    // other CTA's barriers).
    if (!PAIR) {
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], C::STAGE);
        tma_load_2d(smem + i * C::STAGE + C::A_BYTES, &tmB, &full[i], (kb0 + i) * C::BK, n0);
      }
    }
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  // pairs: both CTAs' barriers are initialised before either signals the other
  if (PAIR) cluster_sync();
  // row LayerNorm over a cluster: announce that this CTA runs; the epilogue
  // waits for every peer's announcement before writing into their memory
  // (the cluster instantiation only: the plain one carries no cluster code)
  const bool ln3_cluster = SPLIT && !PAIR && mode == 1 && (e.ln_cfg & 255) == 3;
  if (ln3_cluster) cluster_arrive_relaxed();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The fp16 residual tile of this CTA's 128 rows, as BN/32 boxes of 32
  // columns, into the ring's tail on this CTA's own barrier (pairs too); the
  // epilogue waits for it.
  auto stage_residual = [&]() {
    mbar_arrive_expect_tx(res_bar, C::RES_BYTES);
    for (int cb = 0; cb < BN / 32; ++cb)
      tma_load_3d(smem + nst * C::STAGE + cb * 8192, &tmO2, res_bar, n0 + cb * 32, m0, bzb);
  };

  if (PAIR && warp == 0) {
    if (lane == 0) {
      // Both CTAs load their own A rows and B half; every copy completes on
      // the even CTA's full barrier, which expects the bytes of both.
      auto fbar = [&](int st) { return mapa_shared(smem_u32(&full[st]), lead); };
      for (int i = 0; i < pre; ++i) {
        if (prank == 0) mbar_arrive_expect_tx(&full[i], 2 * C::STAGE);
        tma_load_2d_pair(smem + i * C::STAGE + C::A_BYTES, &tmB, fbar(i), (kb0 + i) * C::BK, nb0);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) {
        const int k = (kb0 + i) * C::BK;
        tma_load_3d_pair(smem + i * C::STAGE, &tmA, fbar(i), k % s.a_kwrap, m0 + k / s.a_kwrap, bzb);
      }
      if (res_tma) stage_residual();
      bool ok = true;
      // Stage, phase and A coordinates advance incrementally: this thread's
      // own instruction latency is on the mainloop's critical path.
      int st = pre == nst ? 0 : pre;
      uint32_t ph = pre == nst ? 1u : 0u;
      int k = (kb0 + pre) * C::BK;
      int kx = k % s.a_kwrap, ky = k / s.a_kwrap;
      for (int i = pre; i < nkl; ++i) {
        if (!mbar_wait(&empty[st], ph ^ 1)) {
          atomicOr(err, kErrWaitProducer);
          ok = false;
          break;
        }
        uint8_t* sa = smem + st * C::STAGE;
        if (prank == 0) mbar_arrive_expect_tx(&full[st], 2 * C::STAGE);
        tma_load_3d_pair(sa, &tmA, fbar(st), kx, m0 + ky, bzb);
        tma_load_2d_pair(sa + C::A_BYTES, &tmB, fbar(st), k, nb0);
        k += C::BK;
        kx += C::BK;
        if (kx == s.a_kwrap) {
          kx = 0;
          ++ky;
        }
        if (++st == nst) {
          st = 0;
          ph ^= 1u;
        }
      }
      // Wait until the last stages have been consumed: every copy into this
      // CTA has landed and every release the MMA issuer sent here has
      // arrived, before this CTA may leave.
      if (ok) {
        for (int i = (nkl > nst ? nkl - nst : 0); i < nkl; ++i)
          if (!mbar_wait(&empty[i % nst], (i / nst) & 1)) {
            atomicOr(err, kErrWaitProducer);
            break;
          }
      }
    }
  } else if (PAIR && warp == 1) {
    if (lane == 0 && prank == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(256, BN);
      const uint64_t dA0 = desc_sw128(smem_u32(smem));
      const uint64_t dB0 = desc_sw128(smem_u32(smem) + C::A_BYTES);
      bool ok = true;
      int st = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nkl; ++i) {
        if (!mbar_wait(&full[st], ph)) {
          atomicOr(err, kErrWaitMma);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t off = static_cast<uint64_t>(st * (C::STAGE >> 4));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16_pair(tmem, dA0 + off + 2 * kk, dB0 + off + 2 * kk, idesc, (i | kk) != 0 ? 1u : 0u);
        umma_commit_pair(&empty[st], pmask);
        if (++st == nst) {
          st = 0;
          ph ^= 1u;
        }
      }
      if (ok) umma_commit_pair(accf, pmask);
    }
  } else if (warp == 0) {
    if (lane == 0) {
      pdl_wait();
      for (int i = 0; i < pre; ++i) {
        const int k = (kb0 + i) * C::BK;
        tma_load_3d(smem + i * C::STAGE, &tmA, &full[i], k % s.a_kwrap, m0 + k / s.a_kwrap, bzb);
      }
      if (res_tma) stage_residual();
      int issued = pre;
      bool ok = true;
      // Stage, phase and A coordinates advance incrementally: this thread's
      // own instruction latency is on the mainloop's critical path.
      int st = pre == nst ? 0 : pre;
      uint32_t ph = pre == nst ? 1u : 0u;
      int k = (kb0 + pre) * C::BK;
      int kx = k % s.a_kwrap, ky = k / s.a_kwrap;
      for (int i = pre; i < nkl; ++i) {
        if (!mbar_wait(&empty[st], ph ^ 1)) {
          atomicOr(err, kErrWaitProducer);
          ok = false;
          break;
        }
        uint8_t* sa = smem + st * C::STAGE;
        mbar_arrive_expect_tx(&full[st], C::STAGE);
        tma_load_3d(sa, &tmA, &full[st], kx, m0 + ky, bzb);
        tma_load_2d(sa + C::A_BYTES, &tmB, &full[st], k, n0);
        issued = i + 1;
        k += C::BK;
        kx += C::BK;
        if (kx == s.a_kwrap) {
          kx = 0;
          ++ky;
        }
        if (++st == nst) {
          st = 0;
          ph ^= 1u;
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA exits.
        for (int i = (issued > nst ? issued - nst : 0); i < issued; ++i)
          mbar_wait(&full[i % nst], (i / nst) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, BN);
      // The issuing thread's own instruction latency paces the MMAs, so the
      // shared-memory descriptors are built once: stage st, K step kk is the
      // stage-0 descriptor with (st * STAGE + kk * 32) / 16 added to its
      // 14-bit start-address field (addresses stay below 256 KB: no carry).
      const uint64_t dA0 = desc_sw128(smem_u32(smem));
      const uint64_t dB0 = desc_sw128(smem_u32(smem) + C::A_BYTES);
      bool ok = true;
      int st = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nkl; ++i) {
        if (!mbar_wait(&full[st], ph)) {
          atomicOr(err, kErrWaitMma);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t off = static_cast<uint64_t>(st * (C::STAGE >> 4));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16(tmem, dA0 + off + 2 * kk, dB0 + off + 2 * kk, idesc, (i | kk) != 0 ? 1u : 0u);
        umma_commit(&empty[st]);
        if (++st == nst) {
          st = 0;
          ph ^= 1u;
        }
      }
      if (ok) umma_commit(accf);
    }
  }

  const bool epi = warp >= 2;
  const int et = threadIdx.x - 64;   // 0..255 for the epilogue warps
  const int q = warp & 3;            // TMEM lane quarter this warp may access
  const int half = (warp - 2) >> 2;  // which half of the columns
  const int r = q * 32 + lane;       // tile row of this thread in pass 1
  const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
  const int region = e.qkv_d > 0 ? n0 / e.qkv_d : -1;
  const bool vec = vec_ok != 0;
  const int ln_mode = e.ln_cfg & 255;
  bool ok = true;
  if (epi) {
    for (int i = et; i < BN; i += kEpiThreads) bias_s[i] = (e.bias && n0 + i < s.N) ? e.bias[n0 + i] : 0.f;
    if (ln_mode == 1) {
      for (int i = et; i < BN; i += kEpiThreads) vec_s[i] = n0 + i < s.N ? e.ln_vec[n0 + i] : 0.f;
    } else if (ln_mode == 2 || ln_mode == 3) {
      for (int i = et; i < BN; i += kEpiThreads) {
        vec_s[i] = n0 + i < s.N ? e.ln_vec[n0 + i] : 0.f;
        vec_s[BN + i] = n0 + i < s.N ? e.ln_vec[s.N + n0 + i] : 0.f;
      }
    }
    if (ln_mode == 1 || ln_mode == 2) {
      // Row statistics from the partial sums the producing GEMM stored (it is
      // a previous kernel: wait for it here, while the mainloop runs), added
      // in partial order: rowln_s[row] = (rstd, -mean * rstd).  The width is
      // the A row (mode 1) or the output row (mode 2).
      pdl_wait();
      if (et < C::BM) {
        const int grow = m0 + et;
        float2 f = make_float2(1.f, 0.f);
        if (grow < s.M) {
          // loads issued eight at a time (independent L2 reads), added in
          // partial order
          const int parts = e.ln_cfg >> 8;
          float s1 = 0.f, s2 = 0.f;
          for (int p0 = 0; p0 < parts; p0 += 8) {
            float2 t[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              t[k] = p0 + k < parts ? e.ln_in[static_cast<int64_t>(p0 + k) * s.M + grow] : make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              s1 += t[k].x;
              s2 += t[k].y;
            }
          }
          const float inv = 1.f / static_cast<float>(ln_mode == 1 ? s.K : s.N);
          const float mean = s1 * inv;
          const float rstd = rsqrtf(fmaxf(fmaf(s2, inv, -mean * mean), 0.f) + e.ln_eps);
          f = make_float2(rstd, -mean * rstd);
        }
        rowln_s[et] = f;
      }
    }
    ok = __all_sync(0xffffffffu, mbar_wait(accf, 0));
    if (!ok && lane == 0) atomicOr(err, kErrWaitEpilogue);
    if (res_tma) {  // waited for even after a failure: no copy may land after the CTA leaves
      const bool rok = __all_sync(0xffffffffu, mbar_wait(res_bar, 0));
      if (!rok && lane == 0) atomicOr(err, kErrWaitEpilogue);
      ok = ok && rok;
    }
    tc_fence_after();
  }
  // The LayerNorm factors (rstd, -mean * rstd) of tile row lrow.
  auto row_lnr = [&](int lrow) -> float2 { return ln_mode != 0 ? rowln_s[lrow] : make_float2(1.f, 0.f); };
  // Modes 0 and 2 with partial row sums to store: each epilogue warp takes
  // whole rows (lr0 + lr, lr < nrows, tile rows r0 + lr) and its lanes the
  // rows' 16-byte chunks, so that the sums of each 32-column group (8 chunks,
  // 8 neighbouring lanes) reduce inside the warp in a fixed order; they go to
  // partial (n0 + col) / 32, as in every form.  fetch4(lr, j) gives chunk j of
  // the row's fp32 sums.
  auto finish_rows_stats = [&](int r0, int nrows, void* outp, int ocol0, auto&& fetch4) {
    constexpr int RC = C::ROW_CHUNKS;
    constexpr int RPW = RC >= 32 ? 1 : 32 / RC;  // rows per warp pass
    constexpr int JSTEP = RC >= 32 ? 32 : RC;
    constexpr int NJ = RC >= 32 ? RC / 32 : 1;   // chunks per lane and row
    const int ew = et >> 5;
    const int sub = RC >= 32 ? 0 : lane / RC;
    const int j0 = RC >= 32 ? lane : lane % RC;
#pragma unroll 1
    for (int lb = ew * RPW; lb < nrows; lb += (kEpiThreads / 32) * RPW) {
      const int lr = lb + sub;
      const int grow = m0 + r0 + lr;
      const bool live = lr < nrows && grow < s.M;
      float p1[NJ], p2[NJ];
#pragma unroll
      for (int t = 0; t < NJ; ++t) p1[t] = p2[t] = 0.f;
      if (live) {
        const float2 lnr = row_lnr(r0 + lr);
#pragma unroll
        for (int t = 0; t < NJ; ++t) {
          const int j = j0 + t * JSTEP;
          const int col = n0 + 4 * j;
          if (col >= s.N) continue;
          const int nv = min(4, s.N - col);
          const float4 v = fetch4(lr, j);
          float x[4] = {v.x, v.y, v.z, v.w};
          finish4(x, bias_s, vec_s, BN, lnr, 4 * j, grow, col, nv, bzb, e, outp, ocol0, vec,
                  res_tma ? res_s : nullptr, r0 + lr);
          for (int i = 0; i < nv; ++i) {
            p1[t] += x[i];
            p2[t] = fmaf(x[i], x[i], p2[t]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NJ; ++t) {
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
          p1[t] += __shfl_xor_sync(0xffffffffu, p1[t], o);
          p2[t] += __shfl_xor_sync(0xffffffffu, p2[t], o);
        }
      }
      if (live && (j0 & 7) == 0) {
#pragma unroll
        for (int t = 0; t < NJ; ++t) {
          const int col = n0 + 4 * (j0 + t * JSTEP);
          if (col < s.N) e.ln_out[static_cast<int64_t>(col >> 5) * s.M + grow] = make_float2(p1[t], p2[t]);
        }
      }
    }
  };

  if (mode == 1 && region == 2) {
    // ------------------------------------------- direct, V^T of fused QKV
    // Each warp stages its 32 time steps x 32 dims boxes transposed
    // ([dim][time], 64-byte rows, 64-byte swizzle) and stores them with a TMA
    // tensor store on V^T when its rows lie in one clip at an 8-aligned time
    // offset (always at batch 1); otherwise it scatters from registers, each
    // store instruction covering 32 consecutive time steps of one dim.
    if (epi) {
      named_barrier_sync(1, kEpiThreads);  // bias staged
      const int grow = m0 + r;
      const int rfirst = m0 + q * 32;
      const int clip0 = rfirst / e.t_len;
      const int t_first = rfirst - clip0 * e.t_len;
      const int rlast = min(rfirst + 31, s.M - 1);
      const bool boxed = (rlast / e.t_len == clip0) && (t_first % 8 == 0);
      const int clip = grow / e.t_len;
      const int t = grow - clip * e.t_len;
      uint8_t* stage = smem + (warp - 2) * (BN / 2 / 32) * 4096;
      int nbox = 0;
      const float2 lnr = row_lnr(r);
#pragma unroll 1
      for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 32) {
        float v[32];
        if (ok) tmem_ld32(trow + c, v);
        if (ln_mode == 1) ln1_cols<32>(v, vec_s + c, lnr);
        add_cols<32>(v, bias_s + c);
        act_inplace<32>(v, e.act);
        const int cc = n0 + c - 2 * e.qkv_d;  // column within V: head * 64 + dim
        if (boxed) {
          uint8_t* box = stage + nbox * 4096;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            *reinterpret_cast<__half*>(box + i * 64 + ((((lane >> 3) ^ ((i >> 1) & 3))) << 4) + (lane & 7) * 2) =
                __float2half_rn(v[i]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && ok) tma_store_2d(&tmV, box, t_first, (clip0 * e.n_heads + (cc >> 6)) * 64 + (cc & 63));
          ++nbox;
        } else if (ok && grow < s.M) {
          __half* dst = static_cast<__half*>(e.vt) +
                        (static_cast<int64_t>(clip * e.n_heads + (cc >> 6)) * 64 + (cc & 63)) * e.t_pad + t;
#pragma unroll
          for (int i = 0; i < 32; ++i) dst[static_cast<int64_t>(i) * e.t_pad] = __float2half_rn(v[i]);
        }
      }
      // The staging boxes must stay valid until the stores have read them;
      // the grid boundary makes the global writes visible to the next kernel.
      if (lane == 0) {
        bulk_commit_group();
        bulk_wait_read_all();
      }
    }
    tc_fence_before();
    __syncthreads();
  } else if (mode == 1 || (SPLIT && (mode == 3 || mode == 4))) {
    // ------------------------------------------------------------- direct
    // mode 3 = split-K through L2, finished by the last arrival: the S CTAs
    // of a tile (grid z, no cluster) each TMA-store their fp32 partial boxes
    // to their plane of the scratch (map in tmV's slot), then take a ticket
    // (one counter per tile, at e.out_k); the CTA that arrives last TMA-loads
    // the other planes' boxes of its rows (into the drained operand ring), adds
    // the partials in split order 0..S-1 (deterministic: its own from TMEM in
    // its place) and finishes as in the direct form; it resets the counter.
    // No CTA waits for another: the others are done once their partial and
    // ticket are out.
    //
    // mode 4 = split-K through the cluster (grid z, cluster of S along z),
    // each CTA finishing a group of columns: the tile's columns form S groups
    // of W = BN / S (a multiple of 64); cluster CTA k, which also computed K
    // split k, finishes group k.  After a cluster barrier (every ring is
    // drained) each warp writes its rows of the other groups' columns, fp32,
    // into the owners' shared memory (slot of this sender, 4 KB boxes of 32
    // rows x 32 columns); after a second barrier each owner adds the S partials
    // in split order 0..S-1 (its own from TMEM in its place) and finishes its
    // columns as in the direct form, every epilogue warp on W / 2 of them.
    constexpr int kChunks = BN / 2 / 32;  // 32-column boxes per warp
    const bool m3 = SPLIT && mode == 3;
    const bool m4 = SPLIT && mode == 4;
    bool owner = true;
    const int gw = m4 ? BN / S : BN;  // width of the column group this CTA finishes
    const int kc4 = gw / 64;          // boxes per warp in mode 4
    // this warp's columns of the tile in the finishing loop
    const int cbeg = (m4 ? split * gw : 0) + half * (gw / 2);
    const int cend = cbeg + gw / 2;
    // Staging of the boxes of the other splits for warp w (0..7), split slot
    // pi (0..S-2): mode 3 after the eight warps' own output staging; mode 4 at
    // the start of the ring, the output staging after it.
    auto peer_region = [&](int pi) -> uint8_t* {
      if (m4) return smem + ((pi * 8 + (warp - 2)) * kc4) * 4096;
      return smem + (8 * kChunks + ((warp - 2) * (S - 1) + pi) * kChunks) * 4096;
    };
    if (m4) {
      cluster_sync();  // every accumulator of the cluster is final: all rings are free
      if (epi && ok) {
#pragma unroll 1
        for (int g = 0; g < S; ++g) {
          if (g == split) continue;
          const int si = split < g ? split : split - 1;  // this CTA's slot at owner g
#pragma unroll 1
          for (int cb = 0; cb < kc4; ++cb) {
            float v[32];
            tmem_ld32(trow + g * gw + half * (gw / 2) + cb * 32, v);
            const uint32_t dst =
                mapa_shared(smem_u32(smem) + static_cast<uint32_t>(((si * 8 + (warp - 2)) * kc4 + cb) * 4096 + lane * 128),
                            static_cast<uint32_t>(g));
#pragma unroll
            for (int k = 0; k < 8; ++k)
              st_dsmem_f4(dst + ((k ^ (lane & 7)) << 4), make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]));
          }
        }
      }
      tc_fence_before();
      cluster_sync();  // every partial has landed in its owner's shared memory
      tc_fence_after();
    }
    if (m3) {
      int* tickets = static_cast<int*>(e.out_k);
      const int tile = static_cast<int>(blockIdx.y) * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
      int* last_s = reinterpret_cast<int*>(tmem_slot + 1);
      if (epi && ok) {
        uint8_t* stg = smem + (warp - 2) * kChunks * 4096;
#pragma unroll 1
        for (int cb = 0; cb < kChunks; ++cb) {
          const int c = half * (BN / 2) + cb * 32;
          float v[32];
          tmem_ld32(trow + c, v);
          uint8_t* box = stg + cb * 4096;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<float4*>(box + lane * 128 + ((k ^ (lane & 7)) << 4)) =
                make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) tma_store_3d(&tmV, box, n0 + c, m0 + q * 32, split);
        }
        if (lane == 0) {
          bulk_commit_group();
          bulk_wait_all();  // the partial is in global memory
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
      }
      if (epi) {
        __threadfence();
        named_barrier_sync(2, kEpiThreads);  // every box of this CTA is out
        if (et == 0) *last_s = atomicAdd(&tickets[tile], 1) == S - 1 ? 1 : 0;
        named_barrier_sync(2, kEpiThreads);
        owner = *last_s != 0;
      }
      if (epi && owner) {
        // the other splits' partials are complete: load this warp's boxes of them
        __threadfence();
        asm volatile("fence.proxy.async.global;" ::: "memory");
        if (ok && lane == 0) {
          mbar_arrive_expect_tx(&peer_bar[warp - 2], static_cast<uint32_t>((S - 1) * kChunks * 4096));
          int pi = 0;
          for (int k = 0; k < S; ++k) {
            if (k == split) continue;
            uint8_t* dst = peer_region(pi);
            for (int cb = 0; cb < kChunks; ++cb)
              tma_load_3d(dst + cb * 4096, &tmV, &peer_bar[warp - 2], n0 + half * (BN / 2) + cb * 32, m0 + q * 32, k);
            ++pi;
          }
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&peer_bar[warp - 2], 0));
        if (!ok && lane == 0) atomicOr(err, kErrWaitEpilogue);
        if (et == 0) tickets[tile] = 0;  // ready for the next launch
      }
    }
    if (ln3_cluster) {
      // LayerNorm of each output row over all N columns, held by the CY =
      // gridDim.y CTAs of this cluster (BN each), applied to acc + bias before
      // the activation.  Each thread takes (count, mean, centred sum of
      // squares) of its row's half tile (two passes over TMEM), and the parts
      // combine by Chan's formula in a fixed order: the two halves in shared
      // memory, then one slot per cluster CTA through distributed shared
      // memory (every CTA writes its row parts into every CTA's slot).
      float4* half_s = reinterpret_cast<float4*>(smem + C::LN3_OFF);      // [2][128]
      float4* slot_s = half_s + 2 * 128;                                 // [CY][128]
      const int cy = static_cast<int>(gridDim.y);
      const uint32_t crank = cluster_ctarank();
      cluster_wait();  // every CTA of the cluster is running
      auto chan = [](float4 a, float4 b) -> float4 {
        const float n = a.x + b.x;
        if (n == 0.f) return a;
        const float d = b.y - a.y;
        return make_float4(n, a.y + d * (b.x / n), a.z + b.z + d * d * (a.x * b.x / n), 0.f);
      };
      if (epi) {
        named_barrier_sync(1, kEpiThreads);  // bias staged
        float cnt = 0.f, sum = 0.f;
#pragma unroll 1
        for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 32) {
          float v[32];
          if (ok) tmem_ld32(trow + c, v);
          add_cols<32>(v, bias_s + c);
          const int nv = min(32, s.N - (n0 + c));
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nv) sum += v[i];
          cnt += static_cast<float>(max(nv, 0));
        }
        const float mu = cnt > 0.f ? sum / cnt : 0.f;
        float m2 = 0.f;
#pragma unroll 1
        for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += 32) {
          float v[32];
          if (ok) tmem_ld32(trow + c, v);
          add_cols<32>(v, bias_s + c);
          const int nv = min(32, s.N - (n0 + c));
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < nv) {
              const float dv = v[i] - mu;
              m2 = fmaf(dv, dv, m2);
            }
        }
        half_s[half * 128 + r] = make_float4(cnt, mu, m2, 0.f);
        named_barrier_sync(1, kEpiThreads);
        if (half == 0) {
          const float4 part = chan(half_s[r], half_s[128 + r]);
          const uint32_t dst = smem_u32(slot_s + crank * 128 + r);
          for (int p = 0; p < cy; ++p)
            st_dsmem_f4(mapa_shared(dst, static_cast<uint32_t>(p)), part);
        }
      }
      cluster_sync();  // every CTA's row parts are in every CTA's slots
      if (epi) {
        if (half == 0) {
          float4 tot = slot_s[r];
          for (int p = 1; p < cy; ++p) tot = chan(tot, slot_s[p * 128 + r]);
          const float var = tot.x > 0.f ? tot.z / tot.x : 0.f;
          const float rstd = rsqrtf(var + e.ln_eps);
          rowln_s[r] = make_float2(rstd, -tot.y * rstd);
        }
        named_barrier_sync(1, kEpiThreads);
      }
    }
    if (epi && owner) {
      if (mode == 1 && !ln3_cluster) named_barrier_sync(1, kEpiThreads);  // bias staged (mode 3: the ticket barriers)
      const int grow = m0 + r;
      void* outp = region == 1 ? e.out_k : e.out;
      const int ocol0 = region > 0 ? region * e.qkv_d : 0;
      const CUtensorMap* om = region == 1 ? &tmO2 : &tmO;
      // Staging: this warp's boxes of 32 rows x 32 columns, 4 KB apart.
      uint8_t* stage = smem + ((m4 ? (S - 1) * 8 * kc4 : 0) + (warp - 2) * ((cend - cbeg) / 32)) * 4096;
      int nbox = 0;
      const float2 lnr = row_lnr(r);
#pragma unroll 1
      for (int c = cbeg; c < cend; c += 32) {
        float v[32];
        if (ok) tmem_ld32(trow + c, v);
        if ((m3 || m4) && ok) {
          // partials in split order 0..S-1, this CTA's own (TMEM) in its place
          const int cb = (c - cbeg) / 32;
          float acc[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = 0.f;
          int pi = 0;
          for (int k = 0; k < S; ++k) {
            if (k == split) {
#pragma unroll
              for (int i = 0; i < 32; ++i) acc[i] += v[i];
              continue;
            }
            const uint8_t* src = peer_region(pi) + cb * 4096;
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4) {
              const float4 pv = *reinterpret_cast<const float4*>(src + lane * 128 + ((k4 ^ (lane & 7)) << 4));
              acc[4 * k4] += pv.x; acc[4 * k4 + 1] += pv.y; acc[4 * k4 + 2] += pv.z; acc[4 * k4 + 3] += pv.w;
            }
            ++pi;
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = acc[i];
        }
        if (ln_mode == 1) ln1_cols<32>(v, vec_s + c, lnr);
        add_cols<32>(v, bias_s + c);
        if (ln3_cluster) {  // (v - mean) * rstd * gamma + beta (cluster instantiation only)
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 g = *reinterpret_cast<const float4*>(vec_s + c + i);
            const float4 b = *reinterpret_cast<const float4*>(vec_s + BN + c + i);
            v[i] = fmaf(fmaf(v[i], lnr.x, lnr.y), g.x, b.x);
            v[i + 1] = fmaf(fmaf(v[i + 1], lnr.x, lnr.y), g.y, b.y);
            v[i + 2] = fmaf(fmaf(v[i + 2], lnr.x, lnr.y), g.z, b.z);
            v[i + 3] = fmaf(fmaf(v[i + 3], lnr.x, lnr.y), g.w, b.w);
          }
        }
        act_inplace<32>(v, e.act);
        const int col = n0 + c;
        const int nv = min(32, s.N - col);
        if (e.residual && grow < s.M) {
          const int64_t roff =
              static_cast<int64_t>(bzb) * e.res_batch_stride + static_cast<int64_t>(grow) * e.ldr + col;
          float f[32];
          if (e.res_f32) {
            const float* rp = static_cast<const float*>(e.residual) + roff;
            if (nv == 32) {
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                const float4 rv = *reinterpret_cast<const float4*>(rp + i);
                f[i] = rv.x;
                f[i + 1] = rv.y;
                f[i + 2] = rv.z;
                f[i + 3] = rv.w;
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) f[i] = i < nv ? rp[i] : 0.f;
            }
          } else {
            const __half* rp = static_cast<const __half*>(e.residual) + roff;
            // staged: this row's 64 bytes of the column box c / 32 (zeros past N)
            const uint8_t* rb = res_s + (c >> 5) * 8192 + r * 64;
            if (res_tma || nv == 32) {
#pragma unroll
              for (int i = 0; i < 32; i += 8) {
                const uint4 u = res_tma ? *reinterpret_cast<const uint4*>(rb + (((i >> 3) ^ ((r >> 1) & 3)) << 4))
                                        : *reinterpret_cast<const uint4*>(rp + i);
                const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float2 t = __half22float2(h[k]);
                  f[i + 2 * k] = t.x;
                  f[i + 2 * k + 1] = t.y;
                }
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) f[i] = i < nv ? __half2float(rp[i]) : 0.f;
            }
          }
          add_residual<32>(v, f, ln_mode, vec_s + c, BN, lnr);
        }
        if (e.ln_out) {  // this row's partial sums over these 32 columns
          float st1 = 0.f, st2 = 0.f;
          if (nv == 32) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              st1 += v[i];
              st2 = fmaf(v[i], v[i], st2);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < nv) {
                st1 += v[i];
                st2 = fmaf(v[i], v[i], st2);
              }
          }
          if (ok && grow < s.M && nv > 0) e.ln_out[static_cast<int64_t>(col >> 5) * s.M + grow] = make_float2(st1, st2);
        }
        uint8_t* box = stage + nbox * 4096;
        if (e.out_f32) {
          // 128-byte rows, 128-byte swizzle: chunk k of row lane at k ^ (lane & 7)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<float4*>(box + lane * 128 + ((k ^ (lane & 7)) << 4)) =
                make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        } else {
          // 64-byte rows, 64-byte swizzle: chunk k of row lane at k ^ ((lane >> 1) & 3)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            *reinterpret_cast<uint4*>(box + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(pack_h2(v[8 * k], v[8 * k + 1]), pack_h2(v[8 * k + 2], v[8 * k + 3]),
                           pack_h2(v[8 * k + 4], v[8 * k + 5]), pack_h2(v[8 * k + 6], v[8 * k + 7]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok && col < s.N) tma_store_3d(om, box, col - ocol0, m0 + q * 32, bzb);
        ++nbox;
      }
      if (lane == 0) {  // as above: wait until the boxes have been read
        bulk_commit_group();
        bulk_wait_read_all();
      }
      (void)outp;
    }
    tc_fence_before();
    __syncthreads();
  } else if (SPLIT && mode == 2) {
    // ------------------------------------------------------------ split-K
    const int rows_max = (C::BM + S - 1) / S;
    const uint32_t slot_bytes = static_cast<uint32_t>(rows_max) * C::ROW_CHUNKS * 16;
    const int rank = static_cast<int>(cluster_ctarank());
    cluster_sync();  // every accumulator of the cluster is final: all rings are free
    if (epi && ok) {
      // Rows [o*128/S, (o+1)*128/S) belong to cluster CTA o.
      const int owner = ((r + 1) * S + C::BM - 1) / C::BM - 1;
      const int lrow = r - owner * C::BM / S;
      const uint32_t dst0 = mapa_shared(smem_u32(smem) + rank * slot_bytes, owner);
#pragma unroll 1
      for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += C::CHUNK) {
        float v[32];
        if (C::CHUNK == 32) {
          tmem_ld32(trow + c, v);
        } else {
          float w[16];
          tmem_ld16(trow + c, w);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = w[i];
        }
#pragma unroll
        for (int i = 0; i < C::CHUNK; i += 4)
          st_dsmem_f4(dst0 + swz_off(C::ROW_CHUNKS, lrow, (c + i) >> 2), make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]));
      }
    }
    tc_fence_before();
    cluster_sync();  // every partial has landed in its owner's shared memory
    if (epi && ok) {
      const int r0 = rank * C::BM / S;
      const int nrows = (rank + 1) * C::BM / S - r0;
      auto fetch = [&](int lr, int j) -> float4 {
        float4 a = *reinterpret_cast<const float4*>(smem + swz_off(C::ROW_CHUNKS, lr, j));
        for (int p = 1; p < S; ++p) {
          const float4 b = *reinterpret_cast<const float4*>(smem + p * slot_bytes + swz_off(C::ROW_CHUNKS, lr, j));
          a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        return a;
      };
      if (region == 2) {
        const int total = nrows * C::ROW_CHUNKS;
#pragma unroll 1
        for (int idx = et; idx < total; idx += kEpiThreads) {
          const int j = idx / nrows;
          const int lr = idx - j * nrows;
          const int grow = m0 + r0 + lr;
          const int col = n0 + 4 * j;
          if (grow >= s.M || col >= s.N) continue;
          const float4 v = fetch(lr, j);
          float x[4] = {v.x, v.y, v.z, v.w};
          if (ln_mode == 1) ln1_cols<4>(x, vec_s + 4 * j, row_lnr(r0 + lr));
          add_cols<4>(x, bias_s + 4 * j);
          act_inplace<4>(x, e.act);
          const int cc = col - 2 * e.qkv_d;
          const int clip = grow / e.t_len;
          const int t = grow - clip * e.t_len;
          __half* dst = static_cast<__half*>(e.vt) +
                        (static_cast<int64_t>(clip * e.n_heads + (cc >> 6)) * 64 + (cc & 63)) * e.t_pad + t;
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[static_cast<int64_t>(i) * e.t_pad] = __float2half_rn(x[i]);
        }
      } else {
        // Every partial, this CTA's own included, is in shared memory, so any
        // warp can finish any row: lane = row (band rows 32 g .. 32 g + 31,
        // g = epilogue warp / 4), and the warp's 32-column chunks are
        // (epilogue warp % 4) + 4 k.  The direct form's chunk arithmetic, the
        // partial sums in split order 0..S-1, 16-byte stores from registers.
        void* outp = region == 1 ? e.out_k : e.out;
        const int ocol0 = region > 0 ? region * e.qkv_d : 0;
        const int ew = warp - 2;
        const int lr = (ew >> 2) * 32 + lane;
        const int rt = r0 + lr;  // tile row
        const int grow = m0 + rt;
        const bool live = lr < nrows && grow < s.M;
        const float2 lnr = live ? row_lnr(rt) : make_float2(1.f, 0.f);
        const bool vec16 = vec && ((e.ldo * (e.out_f32 ? 4 : 2)) % 16 == 0);
#pragma unroll 1
        for (int cb = ew & 3; cb < BN / 32 && (ew >> 2) * 32 < nrows; cb += 4) {
          const int c = cb * 32;
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
          if (live) {
            for (int p = 0; p < S; ++p) {
              const uint8_t* src = smem + p * slot_bytes;
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const float4 pv = *reinterpret_cast<const float4*>(src + swz_off(C::ROW_CHUNKS, lr, (c >> 2) + k));
                v[4 * k] += pv.x;
                v[4 * k + 1] += pv.y;
                v[4 * k + 2] += pv.z;
                v[4 * k + 3] += pv.w;
              }
            }
          }
          if (ln_mode == 1) ln1_cols<32>(v, vec_s + c, lnr);
          add_cols<32>(v, bias_s + c);
          act_inplace<32>(v, e.act);
          const int col = n0 + c;
          const int nv = min(32, s.N - col);
          if (!live || nv <= 0) continue;
          if (e.residual) {
            const int64_t roff =
                static_cast<int64_t>(bzb) * e.res_batch_stride + static_cast<int64_t>(grow) * e.ldr + col;
            float f[32];
            if (res_tma) {
              const uint8_t* rb = res_s + cb * 8192 + rt * 64;
#pragma unroll
              for (int i = 0; i < 32; i += 8) {
                const uint4 u = *reinterpret_cast<const uint4*>(rb + (((i >> 3) ^ ((rt >> 1) & 3)) << 4));
                const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float2 t = __half22float2(h[k]);
                  f[i + 2 * k] = t.x;
                  f[i + 2 * k + 1] = t.y;
                }
              }
            } else if (e.res_f32) {
              const float* rp = static_cast<const float*>(e.residual) + roff;
#pragma unroll
              for (int i = 0; i < 32; ++i) f[i] = i < nv ? rp[i] : 0.f;
            } else {
              const __half* rp = static_cast<const __half*>(e.residual) + roff;
#pragma unroll
              for (int i = 0; i < 32; ++i) f[i] = i < nv ? __half2float(rp[i]) : 0.f;
            }
            add_residual<32>(v, f, ln_mode, vec_s + c, BN, lnr);
          }
          if (e.ln_out) {
            float st1 = 0.f, st2 = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < nv) {
                st1 += v[i];
                st2 = fmaf(v[i], v[i], st2);
              }
            e.ln_out[static_cast<int64_t>(col >> 5) * s.M + grow] = make_float2(st1, st2);
          }
          const int64_t ooff =
              static_cast<int64_t>(bzb) * e.out_batch_stride + static_cast<int64_t>(grow) * e.ldo + (col - ocol0);
          if (e.out_f32) {
            float* op = static_cast<float*>(outp) + ooff;
            if (vec16 && nv == 32) {
#pragma unroll
              for (int k = 0; k < 32; k += 4)
                *reinterpret_cast<float4*>(op + k) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (k < nv) op[k] = v[k];
            }
          } else {
            __half* op = static_cast<__half*>(outp) + ooff;
            if (vec16 && nv == 32) {
#pragma unroll
              for (int k = 0; k < 32; k += 8)
                *reinterpret_cast<uint4*>(op + k) = make_uint4(pack_h2(v[k], v[k + 1]), pack_h2(v[k + 2], v[k + 3]),
                                                               pack_h2(v[k + 4], v[k + 5]), pack_h2(v[k + 6], v[k + 7]));
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (k < nv) op[k] = __float2half_rn(v[k]);
            }
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  } else {
    // ------------------------------------------------------------ generic
    uint8_t* park = smem;
    if (epi && ok) {
#pragma unroll 1
      for (int c = half * (BN / 2); c < (half + 1) * (BN / 2); c += C::CHUNK) {
        float v[32];
        if (C::CHUNK == 32) {
          tmem_ld32(trow + c, v);
        } else {
          float w[16];
          tmem_ld16(trow + c, w);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = w[i];
        }
#pragma unroll
        for (int i = 0; i < C::CHUNK; i += 4)
          *reinterpret_cast<float4*>(park + swz_off(C::ROW_CHUNKS, r, (c + i) >> 2)) =
              make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      }
    }
    tc_fence_before();
    __syncthreads();
    if (epi && ok) {
      const int total = C::BM * C::ROW_CHUNKS;
      if (region == 2) {
#pragma unroll 1
        for (int idx = et; idx < total; idx += kEpiThreads) {
          const int j = idx / C::BM;
          const int rr = idx - j * C::BM;
          const int grow = m0 + rr;
          const int col = n0 + 4 * j;
          if (grow >= s.M || col >= s.N) continue;
          const float4 v = *reinterpret_cast<const float4*>(park + swz_off(C::ROW_CHUNKS, rr, j));
          float x[4] = {v.x, v.y, v.z, v.w};
          if (ln_mode == 1) ln1_cols<4>(x, vec_s + 4 * j, rowln_s[rr]);
          add_cols<4>(x, bias_s + 4 * j);
          act_inplace<4>(x, e.act);
          const int cc = col - 2 * e.qkv_d;
          const int clip = grow / e.t_len;
          const int t = grow - clip * e.t_len;
          __half* dst = static_cast<__half*>(e.vt) +
                        (static_cast<int64_t>(clip * e.n_heads + (cc >> 6)) * 64 + (cc & 63)) * e.t_pad + t;
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[static_cast<int64_t>(i) * e.t_pad] = __float2half_rn(x[i]);
        }
      } else {
        void* outp = region == 1 ? e.out_k : e.out;
        const int ocol0 = region > 0 ? region * e.qkv_d : 0;
        if (e.ln_out)
          finish_rows_stats(0, C::BM, outp, ocol0, [&](int rr, int j) -> float4 {
            return *reinterpret_cast<const float4*>(park + swz_off(C::ROW_CHUNKS, rr, j));
          });
#pragma unroll 2
        for (int idx = et; idx < (e.ln_out ? 0 : total); idx += kEpiThreads) {
          const int rr = idx / C::ROW_CHUNKS;
          const int j = idx - rr * C::ROW_CHUNKS;
          const int grow = m0 + rr;
          const int col = n0 + 4 * j;
          if (grow >= s.M || col >= s.N) continue;
          const float4 v = *reinterpret_cast<const float4*>(park + swz_off(C::ROW_CHUNKS, rr, j));
          float x[4] = {v.x, v.y, v.z, v.w};
          finish4(x, bias_s, vec_s, BN, row_lnr(rr), 4 * j, grow, col, min(4, s.N - col), bzb, e, outp, ocol0,
                  vec);
        }
      }
    }
    __syncthreads();
  }

  if (PAIR) {
    // neither CTA of the pair leaves (or frees the pair's TMEM) while the
    // other may still touch its shared memory, barriers or TMEM
    tc_fence_before();
    cluster_sync();
  }
  if (warp == 1) {
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem, C::TMEM_COLS);
    else
      tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- persistent
// Persistent form for GEMMs with more output tiles than SMs: one CTA per SM
// walks the tiles t = blockIdx.x, blockIdx.x + gridDim.x, ... (row tile
// fastest, then column tile, then batch item).  Operand stages flow through
// one ring across tiles, and the accumulator is double-buffered in TMEM: the
// MMA thread fills one buffer while the epilogue warps drain the other, so a
// tile's epilogue runs under the next tile's mainloop.  The epilogue is the
// direct form's arithmetic (folded LayerNorm, bias, activation, residual,
// partial row sums) with plain vector stores from registers (no staging);
// the bias, LN vectors and row factors are reloaded for each tile.
template <int BN>
struct GemmPCfg {
  static constexpr int BM = 128;
  static constexpr int BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int RING_MAX = 200 * 1024;
  static constexpr int STAGES = (RING_MAX / STAGE) > 8 ? 8 : (RING_MAX / STAGE);
  static constexpr int RING = STAGES * STAGE;
  static constexpr int ACC_COLS = BN <= 64 ? 64 : (BN <= 128 ? 128 : 256);  // one accumulator
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int BIAS_OFF = RING;
  static constexpr int VEC_OFF = BIAS_OFF + BN * 4;
  static constexpr int ROWLN_OFF = VEC_OFF + 2 * BN * 4;
  static constexpr int BAR_OFF = ROWLN_OFF + 128 * 8;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static_assert(BN >= 64 && BN % 32 == 0, "persistent tiles are 64..256 wide");
};

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_persist_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmDims s,
                    GemmEpiArgs e, int n_mt, int n_nt, int vec_ok, int* err) {
  using C = GemmPCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* bias_s = reinterpret_cast<float*>(smem + C::BIAS_OFF);
  float* vec_s = reinterpret_cast<float*>(smem + C::VEC_OFF);
  float2* rowln_s = reinterpret_cast<float2*>(smem + C::ROWLN_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;  // [2] accumulator b complete
  uint64_t* tempty = tfull + 2;         // [2] accumulator b drained (one arrival per epilogue warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nk = s.K / C::BK;
  const int n_tiles = n_mt * n_nt * s.batch;
  auto tile_of = [&](int t, int& m0, int& n0, int& bz) {
    const int mt = t % n_mt;
    const int rest = t / n_mt;
    m0 = mt * C::BM;
    n0 = (rest % n_nt) * BN;
    bz = rest / n_nt;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&tfull[0], 1);
    mbar_init(&tfull[1], 1);
    mbar_init(&tempty[0], kEpiThreads / 32);
    mbar_init(&tempty[1], kEpiThreads / 32);
    fence_mbar_init();
    pdl_launch_dependents();
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
      pdl_wait();
      int st = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int m0, n0, bz;
        tile_of(t, m0, n0, bz);
        int kx = 0, ky = 0;  // A coordinates, advanced incrementally
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[st], ph ^ 1)) {
            atomicOr(err, kErrWaitProducer);
            ok = false;
            break;
          }
          uint8_t* sa = smem + st * C::STAGE;
          mbar_arrive_expect_tx(&full[st], C::STAGE);
          tma_load_3d(sa, &tmA, &full[st], kx, m0 + ky, bz);
          tma_load_2d(sa + C::A_BYTES, &tmB, &full[st], kb * C::BK, n0);
          kx += C::BK;
          if (kx == s.a_kwrap) {
            kx = 0;
            ++ky;
          }
          ++issued;
          if (++st == C::STAGES) {
            st = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA exits.
        for (int i = (issued > C::STAGES ? issued - C::STAGES : 0); i < issued; ++i)
          mbar_wait(&full[i % C::STAGES], (i / C::STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, BN);
      const uint64_t dA0 = desc_sw128(smem_u32(smem));
      const uint64_t dB0 = desc_sw128(smem_u32(smem) + C::A_BYTES);
      int st = 0;
      uint32_t ph = 0;
      int i = 0;
      for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
        const int b = i & 1;
        if (!mbar_wait(&tempty[b], ((i >> 1) & 1) ^ 1)) {
          atomicOr(err, kErrWaitMma);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(b * C::ACC_COLS);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[st], ph)) {
            atomicOr(err, kErrWaitMma);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t off = static_cast<uint64_t>(st * (C::STAGE >> 4));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16(d, dA0 + off + 2 * kk, dB0 + off + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&empty[st]);
          if (++st == C::STAGES) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[b]);
      }
    }
  } else {
    const int et = threadIdx.x - 64;
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = q * 32 + lane;
    const int ln_mode = e.ln_cfg & 255;
    const bool vec = vec_ok != 0;
    bool ok = true;
    pdl_wait();  // row partial sums and residuals come from earlier kernels
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      int m0, n0, bz;
      tile_of(t, m0, n0, bz);
      // this tile's column vectors and row factors (the previous tile's
      // readers are past the barrier)
      named_barrier_sync(1, kEpiThreads);
      for (int c = et; c < BN; c += kEpiThreads) {
        const bool in = n0 + c < s.N;
        bias_s[c] = (e.bias && in) ? e.bias[n0 + c] : 0.f;
        if (ln_mode != 0) vec_s[c] = in ? e.ln_vec[n0 + c] : 0.f;
        if (ln_mode == 2) vec_s[BN + c] = in ? e.ln_vec[s.N + n0 + c] : 0.f;
      }
      if (ln_mode != 0 && et < C::BM) {
        const int grow = m0 + et;
        float2 f = make_float2(1.f, 0.f);
        if (grow < s.M) {
          const int parts = e.ln_cfg >> 8;
          float s1 = 0.f, s2 = 0.f;
          for (int p0 = 0; p0 < parts; p0 += 8) {
            float2 tv[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              tv[k] = p0 + k < parts ? e.ln_in[static_cast<int64_t>(p0 + k) * s.M + grow] : make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              s1 += tv[k].x;
              s2 += tv[k].y;
            }
          }
          const float inv = 1.f / static_cast<float>(ln_mode == 1 ? s.K : s.N);
          const float mean = s1 * inv;
          const float rstd = rsqrtf(fmaxf(fmaf(s2, inv, -mean * mean), 0.f) + e.ln_eps);
          f = make_float2(rstd, -mean * rstd);
        }
        rowln_s[et] = f;
      }
      named_barrier_sync(1, kEpiThreads);
      const int b = i & 1;
      if (ok) {
        ok = __all_sync(0xffffffffu, mbar_wait(&tfull[b], (i >> 1) & 1));
        if (!ok && lane == 0) atomicOr(err, kErrWaitEpilogue);
      }
      tc_fence_after();
      const uint32_t tacc = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * C::ACC_COLS);
      const int grow = m0 + r;
      const float2 lnr = ln_mode != 0 ? rowln_s[r] : make_float2(1.f, 0.f);
#pragma unroll 1
      for (int c = half * (BN / 2); c < (half + 1) * (BN / 2) && ok; c += 32) {
        float v[32];
        tmem_ld32(tacc + c, v);
        if (c + 32 >= (half + 1) * (BN / 2)) {
          // the last read of this accumulator: hand it back to the MMA thread
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[b]);
        }
        if (ln_mode == 1) ln1_cols<32>(v, vec_s + c, lnr);
        add_cols<32>(v, bias_s + c);
        act_inplace<32>(v, e.act);
        const int col = n0 + c;
        const int nv = min(32, s.N - col);
        if (grow >= s.M || nv <= 0) continue;
        if (e.residual) {
          const int64_t roff =
              static_cast<int64_t>(bz) * e.res_batch_stride + static_cast<int64_t>(grow) * e.ldr + col;
          float f[32];
          if (e.res_f32) {
            const float* rp = static_cast<const float*>(e.residual) + roff;
            if (vec && nv == 32) {
#pragma unroll
              for (int k = 0; k < 32; k += 4) {
                const float4 rv = *reinterpret_cast<const float4*>(rp + k);
                f[k] = rv.x;
                f[k + 1] = rv.y;
                f[k + 2] = rv.z;
                f[k + 3] = rv.w;
              }
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k) f[k] = k < nv ? rp[k] : 0.f;
            }
          } else {
            const __half* rp = static_cast<const __half*>(e.residual) + roff;
            if (vec && nv == 32) {
#pragma unroll
              for (int k = 0; k < 32; k += 8) {
                const uint4 u = *reinterpret_cast<const uint4*>(rp + k);
                const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const float2 tf = __half22float2(h[j]);
                  f[k + 2 * j] = tf.x;
                  f[k + 2 * j + 1] = tf.y;
                }
              }
            } else {
#pragma unroll
              for (int k = 0; k < 32; ++k) f[k] = k < nv ? __half2float(rp[k]) : 0.f;
            }
          }
          add_residual<32>(v, f, ln_mode, vec_s + c, BN, lnr);
        }
        if (e.ln_out) {
          float st1 = 0.f, st2 = 0.f;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k < nv) {
              st1 += v[k];
              st2 = fmaf(v[k], v[k], st2);
            }
          e.ln_out[static_cast<int64_t>(col >> 5) * s.M + grow] = make_float2(st1, st2);
        }
        const int64_t ooff = static_cast<int64_t>(bz) * e.out_batch_stride + static_cast<int64_t>(grow) * e.ldo + col;
        if (e.out_f32) {
          float* op = static_cast<float*>(e.out) + ooff;
          if (vec && nv == 32) {
#pragma unroll
            for (int k = 0; k < 32; k += 4)
              *reinterpret_cast<float4*>(op + k) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (k < nv) op[k] = v[k];
          }
        } else {
          __half* op = static_cast<__half*>(e.out) + ooff;
          if (vec && nv == 32) {
#pragma unroll
            for (int k = 0; k < 32; k += 8)
              *reinterpret_cast<uint4*>(op + k) = make_uint4(pack_h2(v[k], v[k + 1]), pack_h2(v[k + 2], v[k + 3]),
                                                             pack_h2(v[k + 4], v[k + 5]), pack_h2(v[k + 6], v[k + 7]));
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (k < nv) op[k] = __float2half_rn(v[k]);
          }
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

// Tile width and split-K factor: the candidate whose launch should finish
// first under a simple model of this kernel on B200 (148 SMs):
//  * MMA time per CTA: per 64-deep K block the larger of the MMA time
//    (2*BN cycles for M=128) and the shared-memory operand reads
//    ((16 KB + BN*128 B) at 128 B/cycle), times waves of CTAs;
//  * operand delivery: every CTA streams its A and B blocks from L2, and one
//    SM takes in about 72 B/cycle of TMA traffic whatever the number of SMs
//    streaming (measured on this B200 with a copy-only kernel: 148 SMs
//    together reach ~21 TB/s from L2), so the per-CTA operand bytes give the
//    floor;
//  * fixed costs: set-up, the epilogue (split S ways), the cluster reduction.
int gemm_pick(GemmShape* s, int bn_divides) {
  const int cands[] = {32, 64, 128, 192, 256};
  const int splits[] = {1, 2, 3, 4, 6, 8};
  const long mt = static_cast<long>((s->M + 127) / 128) * s->batch;
  const long nk = s->K / 64;
  int best_bn = 64, best_s = 1;
  double best_t = 1e30;
  for (int bn : cands) {
    if (bn > 32 && s->N <= bn / 2) continue;  // much wider than N: wasted MMA columns
    if (bn_divides > 0 && bn_divides % bn != 0) continue;
    const long tiles = mt * ((s->N + bn - 1) / bn);
    for (int sp : splits) {
      if (sp > 1 && (s->batch != 1 || sp > nk)) continue;
      const long ctas = tiles * sp;
      const long waves = (ctas + 147) / 148;
      const long nkl = (nk + sp - 1) / sp;
      const double per_k = (2.0 * bn > 128.0 + bn) ? 2.0 * bn : 128.0 + bn;
      const double t_mma = waves * nkl * per_k;
      const double t_sm = waves * nkl * (128.0 + bn) * 128.0 / 72.0;
      const double t_max = t_mma > t_sm ? t_mma : t_sm;
      const double t = t_max + 2000.0 + waves * (600.0 + 6.0 * bn / sp) +
                       (sp > 1 ? 800.0 + 150.0 * sp : 0.0);
      if (t < best_t - 1e-9) {
        best_t = t;
        best_bn = bn;
        best_s = sp;
      }
    }
  }
  s->splits = best_s;
  return best_bn;
}

// Whether a staged residual tile leaves at least two ring stages and room in
// front of it for the epilogue's staging of this form: the output boxes
// (mode 1, 8 warps x BN/64 boxes of 4 KB), the cluster partials (mode 2,
// S slots of ceil(128/S) fp32 rows; mode 4, S - 1 slots of 128 rows x BN/S
// columns and the output boxes) or the L2 form's boxes (mode 3).
template <int BN, bool PAIR>
static bool res_stage_fits_cfg(int mode, int splits) {
  using C = GemmCfg<BN, PAIR>;
  if (BN < 64 || BN > 192) return false;
  const int nst = C::STAGES - C::RES_STAGES;
  if (nst < 2) return false;
  const int room = nst * C::STAGE;
  const int chunks = BN / 64;
  if (mode == 1) return 8 * chunks * 4096 <= room;
  if (mode == 2) return splits * ((C::BM + splits - 1) / splits) * (BN / 4) * 16 <= room;
  if (mode == 3) return 8 * splits * chunks * 4096 <= room;
  if (mode == 4) return 8 * BN / 64 * 4096 <= room;  // the S - 1 senders' slots and the output staging
  return false;
}

bool gemm_res_stage_fits(int bn, bool pair, int mode, int splits) {
  switch (bn) {
    case 64: return pair ? res_stage_fits_cfg<64, true>(mode, splits) : res_stage_fits_cfg<64, false>(mode, splits);
    case 128: return pair ? res_stage_fits_cfg<128, true>(mode, splits) : res_stage_fits_cfg<128, false>(mode, splits);
    case 192: return pair ? res_stage_fits_cfg<192, true>(mode, splits) : res_stage_fits_cfg<192, false>(mode, splits);
    default: return false;
  }
}

// The L2 split form's last arrival keeps its own output staging plus the
// other S-1 splits' boxes of its rows in the drained operand ring.
bool gemm_l2_split_fits(int bn, int splits) {
  const int chunks = bn / 2 / 32;
  int ring = 0;
  switch (bn) {
    case 64: ring = GemmCfg<64>::RING; break;
    case 128: ring = GemmCfg<128>::RING; break;
    case 192: ring = GemmCfg<192>::RING; break;
    case 256: ring = GemmCfg<256>::RING; break;
    default: return false;
  }
  return chunks >= 1 && splits >= 2 && 8 * splits * chunks * 4096 <= ring;
}

template <int BN>
static cudaError_t prepare_bn() {
  cudaError_t r = cudaFuncSetAttribute(gemm_tc_kernel<BN, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       GemmCfg<BN>::SMEM);
  if (r == cudaSuccess)
    r = cudaFuncSetAttribute(gemm_tc_kernel<BN, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<BN>::SMEM_LN3);
  if (r == cudaSuccess && BN >= 64)
    r = cudaFuncSetAttribute(gemm_tc_kernel<BN, false, (BN >= 64)>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GemmCfg<BN, (BN >= 64)>::SMEM);
  if constexpr (BN >= 64) {
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(gemm_persist_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               GemmPCfg<BN>::SMEM);
  }
  return r;
}

cudaError_t gemm_prepare() {
  static cudaError_t done = cudaErrorNotReady;
  if (done == cudaSuccess) return done;
  cudaError_t r;
  if ((r = prepare_bn<32>()) != cudaSuccess) return r;
  if ((r = prepare_bn<64>()) != cudaSuccess) return r;
  if ((r = prepare_bn<128>()) != cudaSuccess) return r;
  if ((r = prepare_bn<192>()) != cudaSuccess) return r;
  done = prepare_bn<256>();
  return done;
}

template <int BN>
static cudaError_t launch_bn(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmO,
                             const CUtensorMap& tmO2, const CUtensorMap& tmV, const GemmShape& s,
                             const GemmEpilogue& e, int vec_ok, int mode, int* err, cudaStream_t st) {
  const int S = s.splits;
  const bool pair = s.pair;
  // pairs: 2 CTAs per 256-row tile (grid x even), one cluster per pair
  dim3 grid(pair ? 2 * ((s.M + 255) / 256) : (s.M + 127) / 128, (s.N + BN - 1) / BN, S > 1 ? S : s.batch);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = pair ? GemmCfg<BN, (BN >= 64)>::SMEM
                              : ((e.ln_cfg & 255) == 3 ? GemmCfg<BN>::SMEM_LN3 : GemmCfg<BN>::SMEM);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = pair ? 2 : 1;
  attr[1].val.clusterDim.y = 1;
  // the cluster forms (modes 2 and 4); the L2 form (mode 3) needs no cluster
  const bool cluster_split = S > 1 && ((mode & 15) == 2 || (mode & 15) == 4);
  // row LayerNorm: the column tiles of a row block form one cluster along y
  const bool cluster_ln = (e.ln_cfg & 255) == 3;
  if (cluster_ln) {
    attr[1].val.clusterDim.y = grid.y;
    if (pair || S > 1 || (mode & 15) != 1) return cudaErrorInvalidValue;
  }
  attr[1].val.clusterDim.z = cluster_split ? S : 1;
  cfg.attrs = attr;
  cfg.numAttrs = (cluster_split || pair || cluster_ln) ? 2 : 1;
  const GemmDims sd = s;      // the kernel's parameter block holds only
  GemmEpiArgs ea = e;         // what it reads
  if ((mode & 15) == 3) ea.out_k = e.split_tickets;  // the L2 form's tickets (out_k is a QKV-only field)
  if (pair) {
    if (BN < 64 || S > 1 || (mode & 15) != 1) return cudaErrorInvalidValue;
    return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, false, (BN >= 64)>, tmA, tmB, tmO, tmO2, tmV, sd, ea, vec_ok,
                              mode, err);
  }
  // the cluster instantiation for split-K and for the row LayerNorm
  return (S > 1 || cluster_ln)
             ? cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, true, false>, tmA, tmB, tmO, tmO2, tmV, sd, ea, vec_ok, mode,
                                  err)
             : cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, false, false>, tmA, tmB, tmO, tmO2, tmV, sd, ea, vec_ok, mode,
                                  err);
}

// The persistent form: no split, pair or QKV split; 16-byte vector stores of
// the output rows and loads of the residual rows.
template <int BN>
static cudaError_t launch_persist_bn(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmShape& s,
                                     const GemmEpilogue& e, int* err, cudaStream_t st) {
  static int n_sm = 0;
  if (n_sm == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n_sm <= 0)
      return cudaErrorInvalidValue;
  }
  const int n_mt = (s.M + 127) / 128, n_nt = (s.N + BN - 1) / BN;
  const long tiles = static_cast<long>(n_mt) * n_nt * s.batch;
  if (tiles <= 0 || tiles > (1L << 30)) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles < n_sm ? tiles : n_sm));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = GemmPCfg<BN>::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const GemmDims sd = s;
  const GemmEpiArgs ea = e;
  return cudaLaunchKernelEx(&cfg, gemm_persist_kernel<BN>, tmA, tmB, sd, ea, n_mt, n_nt, 1, err);
}

static cudaError_t launch_persist(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmShape& s, int bn,
                                  const GemmEpilogue& e, int* err, cudaStream_t st) {
  if (s.splits != 1 || s.split_l2 || s.pair || e.qkv_d > 0 || !e.out || (e.ln_cfg & 255) > 2)
    return cudaErrorInvalidValue;
  const int esz_out = e.out_f32 ? 4 : 2;
  const int esz_res = e.res_f32 ? 4 : 2;
  const bool out_ok = reinterpret_cast<uintptr_t>(e.out) % 16 == 0 && (e.ldo * esz_out) % 16 == 0 &&
                      (s.batch == 1 || (e.out_batch_stride * esz_out) % 16 == 0);
  const bool res_ok = e.residual == nullptr ||
                      (reinterpret_cast<uintptr_t>(e.residual) % 16 == 0 && (e.ldr * esz_res) % 16 == 0 &&
                       (s.batch == 1 || (e.res_batch_stride * esz_res) % 16 == 0));
  if (!out_ok || !res_ok) return cudaErrorInvalidValue;
  switch (bn) {
    case 64: return launch_persist_bn<64>(tmA, tmB, s, e, err, st);
    case 128: return launch_persist_bn<128>(tmA, tmB, s, e, err, st);
    case 192: return launch_persist_bn<192>(tmA, tmB, s, e, err, st);
    case 256: return launch_persist_bn<256>(tmA, tmB, s, e, err, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmShape& s, int bn,
                        const GemmEpilogue& e, int* err, cudaStream_t st) {
  if (s.M <= 0 || s.N <= 0 || s.batch <= 0) return cudaSuccess;
  if (s.K <= 0 || s.K % 64 != 0 || s.a_kwrap <= 0 || s.a_kwrap % 64 != 0) return cudaErrorInvalidValue;
  if (s.splits < 1 || s.splits > 8 || s.splits > s.K / 64 || (s.splits > 1 && s.batch != 1))
    return cudaErrorInvalidValue;
  // pairs: no split, tiles at least 64 wide, the direct (TMA-store) epilogue
  if (s.pair && (s.splits != 1 || s.split_l2 || bn < 64)) return cudaErrorInvalidValue;
  if (s.persist) return launch_persist(tmA, tmB, s, bn, e, err, st);
  if (e.qkv_d > 0 && (e.qkv_d % bn != 0 || s.N != 3 * e.qkv_d || e.t_len <= 0)) return cudaErrorInvalidValue;
  // Folded LayerNorm: row statistics come as partial sums indexed by row
  // (one clip batch); the normalised residual must be fp16.
  const int ln_mode = e.ln_cfg & 255;
  if (ln_mode > 3 || ((ln_mode == 1 || ln_mode == 2) && (!e.ln_vec || !e.ln_in || (e.ln_cfg >> 8) < 1 || s.batch != 1)))
    return cudaErrorInvalidValue;
  // Row LayerNorm of the output (ln_mode 3): the N / bn column tiles of a row
  // block form a cluster (at most 8), one CTA per tile, the direct epilogue.
  if (ln_mode == 3 && (!e.ln_vec || s.N % bn != 0 || s.N / bn > 8 || s.splits != 1 || s.split_l2 || s.pair ||
                       s.persist || e.qkv_d > 0 || e.residual || e.ln_out || bn < 64))
    return cudaErrorInvalidValue;
  if (ln_mode == 2 && (!e.residual || e.res_f32)) return cudaErrorInvalidValue;
  if (e.ln_out && (s.batch != 1 || e.qkv_d > 0)) return cudaErrorInvalidValue;
  // Vector loads/stores need 16-byte aligned bases and 4-element-aligned rows.
  const int esz_out = e.out_f32 ? 4 : 2;
  const int esz_res = e.res_f32 ? 4 : 2;
  bool vec = (reinterpret_cast<uintptr_t>(e.out) % 16 == 0) && (e.ldo % 4 == 0) &&
             ((e.out_batch_stride * esz_out) % 16 == 0);
  if (e.residual)
    vec = vec && (reinterpret_cast<uintptr_t>(e.residual) % 16 == 0) && (e.ldr % 4 == 0) &&
          ((e.res_batch_stride * esz_res) % 16 == 0);
  if (e.qkv_d > 0) vec = vec && (reinterpret_cast<uintptr_t>(e.out_k) % 16 == 0);
  // Direct (TMA-store) epilogue: rows must be 16-byte multiples and any
  // residual vector-loadable; tiles at least 64 wide.
  CUtensorMap tmO, tmO2, tmV;
  std::memset(&tmO, 0, sizeof tmO);
  std::memset(&tmO2, 0, sizeof tmO2);
  std::memset(&tmV, 0, sizeof tmV);
  int mode = s.splits > 1 ? 2 : 0;
  // split-K through L2 (mode 3): S = 2..4, the scratch, a ticket per tile, the
  // last arrival's staging in shared memory, and a TMA-storable output
  const int64_t n_tiles = static_cast<int64_t>((s.M + 127) / 128) * ((s.N + bn - 1) / bn);
  const bool l2split = s.split_l2 && s.splits >= 2 && s.splits <= 4 && gemm_l2_split_fits(bn, s.splits) &&
                       e.part_ws && e.split_tickets && n_tiles <= e.ticket_cap && e.qkv_d == 0 &&
                       s.N <= e.ws_ld && e.ws_ld % 4 == 0 && e.ws_rows >= 128L * ((s.M + 127) / 128) &&
                       (reinterpret_cast<uintptr_t>(e.part_ws) % 16) == 0;
  if (s.split_l2 && !l2split) return cudaErrorInvalidValue;
  // split-K through the cluster with column groups (mode 4): groups of a
  // multiple of 64 columns, the direct epilogue's stores
  const bool colsplit = s.splits > 1 && !s.split_l2 && e.qkv_d == 0 && bn % s.splits == 0 &&
                        (bn / s.splits) % 64 == 0;
  const bool tma_ok = (s.splits == 1 || l2split || colsplit) && bn >= 64 && vec && (e.ldo * esz_out) % 16 == 0 &&
                      (e.residual == nullptr || (e.ldr * esz_res) % 16 == 0);
  if (tma_ok) {
    const uint64_t cols = e.qkv_d > 0 ? static_cast<uint64_t>(e.qkv_d) : static_cast<uint64_t>(s.N);
    const uint64_t dims[3] = {cols, static_cast<uint64_t>(s.M), static_cast<uint64_t>(s.batch)};
    const uint64_t bstride = s.batch > 1 ? static_cast<uint64_t>(e.out_batch_stride) * esz_out
                                         : static_cast<uint64_t>(s.M) * e.ldo * esz_out;
    const uint64_t str[2] = {static_cast<uint64_t>(e.ldo) * esz_out, bstride};
    const uint32_t box[3] = {32, 32, 1};
    const int swz = e.out_f32 ? 128 : 64;
    bool built = make_tmap(&tmO, e.out, 3, dims, str, box, esz_out, swz) == cudaSuccess;
    if (built && e.qkv_d > 0) {
      built = make_tmap(&tmO2, e.out_k, 3, dims, str, box, esz_out, swz) == cudaSuccess;
      // V^T [clip][head][64][t_pad]: time innermost, one row per (clip, head, dim)
      const uint64_t vd[2] = {static_cast<uint64_t>(e.t_len),
                              static_cast<uint64_t>(s.M / e.t_len) * e.n_heads * 64};
      const uint64_t vs[1] = {static_cast<uint64_t>(e.t_pad) * 2};
      const uint32_t vb[2] = {32, 32};
      built = built && !e.out_f32 && e.t_pad % 8 == 0 &&
              make_tmap(&tmV, e.vt, 2, vd, vs, vb, 2, 64) == cudaSuccess;
    }
    if (built && l2split) {
      // the scratch planes [S][ws_rows][ws_ld] fp32, 32 x 32 boxes, 128-byte swizzle
      const uint64_t wd[3] = {static_cast<uint64_t>(e.ws_ld), static_cast<uint64_t>(e.ws_rows),
                              static_cast<uint64_t>(s.splits)};
      const uint64_t ws[2] = {static_cast<uint64_t>(e.ws_ld) * 4, static_cast<uint64_t>(e.ws_rows * e.ws_ld) * 4};
      built = make_tmap(&tmV, e.part_ws, 3, wd, ws, box, 4, 128) == cudaSuccess;
    }
    if (built) mode = l2split ? 3 : (colsplit ? 4 : 1);
  }
  if (l2split && mode != 3) return cudaErrorInvalidValue;
  if (s.pair && mode != 1) return cudaErrorInvalidValue;
  if (ln_mode == 3 && mode != 1) return cudaErrorInvalidValue;
  // An fp16 residual is staged in shared memory by TMA while the mainloop
  // runs (boxes of 32 columns x 128 rows, 64-byte swizzle), when the ring's
  // remaining stages still hold the epilogue's own staging.
  if (mode >= 1 && e.residual && !e.res_f32 && e.qkv_d == 0 && (e.ldr * 2) % 16 == 0 &&
      reinterpret_cast<uintptr_t>(e.residual) % 16 == 0 && (s.batch == 1 || (e.res_batch_stride * 2) % 16 == 0) &&
      gemm_res_stage_fits(bn, s.pair, mode, s.splits)) {
    const uint64_t dims[3] = {static_cast<uint64_t>(s.N), static_cast<uint64_t>(s.M), static_cast<uint64_t>(s.batch)};
    const uint64_t bstride = s.batch > 1 ? static_cast<uint64_t>(e.res_batch_stride) * 2
                                         : static_cast<uint64_t>(s.M) * e.ldr * 2;
    const uint64_t str[2] = {static_cast<uint64_t>(e.ldr) * 2, bstride};
    const uint32_t box[3] = {32, 128, 1};
    if (make_tmap(&tmO2, e.residual, 3, dims, str, box, 2, 64) == cudaSuccess) mode |= kModeResTma;
  }
  switch (bn) {
    case 32: return launch_bn<32>(tmA, tmB, tmO, tmO2, tmV, s, e, vec, mode, err, st);
    case 64: return launch_bn<64>(tmA, tmB, tmO, tmO2, tmV, s, e, vec, mode, err, st);
    case 128: return launch_bn<128>(tmA, tmB, tmO, tmO2, tmV, s, e, vec, mode, err, st);
    case 192: return launch_bn<192>(tmA, tmB, tmO, tmO2, tmV, s, e, vec, mode, err, st);
    case 256: return launch_bn<256>(tmA, tmB, tmO, tmO2, tmV, s, e, vec, mode, err, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace w2v
