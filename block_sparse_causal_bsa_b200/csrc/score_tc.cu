// K-min/K-max block scores on Blackwell tensor cores (tcgen05 + TMEM + TMA). The
// mean-pooled backbones run in score_rank.cu; this kernel keeps the two-operand bounds
// form with bf16 hi/lo operands.
//
// s(t,j) = max over the tile's rows i of q_i . Kbar_j ([UGS] step 2: the
// tile's block score is the max over its rows; step 1: mean-pooled keys),
// times w_j = ||mean V_j|| for the output-aware form, -inf for j > J_t.
//
// The contraction runs transposed: D[128 blocks x 128*HP query rows] =
// Kbar_chunk . [Q_h0 ; Q_h1]^T, so each TMEM lane holds one block and its
// thread takes the row max locally. HP = 2 query heads of one KV group share
// every pooled-key chunk (N = 256). Kbar is fp32; it enters the MMA as a bf16
// hi/lo pair (Kbar = hi + lo to ~2^-17 relative) over two K = d passes into
// the same fp32 accumulator, so the scores keep ~fp32 accuracy with bf16
// operands (Q is exactly bf16 already).
//
// One CTA per (batch, KV head, query tile, head pair); 192 threads:
//   warp 0: TMA producer (Q tiles once, then pooled-key chunks of 128 blocks,
//           hi and lo, double-buffered);
//   warp 1: MMA issuer (16 MMAs of M128 N256 K16 per chunk into one of two
//           TMEM accumulators);
//   warps 2-5: epilogue (TMEM -> row max -> scores row, times or plus the
//           block's value term for the output-aware forms), overlapping the
//           next chunk's MMAs.
// K-min/K-max bounds backbone (BND): sum_c max(q_c kmin_c, q_c kmax_c) =
// q . mid + |q| . rad with mid = (kmin+kmax)/2, rad = (kmax-kmin)/2 >= 0, a
// contraction over 2d: each chunk is two half-chunks (mid hi/lo against Q,
// then rad hi/lo against |Q|) accumulated into the same TMEM columns. |Q| is
// made once per CTA by the epilogue warps (sign bits cleared in a shared-memory
// copy of the Q tile). One query head per CTA (N = 128) so that Q, |Q| and two
// half-chunk stages fit in shared memory.
// Shapes: bf16, d = 128, query tile 128, key block 64 or 128.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace bsa {

namespace {
constexpr int TQ = 128;           // query tile rows
constexpr int HD = 128;           // head dim
constexpr int CB = 128;           // blocks per chunk (MMA M)
constexpr int kThreads = 192;
constexpr uint32_t kQHalf = 16384;         // one head: 128 rows x 128 bytes
constexpr uint32_t kChunkHalf = 16384;     // 128 blocks x 128 bytes
constexpr uint32_t kStage = 4 * kChunkHalf;  // hi (2 halves) + lo (2 halves)
constexpr uint32_t kTmemCols = 512;

template <int HP, bool BND>
struct Layout {
  static constexpr uint32_t qhalf = HP * kQHalf;               // one d-half for all HP heads
  static constexpr size_t smem_q = 0;
  static constexpr size_t smem_qa = 2 * qhalf;                  // |Q| (BND)
  static constexpr size_t smem_k = (BND ? 4 : 2) * qhalf;
  static constexpr size_t smem_ctrl = smem_k + 2 * kStage;
  static constexpr uint32_t dcols = HP * TQ;                    // accumulator columns per buffer
};

struct __align__(8) Ctrl {
  uint64_t q_full, qa_full;
  uint64_t kb_full[2], kb_empty[2];
  uint64_t d_full[2], d_free[2];
  uint64_t done;
  uint32_t tmem;
  int abort_flag;
};

__device__ __forceinline__ bool warp_all(bool x) { return __all_sync(0xffffffffu, x); }
}  // namespace

template <int HP, bool BND>
__global__ void __launch_bounds__(kThreads, 1) score_tc_kernel(
    const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmhi,
    const __grid_constant__ CUtensorMap tmlo, const __grid_constant__ CUtensorMap tmhi2,
    const __grid_constant__ CUtensorMap tmlo2, const float* __restrict__ wnorm, int wmode,
    float* __restrict__ scores, int32_t* dev_status, int N, int Hq, int Hkv, int n_qt, int n_kb,
    int block_k) {
  using L = Layout<HP, BND>;
  constexpr int PARTS = BND ? 2 : 1;                // half-chunks per chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl& c = *reinterpret_cast<Ctrl*>(sm + L::smem_ctrl);
  const uint32_t sQ = tc::smem_u32(sm + L::smem_q);
  const uint32_t sQa = tc::smem_u32(sm + L::smem_qa);
  const uint32_t sK = tc::smem_u32(sm + L::smem_k);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const int G = Hq / Hkv;
  const int npair = G / HP;
  int x = blockIdx.x;
  const int pr = x % npair;
  x /= npair;
  const int t = n_qt - 1 - (x % n_qt);             // longest rows first
  const int bgi = x / n_qt;
  const int b = bgi / Hkv, g = bgi % Hkv;
  const int h0 = g * G + pr * HP;
  const int J = (int)(((long long)(t + 1) * TQ - 1) / block_k);
  const int nc = (J + 1 + CB - 1) / CB;
  const int kb_row0 = bgi * n_kb;

  if (threadIdx.x == 0) {
    tc::mbar_init(&c.q_full, 1);
    tc::mbar_init(&c.qa_full, 4);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&c.kb_full[i], 1);
      tc::mbar_init(&c.kb_empty[i], 1);
      tc::mbar_init(&c.d_full[i], 1);
      tc::mbar_init(&c.d_free[i], 4);
    }
    tc::mbar_init(&c.done, 1);
    c.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&c.tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = c.tmem;
  volatile int* abort_flag = &c.abort_flag;
  int kb_issued = 0;
  bool mma_issued = false;

  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmhi);
    tc::prefetch_tmap(&tmlo);
    if (BND) {
      tc::prefetch_tmap(&tmhi2);
      tc::prefetch_tmap(&tmlo2);
    }
    tc::mbar_arrive_expect_tx(&c.q_full, 2 * L::qhalf);
    for (int hp = 0; hp < HP; ++hp) {
      const int qrow = (int)(((size_t)b * Hq + h0 + hp) * N + (size_t)t * TQ);
      tc::tma_load_2d(sm + L::smem_q + hp * kQHalf, &tmq, 0, qrow, &c.q_full);
      tc::tma_load_2d(sm + L::smem_q + L::qhalf + hp * kQHalf, &tmq, 64, qrow, &c.q_full);
    }
    for (int u = 0; u < nc * PARTS; ++u) {        // u: half-chunk (BND) or chunk
      const int s = u & 1;
      if (u >= 2 && !tc::mbar_wait(&c.kb_empty[s], ((u >> 1) - 1) & 1, abort_flag, dev_status)) break;
      uint8_t* dst = sm + L::smem_k + s * kStage;
      const int row = kb_row0 + (u / PARTS) * CB;
      const bool second = BND && (u & 1);
      const CUtensorMap* mh = second ? &tmhi2 : &tmhi;
      const CUtensorMap* ml = second ? &tmlo2 : &tmlo;
      tc::mbar_arrive_expect_tx(&c.kb_full[s], kStage);
      tc::tma_load_2d(dst, mh, 0, row, &c.kb_full[s]);
      tc::tma_load_2d(dst + kChunkHalf, mh, 64, row, &c.kb_full[s]);
      tc::tma_load_2d(dst + 2 * kChunkHalf, ml, 0, row, &c.kb_full[s]);
      tc::tma_load_2d(dst + 3 * kChunkHalf, ml, 64, row, &c.kb_full[s]);
      kb_issued = u + 1;
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = tc::idesc_bf16_f32(128, HP * TQ, false, false);
    bool ok = tc::mbar_wait(&c.q_full, 0, abort_flag, dev_status) &&
              (!BND || tc::mbar_wait(&c.qa_full, 0, abort_flag, dev_status));
    for (int ch = 0; ok && ch < nc; ++ch) {
      const int db = ch & 1;
      ok = ch < 2 || tc::mbar_wait(&c.d_free[db], ((ch >> 1) - 1) & 1, abort_flag, dev_status);
      const uint32_t d = tmem + db * L::dcols;
      for (int part = 0; ok && part < PARTS; ++part) {
        const int u = ch * PARTS + part;
        const int s = u & 1;
        ok = tc::mbar_wait(&c.kb_full[s], (u >> 1) & 1, abort_flag, dev_status);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t kb = sK + s * kStage;
        const uint32_t qb = part == 0 ? sQ : sQa;       // Q against mid, |Q| against rad
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {        // hi, then lo
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t aoff = pass * 2 * kChunkHalf + (kk >> 2) * kChunkHalf + (kk & 3) * 32;
            const uint32_t boff = (kk >> 2) * L::qhalf + (kk & 3) * 32;
            tc::umma_bf16(d, tc::sdesc_sw128(kb + aoff, 16, 1024), tc::sdesc_sw128(qb + boff, 16, 1024),
                          idesc, (part > 0 || pass > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_issued = true;
        tc::umma_commit(&c.kb_empty[s]);
      }
      if (!ok) break;
      tc::umma_commit(&c.d_full[db]);
    }
  } else if (warp >= 2) {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // block within the chunk == TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const float* wrow = wnorm ? wnorm + (size_t)bgi * n_kb : nullptr;
    bool qa_ok = true;
    if (BND) {
      // |Q|: a copy of the swizzled Q tile with the sign bits cleared (same layout)
      qa_ok = warp_all(tc::mbar_wait(&c.q_full, 0, abort_flag, dev_status));
      if (qa_ok) {
        const uint4* src = reinterpret_cast<const uint4*>(sm + L::smem_q);
        uint4* dst = reinterpret_cast<uint4*>(sm + L::smem_qa);
        for (int i = threadIdx.x - 64; i < (int)(2 * L::qhalf / 16); i += 128) {
          uint4 w = src[i];
          w.x &= 0x7fff7fffu; w.y &= 0x7fff7fffu; w.z &= 0x7fff7fffu; w.w &= 0x7fff7fffu;
          dst[i] = w;
        }
        tc::fence_proxy_async_smem();                  // generic writes -> tensor-core reads
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&c.qa_full);
      }
    }
    for (int ch = 0; qa_ok && ch < nc; ++ch) {
      const int s = ch & 1;
      if (!warp_all(tc::mbar_wait(&c.d_full[s], (ch >> 1) & 1, abort_flag, dev_status))) break;
      tc::tc_fence_after();
      const int j = ch * CB + r;
#pragma unroll
      for (int hp = 0; hp < HP; ++hp) {
        float m = -INFINITY;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t v[32];
          tc::tmem_ld32(tl + s * L::dcols + hp * TQ + cc * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) m = fmaxf(m, __uint_as_float(v[i]));
        }
        if (j <= J) {
          if (wrow) m = wmode == 2 ? m + wrow[j] : m * wrow[j];
          scores[(((size_t)b * Hq + h0 + hp) * n_qt + t) * n_kb + j] = m;
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.d_free[s]);
    }
    // blocks no row of the tile can see
    for (int hp = 0; hp < HP; ++hp) {
      float* row = scores + (((size_t)b * Hq + h0 + hp) * n_qt + t) * n_kb;
      for (int j = J + 1 + (threadIdx.x - 64); j < n_kb; j += 128) row[j] = -INFINITY;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0) {
    tc::mbar_wait_timed(&c.q_full, 0);
    for (int u = kb_issued - 2 < 0 ? 0 : kb_issued - 2; u < kb_issued; ++u)
      tc::mbar_wait_timed(&c.kb_full[u & 1], (u >> 1) & 1);
  }
  if (warp == 1) {
    if (lane == 0 && mma_issued) {
      tc::umma_commit(&c.done);
      tc::mbar_wait_timed(&c.done, 0);
    }
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

bool score_tc_supported(const bsa_shape& s) {
  return s.dtype == BSA_BF16 && s.d == HD && s.tile_q == TQ &&
         (long long)s.B * s.Hq * s.N < (1ll << 31) &&
         (long long)s.B * s.Hkv * (s.N / s.block_k) < (1ll << 31);
}

template <int HP, bool BND>
static cudaError_t launch_score_tc_t(const bsa_shape& s, const CUtensorMap& mq, const CUtensorMap& mh,
                                     const CUtensorMap& ml, const CUtensorMap& mh2,
                                     const CUtensorMap& ml2, const float* wnorm, int wmode,
                                     float* scores, int32_t* dev_status, cudaStream_t st) {
  using L = Layout<HP, BND>;
  const size_t smem = L::smem_ctrl + sizeof(Ctrl) + 1024;
  cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<HP, BND>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n_qt = s.N / TQ;
  const long long grid = (long long)s.B * s.Hkv * n_qt * ((s.Hq / s.Hkv) / HP);
  score_tc_kernel<HP, BND><<<(unsigned)grid, kThreads, smem, st>>>(
      mq, mh, ml, mh2, ml2, wnorm, wmode, scores, dev_status, s.N, s.Hq, s.Hkv, n_qt, s.N / s.block_k,
      s.block_k);
  return cudaGetLastError();
}

cudaError_t launch_score_tc_bounds(const bsa_shape& s, const void* q, const uint16_t* mid_hi,
                                   const uint16_t* mid_lo, const uint16_t* rad_hi,
                                   const uint16_t* rad_lo, float* scores, int32_t* dev_status,
                                   cudaStream_t st) {
  CUtensorMap mq, mh, ml, mh2, ml2;
  const uint64_t qrows = (uint64_t)s.B * s.Hq * s.N;
  const uint64_t krows = (uint64_t)s.B * s.Hkv * (s.N / s.block_k);
  if (!make_tmap_bf16_2d(&mq, q, qrows, HD, 64, TQ) || !make_tmap_bf16_2d(&mh, mid_hi, krows, HD, 64, CB) ||
      !make_tmap_bf16_2d(&ml, mid_lo, krows, HD, 64, CB) || !make_tmap_bf16_2d(&mh2, rad_hi, krows, HD, 64, CB) ||
      !make_tmap_bf16_2d(&ml2, rad_lo, krows, HD, 64, CB))
    return cudaErrorInvalidValue;
  return launch_score_tc_t<1, true>(s, mq, mh, ml, mh2, ml2, nullptr, 0, scores, dev_status, st);
}

}  // namespace bsa
