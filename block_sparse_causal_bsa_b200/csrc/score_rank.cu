// Block scores on Blackwell tensor cores, optionally fused with the per-tile
// ranking of the selection ([UGS] steps 1-3: mean-pooled keys, the tile's block
// score as the max over its rows, top-k with the cut margin sigma; [Stem] 2.B for
// the output-aware value terms).
//
// s(t,j) = max over the tile's rows i of q_i . Kbar_j (times w_j, or plus w_j, for
// the output-aware forms), for j <= J_t.
//
// Contraction. D[128 blocks x 128*HP rows] = Kbar_chunk . [Q_h0; Q_h1]^T on tcgen05,
// so each TMEM lane holds one block and its thread takes the max over rows locally.
// Both operands are fp16, one pass: each head's query tile is scaled by a power of
// two 2^s (chosen from the tile's largest |q| so that it lands in [2^14, 2^15)) when
// it is converted from bf16 in shared memory, and each pooled-key block by its own
// power of two 2^r (chosen the same way by the pool kernel). Scaling by a power of
// two is exact, so the accumulated dot product is q . Kbar * 2^(s + r) with the
// only rounding the fp16 rounding of Kbar (relative 2^-12; Q converts exactly
// unless an element lies more than 2^-24 below the tile's largest) and the fp32
// accumulation; the epilogue multiplies the row max by 2^-s and 2^-r, again exactly.
//
// The K-min/K-max backbone ([UGS] Metodologia step 1, per-coordinate upper bounds) runs
// in the same kernel (BOUNDS): s(t,j) = max over rows of sum_c max(q_c kmin_jc, q_c kmax_jc)
// = q . mid_j + |q| . rad_j with mid = (kmin+kmax)/2 and rad = (kmax-kmin)/2 >= 0, so each
// chunk is two fp16 passes into one accumulator, mid against Q and rad against |Q| (written
// by the conversion beside Q). One head per unit: two heads' Q and |Q|, double-buffered,
// would not fit in shared memory.
//
// Persistent: one CTA per SM walks units (batch, KV head, query tile, head pair),
// longest tiles first. Warps:
//   0 (one thread)  TMA: each unit's query tiles (bf16) into one of two Q buffers,
//                   the next unit's as soon as its buffer is free; pooled-key chunks
//                   of 128 blocks (fp16) into two stages.
//   1 (one thread)  MMA: 8 x (M128 N128*HP K16) per chunk into one of two TMEM
//                   accumulators.
//   2-5             epilogue: convert a Q buffer in place (bf16 -> scaled fp16) ahead
//                   of its unit; per chunk, the row max from TMEM, the exact rescale,
//                   the value term, and the row written to the scores array or to an
//                   L2-resident ring; per unit, the row's min / max / finiteness.
//   6-10 (RANK)     five rank warps: each ranks whole rows (rank_row), rows taken in
//                   unit order round-robin, reading the row from L2 in every pass, while
//                   the tensor cores score later units; writes the top-M list with the
//                   top-m flag and sigma. The rows of up to 8 units wait in the ring, so
//                   the epilogue runs ahead of the ranking.
// Every wait is bounded (tc::mbar_wait); a timeout raises BSA_DEV_TIMEOUT and the CTA
// unwinds, waits for its own copies and MMAs, and frees its TMEM.
// Shapes: bf16 inputs, d = 128, query tile 128, key block 64 or 128.
#include <math.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "rank_row.cuh"
#include "tc_common.cuh"

namespace bsa {

namespace {
constexpr int TQ = 128;                       // query tile rows
constexpr int HD = 128;                       // head dim
constexpr int CB = 128;                       // blocks per chunk (MMA M)
constexpr int kEpiWarps = 4;
constexpr uint32_t kHalfTile = 16384;         // 128 rows x 128 bytes: one 64-column half
constexpr uint32_t kChunk = 2 * kHalfTile;    // one pooled-key chunk (128 blocks x 128 dims, fp16)

constexpr int kRankWarpsF = 5;                // rank warps of the fused kernel
constexpr int kRing = kScoreRankRing;         // units whose rows the L2 ring holds

template <int HP, bool RANK, bool BOUNDS>
struct SRLayout {
  static constexpr int rank_warps = RANK ? kRankWarpsF : 0;
  static constexpr int threads = (2 + kEpiWarps + rank_warps) * 32;
  static constexpr uint32_t qhalf = HP * kHalfTile;     // one d-half of all HP heads' tiles
  static constexpr uint32_t qabs = 2 * qhalf;           // K-min/K-max: |Q| behind Q in the buffer
  static constexpr uint32_t qbuf = (BOUNDS ? 2 : 1) * 2 * qhalf;   // one Q buffer
  static constexpr size_t smem_q = 0;                   // two Q buffers
  static constexpr size_t smem_k = 2 * (size_t)qbuf;    // two chunk stages
  static constexpr size_t smem_rank = smem_k + 2 * (size_t)kChunk;
  static constexpr size_t smem_ctrl = smem_rank + (size_t)rank_warps * kRankSliceWords * 4;
  static constexpr uint32_t dcols = HP * TQ;            // accumulator columns per buffer
  static constexpr uint32_t tmem_cols = 2 * dcols;
};

struct RowStat {
  float mn, mx;
  int bad;
};

template <int HP>
struct __align__(8) SRCtrl {
  uint64_t q_full[2], qc_full[2], q_empty[2];
  uint64_t kb_full[2], kb_empty[2];
  uint64_t d_full[2], d_free[2];
  uint64_t row_full[kRing], row_free[kRing];
  uint64_t qmax_bar;
  uint64_t done;
  uint32_t tmem;
  int abort_flag;
  uint32_t qmax_part[2][HP][kEpiWarps];   // by phase parity of qmax_bar, head, epilogue warp
  RowStat stat[kRing][HP][kEpiWarps];     // per ring slot, head, epilogue warp
};

__device__ __forceinline__ bool warp_all(bool x) { return __all_sync(0xffffffffu, x); }

// 2^e as a float, e in [-126, 127]
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// Power-of-two exponent that brings a largest magnitude x into [2^14, 2^15): 0 for
// x = 0 or a non-finite x, clamped to [-126, 126].
__device__ __forceinline__ int fp16_scale_exp(float x) {
  const uint32_t u = __float_as_uint(x) & 0x7fffffffu;
  if (u == 0u || u >= 0x7f800000u) return 0;
  const int e = (int)(u >> 23) - 127;           // floor(log2 x) for normal x; -127 for subnormal
  const int s = 14 - e;
  return s < -126 ? -126 : (s > 126 ? 126 : s);
}

struct SRArgs {
  const float* kinv;      // [B*Hkv*n_kb] 2^-r of each pooled-key block's fp16 scaling
  const float* wnorm;     // value term per block, or null
  int wmode;              // 0 none, 1 times w, 2 plus w
  float* scores;          // [B,Hq,n_qt,n_kb] or null (ranking only)
  float* ring;            // [grid][kRing][HP][n_kb] when scores is null
  int32_t* ranked;        // [B*Hq*n_qt][W] top-M lists (ranking)
  float* sigma;           // [B*Hq*n_qt]
  int W;
  int k_first, k_last, rho;
  int32_t* dev_status;
  int N, Hq, Hkv, n_qt, n_kb, block_k;
  int units;
};

__device__ __forceinline__ void unit_coords(int u, int npair, int BG, int n_qt, int& t, int& bg,
                                            int& pr) {
  pr = u % npair;
  const int x = u / npair;
  bg = x % BG;
  t = n_qt - 1 - x / BG;                        // longest tiles first
}
}  // namespace

// BOUNDS: the K-min/K-max backbone (one head per unit, no ranking). tmk then holds the
// per-block mid = (kmin+kmax)/2 and tmk2 the rad = (kmax-kmin)/2 >= 0 (fp16, one power-of-two
// scale per block, as for the mean), and each chunk is two passes into one accumulator,
// mid against Q and rad against |Q|: sum_c max(q_c kmin_c, q_c kmax_c) = q . mid + |q| . rad.
template <int HP, bool RANK, bool BOUNDS>
__global__ void __launch_bounds__(SRLayout<HP, RANK, BOUNDS>::threads, 1) score_rank_kernel(
    const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
    const __grid_constant__ CUtensorMap tmk2, const SRArgs a) {
  static_assert(!BOUNDS || (HP == 1 && !RANK), "the K-min/K-max variant scores one head per unit");
  using L = SRLayout<HP, RANK, BOUNDS>;
  constexpr int kParts = BOUNDS ? 2 : 1;        // pooled-key half-chunks per chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SRCtrl<HP>& c = *reinterpret_cast<SRCtrl<HP>*>(sm + L::smem_ctrl);
  const uint32_t sQ = tc::smem_u32(sm + L::smem_q);
  const uint32_t sK = tc::smem_u32(sm + L::smem_k);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = a.Hq / a.Hkv;
  const int npair = G / HP;
  const int BG = (a.units / a.n_qt) / npair;    // B * Hkv
  const int stride = gridDim.x;
  int32_t* dev_status = a.dev_status;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&c.q_full[i], 1);
      tc::mbar_init(&c.qc_full[i], kEpiWarps);
      tc::mbar_init(&c.q_empty[i], 1);
      tc::mbar_init(&c.kb_full[i], 1);
      tc::mbar_init(&c.kb_empty[i], 1);
      tc::mbar_init(&c.d_full[i], 1);
      tc::mbar_init(&c.d_free[i], kEpiWarps);
    }
    for (int i = 0; i < kRing; ++i) {
      tc::mbar_init(&c.row_full[i], kEpiWarps);
      tc::mbar_init(&c.row_free[i], HP);
    }
    tc::mbar_init(&c.qmax_bar, kEpiWarps);
    tc::mbar_init(&c.done, 1);
    c.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&c.tmem, L::tmem_cols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = c.tmem;
  volatile int* abort_flag = &c.abort_flag;
  int q_issued = 0, kb_issued = 0;
  bool mma_issued = false;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    if (BOUNDS) tc::prefetch_tmap(&tmk2);
    auto issue_q = [&](int li, int u) -> bool {
      const int qb = li & 1;
      if (li >= 2 && !tc::mbar_wait(&c.q_empty[qb], ((li >> 1) - 1) & 1, abort_flag, dev_status)) return false;
      int t, bg, pr;
      unit_coords(u, npair, BG, a.n_qt, t, bg, pr);
      const int b = bg / a.Hkv, g = bg % a.Hkv;
      const int h0 = g * G + pr * HP;
      uint8_t* dst = sm + L::smem_q + qb * L::qbuf;
      tc::mbar_arrive_expect_tx(&c.q_full[qb], 2 * L::qhalf);   // the bf16 tiles (|Q| is made here)
      for (int hp = 0; hp < HP; ++hp) {
        const int qrow = (int)(((size_t)b * a.Hq + h0 + hp) * a.N + (size_t)t * TQ);
        tc::tma_load_2d(dst + hp * kHalfTile, &tmq, 0, qrow, &c.q_full[qb]);
        tc::tma_load_2d(dst + L::qhalf + hp * kHalfTile, &tmq, 64, qrow, &c.q_full[qb]);
      }
      q_issued = li + 1;
      return true;
    };
    bool ok = (int)blockIdx.x >= a.units || issue_q(0, blockIdx.x);
    int gk = 0;                                   // half-chunk loads (one per chunk unless BOUNDS)
    for (int li = 0, u = blockIdx.x; ok && u < a.units; ++li, u += stride) {
      int t, bg, pr;
      unit_coords(u, npair, BG, a.n_qt, t, bg, pr);
      const int J = (int)(((long long)(t + 1) * TQ - 1) / a.block_k);
      const int nc = (J + 1 + CB - 1) / CB;
      for (int ch = 0; ok && ch < nc; ++ch) {
        for (int part = 0; part < kParts; ++part, ++gk) {
          const int s = gk & 1;
          if (gk >= 2 && !tc::mbar_wait(&c.kb_empty[s], ((gk >> 1) - 1) & 1, abort_flag, dev_status)) {
            ok = false;
            break;
          }
          uint8_t* dst = sm + L::smem_k + s * kChunk;
          const int row = bg * a.n_kb + ch * CB;
          const CUtensorMap* m = part ? &tmk2 : &tmk;
          tc::mbar_arrive_expect_tx(&c.kb_full[s], kChunk);
          tc::tma_load_2d(dst, m, 0, row, &c.kb_full[s]);
          tc::tma_load_2d(dst + kHalfTile, m, 64, row, &c.kb_full[s]);
          kb_issued = gk + 1;
        }
        // the next unit's query tiles, as soon as their buffer is free
        if (ok && ch == 0 && u + stride < a.units && !issue_q(li + 1, u + stride)) ok = false;
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idesc = tc::idesc_f16_f32(CB, HP * TQ, false, false);
    bool ok = true;
    int gc = 0, gk = 0;
    for (int li = 0, u = blockIdx.x; ok && u < a.units; ++li, u += stride) {
      const int qb = li & 1;
      if (!tc::mbar_wait(&c.qc_full[qb], (li >> 1) & 1, abort_flag, dev_status)) break;
      int t, bg, pr;
      unit_coords(u, npair, BG, a.n_qt, t, bg, pr);
      const int J = (int)(((long long)(t + 1) * TQ - 1) / a.block_k);
      const int nc = (J + 1 + CB - 1) / CB;
      const uint32_t qbase = sQ + qb * L::qbuf;
      for (int ch = 0; ch < nc; ++ch, ++gc) {
        const int db = gc & 1;
        ok = gc < 2 || tc::mbar_wait(&c.d_free[db], ((gc >> 1) - 1) & 1, abort_flag, dev_status);
        const uint32_t d = tmem + db * L::dcols;
        for (int part = 0; ok && part < kParts; ++part, ++gk) {
          const int s = gk & 1;
          ok = tc::mbar_wait(&c.kb_full[s], (gk >> 1) & 1, abort_flag, dev_status);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t kb = sK + s * kChunk;
          const uint32_t qpart = qbase + (part ? L::qabs : 0u);   // Q against mid, |Q| against rad
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t aoff = (kk >> 2) * kHalfTile + (kk & 3) * 32;
            const uint32_t boff = (kk >> 2) * L::qhalf + (kk & 3) * 32;
            tc::umma_bf16(d, tc::sdesc_sw128(kb + aoff, 16, 1024), tc::sdesc_sw128(qpart + boff, 16, 1024),
                          idesc, (part > 0 || kk > 0) ? 1u : 0u);
          }
          mma_issued = true;
          tc::umma_commit(&c.kb_empty[s]);
        }
        if (!ok) break;
        tc::umma_commit(&c.d_full[db]);
      }
      if (!ok) break;
      tc::umma_commit(&c.q_empty[qb]);          // every MMA of this unit read its Q buffer
    }
  } else if (warp >= 2 && warp < 2 + kEpiWarps) {
    // ---------------- epilogue (and Q conversion) ----------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;          // block within the chunk == TMEM lane; Q row
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    int qmax_phase = 0;
    float qs0[HP], qs1[HP];                     // 2^-s per head of Q buffers 0 and 1 (every
                                                // epilogue thread computes its own copy)
    // Q buffer of local unit li: bf16 -> fp16 scaled by 2^s per head, in place (both are
    // 16-bit, so the swizzled layout stays). Thread r owns row r of every head.
    auto convert = [&](int li) -> bool {
      const int qb = li & 1;
      if (!warp_all(tc::mbar_wait(&c.q_full[qb], (li >> 1) & 1, abort_flag, dev_status))) return false;
      uint8_t* base = sm + L::smem_q + qb * L::qbuf;
      for (int hp = 0; hp < HP; ++hp) {
        uint4 v[16];
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          // chunk order XOR-ed with the row's swizzle phase: eight consecutive rows touch
          // eight different 16-byte columns, so the warp's loads do not conflict
          const int half = p >> 3, ck = (p & 7) ^ (r & 7);
          v[p] = *reinterpret_cast<const uint4*>(base + half * L::qhalf + hp * kHalfTile + r * 128 + ck * 16);
        }
        uint32_t mx = 0u;
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          mx = __vmaxu2(mx, v[p].x & 0x7fff7fffu);
          mx = __vmaxu2(mx, v[p].y & 0x7fff7fffu);
          mx = __vmaxu2(mx, v[p].z & 0x7fff7fffu);
          mx = __vmaxu2(mx, v[p].w & 0x7fff7fffu);
        }
        mx = max(mx & 0xffffu, mx >> 16);       // largest bf16 magnitude bits of the row
        mx = warp_max_u32(mx);
        // the parts of phase k are read before any warp arrives for phase k+1, and a warp
        // writes the parts of phase k+2 only after every warp arrived for phase k+1
        const int ph = qmax_phase & 1;
        if (lane == 0) c.qmax_part[ph][hp][quarter] = mx;
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&c.qmax_bar);
        if (!warp_all(tc::mbar_wait(&c.qmax_bar, ph, abort_flag, dev_status))) return false;
        ++qmax_phase;
        uint32_t mb = c.qmax_part[ph][hp][0];
#pragma unroll
        for (int w = 1; w < kEpiWarps; ++w) mb = max(mb, c.qmax_part[ph][hp][w]);
        const int se = fp16_scale_exp(__uint_as_float(mb << 16));
        const float sc = exp2i(se);
        if (qb == 0) qs0[hp] = exp2i(-se);
        else qs1[hp] = exp2i(-se);
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          uint32_t w4[4] = {v[p].x, v[p].y, v[p].z, v[p].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(w4[e] << 16) * sc;
            const float hi = __uint_as_float(w4[e] & 0xffff0000u) * sc;
            const __half2 h2 = __floats2half2_rn(lo, hi);
            w4[e] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          const int half = p >> 3, ck = (p & 7) ^ (r & 7);
          const uint32_t off = half * L::qhalf + hp * kHalfTile + r * 128 + ck * 16;
          *reinterpret_cast<uint4*>(base + off) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          if (BOUNDS)        // |Q| in fp16: the same values with the sign bits cleared
            *reinterpret_cast<uint4*>(base + L::qabs + off) =
                make_uint4(w4[0] & 0x7fff7fffu, w4[1] & 0x7fff7fffu, w4[2] & 0x7fff7fffu, w4[3] & 0x7fff7fffu);
        }
      }
      tc::fence_proxy_async_smem();               // generic writes -> tensor-core reads
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.qc_full[qb]);
      return true;
    };
    bool ok = (int)blockIdx.x >= a.units || convert(0);
    int gc = 0;
    for (int li = 0, u = blockIdx.x; ok && u < a.units; ++li, u += stride) {
      const int slot = li % kRing, qb = li & 1;
      int t, bg, pr;
      unit_coords(u, npair, BG, a.n_qt, t, bg, pr);
      const int b = bg / a.Hkv, g = bg % a.Hkv;
      const int h0 = g * G + pr * HP;
      const int J = (int)(((long long)(t + 1) * TQ - 1) / a.block_k);
      const int f_lo = (int)(((long long)t * TQ) / a.block_k);
      const int nc = (J + 1 + CB - 1) / CB;
      const bool next = u + stride < a.units;
      const int conv_at = nc - 1 < 3 ? nc - 1 : 3;    // chunk before which the next Q is converted
      if (RANK && li >= kRing &&
          !warp_all(tc::mbar_wait(&c.row_free[slot], (li / kRing - 1) & 1, abort_flag, dev_status))) {
        ok = false;
        break;
      }
      float* rows[HP];
#pragma unroll
      for (int hp = 0; hp < HP; ++hp)
        rows[hp] = a.scores ? a.scores + (((size_t)b * a.Hq + h0 + hp) * a.n_qt + t) * a.n_kb
                            : a.ring + (((size_t)blockIdx.x * kRing + slot) * HP + hp) * a.n_kb;
      float mn[HP], mxv[HP];
      bool bad[HP];
#pragma unroll
      for (int hp = 0; hp < HP; ++hp) { mn[hp] = INFINITY; mxv[hp] = -INFINITY; bad[hp] = false; }
      float qi[HP];
#pragma unroll
      for (int hp = 0; hp < HP; ++hp) qi[hp] = qb ? qs1[hp] : qs0[hp];
      const float* kinv = a.kinv + (size_t)bg * a.n_kb;
      const float* wrow = a.wnorm ? a.wnorm + (size_t)bg * a.n_kb : nullptr;
      for (int ch = 0; ch < nc; ++ch, ++gc) {
        if (next && ch == conv_at && !convert(li + 1)) { ok = false; break; }
        const int db = gc & 1;
        const int j = ch * CB + r;
        const float kv = j <= J ? __ldg(kinv + j) : 0.f;
        const float wv = (wrow && j <= J) ? __ldg(wrow + j) : 0.f;
        if (!warp_all(tc::mbar_wait(&c.d_full[db], (gc >> 1) & 1, abort_flag, dev_status))) { ok = false; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int hp = 0; hp < HP; ++hp) {
          float m;
          if constexpr (RANK) {
            // 32 columns per load: the rank warps leave 168 registers per thread
            m = -INFINITY;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t v[32];
              tc::tmem_ld32(tl + db * L::dcols + hp * TQ + cc * 32, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) m = fmaxf(m, __uint_as_float(v[i]));
            }
          } else {
            float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              uint32_t v[64];
              tc::tmem_ld64(tl + db * L::dcols + hp * TQ + cc * 64, v);
#pragma unroll
              for (int i = 0; i < 64; i += 2) {
                m0 = fmaxf(m0, __uint_as_float(v[i]));
                m1 = fmaxf(m1, __uint_as_float(v[i + 1]));
              }
            }
            m = fmaxf(m0, m1);
          }
          float val = (m * qi[hp]) * kv;             // exact: powers of two
          if (a.wmode == 1) val = val * wv;
          else if (a.wmode == 2) val = val + wv;
          if (j <= J) rows[hp][j] = val;
          if (RANK && j < f_lo) {
            mn[hp] = fminf(mn[hp], val);
            mxv[hp] = fmaxf(mxv[hp], val);
            bad[hp] |= !isfinite(val);
          }
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&c.d_free[db]);
      }
      if (!ok) break;
      if (a.scores) {
        // blocks no row of the tile can see
        for (int hp = 0; hp < HP; ++hp)
          for (int j = J + 1 + r; j < a.n_kb; j += kEpiWarps * 32) rows[hp][j] = -INFINITY;
      }
      if (RANK) {
#pragma unroll
        for (int hp = 0; hp < HP; ++hp) {
          const float wmn = warp_min_f32(mn[hp]);
          const float wmx = warp_max_f32(mxv[hp]);
          const bool wbad = __any_sync(0xffffffffu, bad[hp]);
          if (lane == 0) c.stat[slot][hp][quarter] = RowStat{wmn, wmx, wbad ? 1 : 0};
        }
        __threadfence_block();                       // the row's global writes before the release
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&c.row_full[slot]);
      }
    }
  } else if (RANK && warp >= 2 + kEpiWarps) {
    // ---------------- rank warps ----------------
    // Rows are numbered in unit order (row li*HP + hp); rank warp w takes the rows congruent
    // to w modulo kRankWarpsF, so several rows are ranked at once while the tensor cores
    // score later units. A warp reads its row from L2 (the ring, or the scores array) in
    // every ranking pass; the ring slot is freed when the unit's HP rows are ranked.
    const int rw = warp - (2 + kEpiWarps);
    uint32_t* slice = reinterpret_cast<uint32_t*>(sm + L::smem_rank) + (size_t)rw * kRankSliceWords;
    const int li_end = ((int)a.units - (int)blockIdx.x + stride - 1) / stride;   // units of this CTA
    for (int gr = rw; gr < li_end * HP; gr += kRankWarpsF) {
      const int li = gr / HP, hp = gr % HP;
      const int slot = li % kRing;
      if (!warp_all(tc::mbar_wait(&c.row_full[slot], (li / kRing) & 1, abort_flag, dev_status))) break;
      const int u = blockIdx.x + li * stride;
      int t, bg, pr;
      unit_coords(u, npair, BG, a.n_qt, t, bg, pr);
      const int b = bg / a.Hkv, g = bg % a.Hkv;
      const size_t row = ((size_t)b * a.Hq + g * G + pr * HP + hp) * a.n_qt + t;
      const TileSlots sl = tile_slots(t, a.n_qt, TQ, a.block_k, a.k_first, a.k_last, a.rho);
      const int n = sl.f_lo;
      float xmin = c.stat[slot][hp][0].mn, xmax = c.stat[slot][hp][0].mx;
      int anybad = c.stat[slot][hp][0].bad;
#pragma unroll
      for (int w = 1; w < kEpiWarps; ++w) {
        xmin = fminf(xmin, c.stat[slot][hp][w].mn);
        xmax = fmaxf(xmax, c.stat[slot][hp][w].mx);
        anybad |= c.stat[slot][hp][w].bad;
      }
      const bool bad = n > 0 && anybad != 0;
      float sg = 1.0f;
      if (n > 0) {
        const float* src = a.scores ? a.scores + row * a.n_kb
                                    : a.ring + (((size_t)blockIdx.x * kRing + slot) * HP + hp) * a.n_kb;
        sg = rank_row<false>(src, n, sl, xmin, xmax, bad, slice, a.ranked + row * a.W, lane);
      }
      if (lane == 0) {
        if (bad) {
          set_status(dev_status, BSA_DEV_BAD_SCORE);
          sg = __int_as_float(0x7fc00000);
        }
        a.sigma[row] = sg;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.row_free[slot]);
    }
  }

  // ---------------- teardown ----------------
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0) {
    // every TMA copy this CTA issued has landed before the CTA exits
    for (int li = q_issued - 2 < 0 ? 0 : q_issued - 2; li < q_issued; ++li)
      tc::mbar_wait_timed(&c.q_full[li & 1], (li >> 1) & 1);
    for (int gc = kb_issued - 2 < 0 ? 0 : kb_issued - 2; gc < kb_issued; ++gc)
      tc::mbar_wait_timed(&c.kb_full[gc & 1], (gc >> 1) & 1);
  }
  if (warp == 1) {
    if (lane == 0 && mma_issued) {
      tc::umma_commit(&c.done);
      tc::mbar_wait_timed(&c.done, 0);
    }
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, L::tmem_cols);
  }
}

bool score_rank_supported(const bsa_shape& s) {
  return s.dtype == BSA_BF16 && s.d == HD && s.tile_q == TQ &&
         (long long)s.B * s.Hq * s.N < (1ll << 31) &&
         (long long)s.B * s.Hkv * (s.N / s.block_k) < (1ll << 31);
}

bool score_rank_fusable(const bsa_shape& s) { return score_rank_supported(s); }

int score_rank_heads_per_unit(const bsa_shape& s) { return ((s.Hq / s.Hkv) % 2 == 0) ? 2 : 1; }

template <int HP, bool RANK, bool BOUNDS = false>
static cudaError_t launch_sr(const bsa_shape& s, const CUtensorMap& mq, const CUtensorMap& mk,
                             const CUtensorMap& mk2, const SRArgs& a, int grid, cudaStream_t st) {
  using L = SRLayout<HP, RANK, BOUNDS>;
  const size_t smem = L::smem_ctrl + sizeof(SRCtrl<HP>) + 1024;
  static_assert(L::smem_ctrl + sizeof(SRCtrl<HP>) + 1024 <= 227 * 1024, "shared memory");
  cudaError_t e = cudaFuncSetAttribute(score_rank_kernel<HP, RANK, BOUNDS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  score_rank_kernel<HP, RANK, BOUNDS><<<grid, L::threads, smem, st>>>(mq, mk, mk2, a);
  return cudaGetLastError();
}

static int sm_count(int* sms) {
  int dev = 0;
  *sms = 148;
  return cudaGetDevice(&dev) == cudaSuccess &&
         cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
}

cudaError_t launch_score_rank(const bsa_shape& s, const bsa_select_params* p, const void* q,
                              const uint16_t* kbar16, const float* kinv, const float* wnorm, int wmode,
                              float* scores, float* ring, int ring_ctas, int32_t* ranked, float* sigma,
                              int W, int32_t* dev_status, cudaStream_t st) {
  CUtensorMap mq, mk;
  const uint64_t qrows = (uint64_t)s.B * s.Hq * s.N;
  const uint64_t krows = (uint64_t)s.B * s.Hkv * (s.N / s.block_k);
  if (!make_tmap_bf16_2d(&mq, q, qrows, HD, 64, TQ) || !make_tmap_bf16_2d(&mk, kbar16, krows, HD, 64, CB))
    return cudaErrorInvalidValue;
  const int HP = score_rank_heads_per_unit(s);
  const int n_qt = s.N / TQ;
  SRArgs a{};
  a.kinv = kinv;
  a.wnorm = wnorm;
  a.wmode = wmode;
  a.scores = scores;
  a.ring = ring;
  a.ranked = ranked;
  a.sigma = sigma;
  a.W = W;
  a.k_first = p ? p->k_first : 0;
  a.k_last = p ? p->k_last : 0;
  a.rho = p ? p->rho : 1;
  a.dev_status = dev_status;
  a.N = s.N;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.n_qt = n_qt;
  a.n_kb = s.N / s.block_k;
  a.block_k = s.block_k;
  const long long units = (long long)s.B * s.Hkv * n_qt * ((s.Hq / s.Hkv) / HP);
  a.units = (int)units;
  int sms = 148;
  if (!sm_count(&sms)) return cudaErrorInvalidValue;
  long long grid = units < sms ? units : sms;
  if (ranked && !scores && grid > ring_ctas) grid = ring_ctas;
  if (grid < 1) grid = 1;
  if (ranked) {
    return HP == 2 ? launch_sr<2, true>(s, mq, mk, mk, a, (int)grid, st)
                   : launch_sr<1, true>(s, mq, mk, mk, a, (int)grid, st);
  }
  return HP == 2 ? launch_sr<2, false>(s, mq, mk, mk, a, (int)grid, st)
                 : launch_sr<1, false>(s, mq, mk, mk, a, (int)grid, st);
}

cudaError_t launch_score_rank_bounds(const bsa_shape& s, const void* q, const uint16_t* mid16,
                                     const uint16_t* rad16, const float* kinv, float* scores,
                                     int32_t* dev_status, cudaStream_t st) {
  CUtensorMap mq, mm, mr;
  const uint64_t qrows = (uint64_t)s.B * s.Hq * s.N;
  const uint64_t krows = (uint64_t)s.B * s.Hkv * (s.N / s.block_k);
  if (!make_tmap_bf16_2d(&mq, q, qrows, HD, 64, TQ) || !make_tmap_bf16_2d(&mm, mid16, krows, HD, 64, CB) ||
      !make_tmap_bf16_2d(&mr, rad16, krows, HD, 64, CB))
    return cudaErrorInvalidValue;
  const int n_qt = s.N / TQ;
  SRArgs a{};
  a.kinv = kinv;
  a.wmode = 0;
  a.scores = scores;
  a.rho = 1;
  a.dev_status = dev_status;
  a.N = s.N;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.n_qt = n_qt;
  a.n_kb = s.N / s.block_k;
  a.block_k = s.block_k;
  const long long units = (long long)s.B * s.Hkv * n_qt * (s.Hq / s.Hkv);
  a.units = (int)units;
  int sms = 148;
  if (!sm_count(&sms)) return cudaErrorInvalidValue;
  long long grid = units < sms ? units : sms;
  if (grid < 1) grid = 1;
  return launch_sr<1, false, true>(s, mq, mm, mr, a, (int)grid, st);
}

}  // namespace bsa
