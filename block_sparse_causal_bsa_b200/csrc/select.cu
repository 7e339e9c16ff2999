// Per-tile top-k selection, the uncertainty gate and kv_idx
// ([UGS] steps 2-5; [Stem] 2.A for the position-dependent budget).
//
// select_rank: one warp per (b, h, tile). The candidate blocks 0..f_lo-1 are
//   ranked by (score desc, index asc): a value-bucket histogram narrows the top
//   entries to a short list whose exact ranks come from pairwise counts within
//   each bucket (exact radix selection on order-preserving 32-bit keys for the
//   rows where that list is long), and the top-M blocks are written ascending,
//   the top-m ones marked. The cut margin
//   sigma = (s_(m-1) - s_(m)) / (s_(0) - s_(m)) is evaluated in fp32 with
//   correctly rounded operations on the scores read back by index ([UGS] step 3).
// gate: one CTA. sigma_bar[b,t] = fp32 sum of sigma over heads in head order,
//   divided by Hq; theta = linear-interpolation empirical quantile of
//   sigma_bar over the cut tiles of the call; trigger = cut && sigma_bar <
//   theta ([UGS] step 4).
// finalize: one warp per (b, h, tile): the first m_t (or M_t when triggered)
//   ranked candidates, ascending, then the forced blocks, -1 padded to W
//   ([UGS] step 5).
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "rank_row.cuh"

namespace bsa {

__device__ __forceinline__ unsigned next_pow2(unsigned n) {
  unsigned p = 1;
  while (p < n) p <<= 1;
  return p;
}

// In-place bitonic sort of n (a power of two) 64-bit keys in shared memory.
// descending = true sorts largest first. All threads of the CTA take part.
template <typename K>
__device__ void bitonic_sort(K* a, unsigned n, bool descending) {
  for (unsigned size = 2; size <= n; size <<= 1) {
    for (unsigned stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (unsigned i = threadIdx.x; i < n / 2; i += blockDim.x) {
        unsigned lo = 2 * i - (i & (stride - 1));
        unsigned hi = lo + stride;
        bool up = ((lo & size) == 0) != descending;   // ascending segment?
        K x = a[lo], y = a[hi];
        if ((x > y) == up) { a[lo] = y; a[hi] = x; }
      }
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Ranking: one warp per (b, h, tile) row, four rows per CTA. Each pass reads the
// row's scores from global memory (16-byte loads, four per lane in flight); the
// warp's shared-memory slice holds only the histogram and the short list, which
// keeps it small: eight CTAs (32 warps) per SM, bounded by 64 registers per thread.
// The ranking itself (value buckets with an exact radix fallback) is rank_row().

constexpr int kRankWarps = 4;                // rows (warps) per CTA

// Writes, per row, the top-M candidates (M = expanded slots) in ascending block
// order with kInTopM set on the top-m ones, and sigma from ranks 0, m-1, m.
__global__ void __launch_bounds__(kRankWarps * 32, 8) select_rank_kernel(
    const float* __restrict__ scores, int rows_bh, int n_qt, int n_kb, int tile_q, int block_k,
    int k_first, int k_last, int rho, int R, int32_t* __restrict__ ranked, float* __restrict__ sigma,
    int32_t* dev_status) {
  extern __shared__ __align__(16) uint32_t wsm[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y * kRankWarps + warp;
  if (bh >= rows_bh) return;
  const int t = n_qt - 1 - (int)blockIdx.x;          // longest rows first
  const size_t row = (size_t)bh * n_qt + t;
  const TileSlots sl = tile_slots(t, n_qt, tile_q, block_k, k_first, k_last, rho);
  const int n = sl.f_lo;
  const float* s = scores + row * n_kb;
  if (n == 0) {
    if (lane == 0) sigma[row] = 1.0f;
    return;
  }
  float xmin, xmax;
  bool bad;
  row_minmax<true>(s, n, lane, xmin, xmax, bad);
  float sg = rank_row<true>(s, n, sl, xmin, xmax, bad, wsm + (size_t)warp * kRankSliceWords,
                            ranked + row * R, lane);
  if (lane == 0) {
    if (bad) {
      set_status(dev_status, BSA_DEV_BAD_SCORE);
      sg = __int_as_float(0x7fc00000);
    }
    sigma[row] = sg;
  }
}

cudaError_t launch_select_rank(const bsa_shape& s, const bsa_select_params& p, const float* scores,
                               int R, int32_t* ranked, float* sigma, int32_t* dev_status,
                               cudaStream_t st) {
  const int n_qt = s.N / s.tile_q, n_kb = s.N / s.block_k;
  const size_t smem = (size_t)kRankWarps * kRankSliceWords * 4;
  const int rows_bh = s.B * s.Hq;
  dim3 grid(n_qt, (rows_bh + kRankWarps - 1) / kRankWarps);
  cudaError_t e = cudaFuncSetAttribute(select_rank_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // occupancy is set by the slices: ask for the largest shared-memory carve-out
  e = cudaFuncSetAttribute(select_rank_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  select_rank_kernel<<<grid, kRankWarps * 32, smem, st>>>(scores, rows_bh, n_qt, n_kb, s.tile_q,
                                                         s.block_k, p.k_first, p.k_last, p.rho, R,
                                                         ranked, sigma, dev_status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(1024) gate_kernel(const float* __restrict__ sigma, int B, int Hq,
                                                    int n_qt, int tile_q, int block_k, int k_first,
                                                    int k_last, int rho, float q, float fixed,
                                                    float* __restrict__ sigma_bar,
                                                    uint8_t* __restrict__ trigger,
                                                    float* __restrict__ theta) {
  extern __shared__ float pop[];
  __shared__ unsigned cnt;
  __shared__ float th;
  if (threadIdx.x == 0) cnt = 0;
  __syncthreads();
  const int total = B * n_qt;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int b = i / n_qt, t = i % n_qt;
    // eight heads' values in flight at a time, added in head order
    float acc = 0.0f;
    const float* col = sigma + (size_t)b * Hq * n_qt + t;
    for (int h0 = 0; h0 < Hq; h0 += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = h0 + u < Hq ? __ldg(col + (size_t)(h0 + u) * n_qt) : 0.0f;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (h0 + u < Hq) acc = __fadd_rn(acc, v[u]);
    }
    const float sb = __fdiv_rn(acc, (float)Hq);
    sigma_bar[i] = sb;
    if (tile_slots(t, n_qt, tile_q, block_k, k_first, k_last, rho).cut) pop[atomicAdd(&cnt, 1u)] = sb;
  }
  __syncthreads();
  const unsigned M = cnt;
  const bool gated = rho > 1;
  if (gated && q >= 0.0f && M > 0) {
    unsigned P = next_pow2(M);
    for (unsigned i = M + threadIdx.x; i < P; i += blockDim.x) pop[i] = INFINITY;
    bitonic_sort(pop, P, false);
    if (threadIdx.x == 0) {
      double pos = (double)q * (double)(M - 1);
      unsigned lo = (unsigned)floor(pos);
      unsigned hi = lo + 1 < M ? lo + 1 : M - 1;
      float f = __double2float_rn(pos - (double)lo);
      float diff = __fsub_rn(pop[hi], pop[lo]);
      th = __fadd_rn(pop[lo], __fmul_rn(f, diff));
    }
  } else if (threadIdx.x == 0) {
    th = (gated && q < 0.0f) ? fixed : __int_as_float(0x7fc00000);
  }
  __syncthreads();
  const float tv = th;
  if (threadIdx.x == 0 && theta) *theta = tv;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int t = i % n_qt;
    bool trig = gated && tile_slots(t, n_qt, tile_q, block_k, k_first, k_last, rho).cut &&
                (sigma_bar[i] < tv);
    trigger[i] = trig ? 1 : 0;
  }
}

cudaError_t launch_gate(const bsa_shape& s, const bsa_select_params& p, const float* sigma,
                        float* sigma_bar, uint8_t* trigger, float* theta, cudaStream_t st) {
  const int n_qt = s.N / s.tile_q;
  unsigned P = 1;
  while (P < (unsigned)(s.B * n_qt)) P <<= 1;
  size_t smem = (size_t)P * 4;
  cudaError_t e = cudaFuncSetAttribute(gate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  gate_kernel<<<1, 1024, smem, st>>>(sigma, s.B, s.Hq, n_qt, s.tile_q, s.block_k, p.k_first,
                                     p.k_last, p.rho, p.gate_quantile, p.gate_threshold, sigma_bar,
                                     trigger, theta);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------

// One warp per (b, h, tile) row: the triggered tiles take the whole top-M list,
// the others only its kInTopM entries; both are already in ascending block
// order and precede the forced blocks, which follow; -1 pads to W.
__global__ void __launch_bounds__(256) finalize_kernel(
    const int32_t* __restrict__ ranked, int R, const uint8_t* __restrict__ trigger, int rows_bh,
    int Hq, int n_qt, int tile_q, int block_k, int k_first, int k_last, int rho, int W,
    int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y * (blockDim.x / 32) + warp;
  if (bh >= rows_bh) return;
  const int t = blockIdx.x;
  const int b = bh / Hq;
  const size_t row = (size_t)bh * n_qt + t;
  const TileSlots sl = tile_slots(t, n_qt, tile_q, block_k, k_first, k_last, rho);
  const bool all = trigger[(size_t)b * n_qt + t] != 0;
  const int take = all ? sl.M : sl.m;
  const int32_t* in = ranked + row * R;
  int32_t* out = kv_idx + row * W;
  const unsigned lt = (1u << lane) - 1u;
  int pos = 0;
  for (int b0 = 0; b0 < sl.M; b0 += 32) {
    const int i = b0 + lane;
    const int32_t e = i < sl.M ? in[i] : 0;
    const bool keep = i < sl.M && (all || (e & (int32_t)kInTopM));
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) out[pos + __popc(bal & lt)] = e & 0x7fffffff;
    pos += __popc(bal);
  }
  for (int i = take + lane; i < W; i += 32) out[i] = (i < take + sl.nF) ? sl.f_lo + (i - take) : -1;
  if (lane == 0) kv_cnt[row] = take + sl.nF;
}

cudaError_t launch_finalize(const bsa_shape& s, const bsa_select_params& p, const int32_t* ranked,
                            int R, const uint8_t* trigger, int W, int32_t* kv_idx, int32_t* kv_cnt,
                            cudaStream_t st) {
  const int n_qt = s.N / s.tile_q;
  const int rows_bh = s.B * s.Hq;
  dim3 grid(n_qt, (rows_bh + 7) / 8);
  finalize_kernel<<<grid, 256, 0, st>>>(ranked, R, trigger, rows_bh, s.Hq, n_qt, s.tile_q, s.block_k,
                                        p.k_first, p.k_last, p.rho, W, kv_idx, kv_cnt);
  return cudaGetLastError();
}

}  // namespace bsa
