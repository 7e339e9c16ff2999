// Per-tile top-k selection, the uncertainty gate and kv_idx
// ([UGS] steps 2-5; [Stem] 2.A for the position-dependent budget).
//
// select_rank: one CTA per (b, h, tile). The candidate blocks 0..f_lo-1 are
//   ranked by (score desc, index asc) with a bitonic sort of 64-bit keys in
//   shared memory; the first `need` indices go to the ranked list, and the
//   cut margin sigma = (s_(m-1) - s_(m)) / (s_(0) - s_(m)) is evaluated in
//   fp32 with correctly rounded operations ([UGS] step 3).
// gate: one CTA. sigma_bar[b,t] = fp32 sum of sigma over heads in head order,
//   divided by Hq; theta = linear-interpolation empirical quantile of
//   sigma_bar over the cut tiles of the call; trigger = cut && sigma_bar <
//   theta ([UGS] step 4).
// finalize: one CTA per (b, h, tile): forced blocks plus the first m_t (or
//   M_t when triggered) ranked candidates, ascending, -1 padded to W
//   ([UGS] step 5).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

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

__global__ void __launch_bounds__(512) select_rank_kernel(
    const float* __restrict__ scores, int n_qt, int n_kb, int tile_q, int block_k, int k_first,
    int k_last, int rho, int R, int32_t* __restrict__ ranked, float* __restrict__ sigma,
    int32_t* dev_status) {
  extern __shared__ unsigned long long keys[];
  const int t = blockIdx.x;
  const size_t row = (size_t)blockIdx.y * n_qt + t;
  const TileSlots sl = tile_slots(t, n_qt, tile_q, block_k, k_first, k_last, rho);
  const int n = sl.f_lo;
  const float* s = scores + row * n_kb;
  if (n == 0) {
    if (threadIdx.x == 0) sigma[row] = 1.0f;
    return;
  }
  int need = sl.M > sl.m ? sl.M : sl.m;
  if (sl.cut && need < sl.m + 1) need = sl.m + 1;
  if (need > n) need = n;
  const unsigned P = next_pow2((unsigned)n);
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (unsigned i = threadIdx.x; i < P; i += blockDim.x) {
    unsigned long long key = 0ull;            // padding sorts last
    if (i < (unsigned)n) {
      float x = s[i];
      if (!isfinite(x)) bad = 1;
      key = ((unsigned long long)score_key(x) << 32) | (unsigned long long)(~i);
    }
    keys[i] = key;
  }
  bitonic_sort(keys, P, true);
  int32_t* out = ranked + row * R;
  for (int r = threadIdx.x; r < need; r += blockDim.x) out[r] = (int32_t)(~(uint32_t)keys[r]);
  if (threadIdx.x == 0) {
    if (bad) set_status(dev_status, BSA_DEV_BAD_SCORE);
    float sg = 1.0f;
    if (bad) {
      sg = __int_as_float(0x7fc00000);
    } else if (sl.cut) {
      // values read back from the score row, so signed zeros match the input exactly
      float s0 = s[~(uint32_t)keys[0]];
      float a = s[~(uint32_t)keys[sl.m - 1]];
      float b = s[~(uint32_t)keys[sl.m]];
      float num = __fsub_rn(a, b);
      float den = __fsub_rn(s0, b);
      sg = (den == 0.0f) ? 0.0f : __fdiv_rn(num, den);
    }
    sigma[row] = sg;
  }
}

cudaError_t launch_select_rank(const bsa_shape& s, const bsa_select_params& p, const float* scores,
                               int R, int32_t* ranked, float* sigma, int32_t* dev_status,
                               cudaStream_t st) {
  const int n_qt = s.N / s.tile_q, n_kb = s.N / s.block_k;
  unsigned P = 1;
  while (P < (unsigned)n_kb) P <<= 1;
  size_t smem = (size_t)P * 8;
  cudaError_t e = cudaFuncSetAttribute(select_rank_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_qt, s.B * s.Hq);
  select_rank_kernel<<<grid, 512, smem, st>>>(scores, n_qt, n_kb, s.tile_q, s.block_k, p.k_first,
                                              p.k_last, p.rho, R, ranked, sigma, dev_status);
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
    float acc = 0.0f;
    for (int h = 0; h < Hq; ++h) acc = __fadd_rn(acc, sigma[((size_t)b * Hq + h) * n_qt + t]);
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

__global__ void __launch_bounds__(256) finalize_kernel(
    const int32_t* __restrict__ ranked, int R, const uint8_t* __restrict__ trigger, int Hq,
    int n_qt, int tile_q, int block_k, int k_first, int k_last, int rho, int W,
    int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt) {
  extern __shared__ int32_t buf[];
  const int t = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / Hq;
  const size_t row = (size_t)bh * n_qt + t;
  const TileSlots sl = tile_slots(t, n_qt, tile_q, block_k, k_first, k_last, rho);
  const int take = trigger[(size_t)b * n_qt + t] ? sl.M : sl.m;
  const unsigned P = next_pow2((unsigned)(take > 0 ? take : 1));
  for (unsigned i = threadIdx.x; i < P; i += blockDim.x)
    buf[i] = (int)i < take ? ranked[row * R + i] : 0x7fffffff;
  bitonic_sort(buf, P, false);
  int32_t* out = kv_idx + row * W;
  for (int i = threadIdx.x; i < W; i += blockDim.x) {
    int32_t x;
    if (i < take) x = buf[i];
    else if (i < take + sl.nF) x = sl.f_lo + (i - take);
    else x = -1;
    out[i] = x;
  }
  if (threadIdx.x == 0) kv_cnt[row] = take + sl.nF;
}

cudaError_t launch_finalize(const bsa_shape& s, const bsa_select_params& p, const int32_t* ranked,
                            int R, const uint8_t* trigger, int W, int32_t* kv_idx, int32_t* kv_cnt,
                            cudaStream_t st) {
  const int n_qt = s.N / s.tile_q;
  unsigned P = 1;
  while (P < (unsigned)W) P <<= 1;
  size_t smem = (size_t)P * 4;
  cudaError_t e = cudaFuncSetAttribute(finalize_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_qt, s.B * s.Hq);
  finalize_kernel<<<grid, 256, smem, st>>>(ranked, R, trigger, s.Hq, n_qt, s.tile_q, s.block_k,
                                           p.k_first, p.k_last, p.rho, W, kv_idx, kv_cnt);
  return cudaGetLastError();
}

}  // namespace bsa
