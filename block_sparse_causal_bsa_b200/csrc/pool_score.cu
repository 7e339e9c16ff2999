// Key-block pooling and the CUDA-core block score.
//
// Pool ([UGS] step 1, mean-pooled keys; [Stem] Implementação, block
// downsampling): Kbar[b,g,j,:] = (1/block_k) * sum of the block's key rows,
// accumulated in fp32; for the output-aware scores also, from the block's mean
// value vector Vbar_j, either w = ||Vbar_j||_2 (multiplicative form) or
// w = beta * max(0, ln ||Vbar_j||^2) (the additive form of [Stem] 2.B).
// Bounds pool ([UGS] Metodologia step 1, the K-min/K-max backbone): per-coordinate
// minimum and maximum of the block's keys, and for the tensor-core score the
// box centre (kmin+kmax)/2 and half-width (kmax-kmin)/2 as fp16 with a per-block
// power-of-two scale.
//
// Score ([UGS] step 2): s(t,j) = max over the tile's rows of q_i . Kbar_j
// (times w_j, or plus w_j, for the output-aware forms), or of
// sum_c max(q_ic kmin_jc, q_ic kmax_jc) for the bounds backbone; -inf for
// blocks the tile cannot see.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace bsa {

// One CTA per (b, g, key block). 256 threads: each thread owns 8 consecutive
// columns (one 16-byte load for bf16) and a phase of the rows.
// With kbar16 given, the pooled keys are also written as fp16 scaled by a power of two
// 2^r per block (r chosen so that the block's largest |Kbar| lands in [2^14, 2^15)), with
// kinv[block] = 2^-r: the operand of the tensor-core score.
template <typename T, int D>
__global__ void __launch_bounds__(256) pool_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                                   int N, int block_k, float* __restrict__ kbar,
                                                   uint16_t* __restrict__ kbar16,
                                                   float* __restrict__ kinv,
                                                   float* __restrict__ wnorm, int wlog, float beta) {
  constexpr int CPT = 8;                 // columns per thread
  constexpr int TPR = D / CPT;           // threads per row
  constexpr int PHASES = 256 / TPR;      // rows in flight
  __shared__ float red[PHASES][D];
  __shared__ float vsum[D];
  __shared__ float mrow[D];
  __shared__ int rexp;
  const int j = blockIdx.x;
  const size_t bg = blockIdx.y;
  const int n_kb = N / block_k;
  const int c0 = (threadIdx.x % TPR) * CPT;
  const int ph = threadIdx.x / TPR;
  const float inv = 1.0f / (float)block_k;

  for (int pass = 0; pass < (v ? 2 : 1); ++pass) {
    const T* src = (pass == 0 ? k : v) + (bg * N + (size_t)j * block_k) * D;
    float acc[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[c] = 0.f;
    for (int r = ph; r < block_k; r += PHASES) {
      const T* row = src + (size_t)r * D + c0;
      if constexpr (sizeof(T) == 2) {
        uint4 u = *reinterpret_cast<const uint4*>(row);
        const uint16_t* e = reinterpret_cast<const uint16_t*>(&u);
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[c] += bf16_to_f32(e[c]);
      } else {
        float4 a = *reinterpret_cast<const float4*>(row);
        float4 b = *reinterpret_cast<const float4*>(row + 4);
        acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
        acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
      }
    }
#pragma unroll
    for (int c = 0; c < CPT; ++c) red[ph][c0 + c] = acc[c];
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
      float s = 0.f;
      for (int p = 0; p < PHASES; ++p) s += red[p][c];
      float mean = s * inv;
      if (pass == 0) {
        kbar[(bg * n_kb + j) * D + c] = mean;
        mrow[c] = mean;
      } else {
        vsum[c] = mean * mean;
      }
    }
    __syncthreads();
    if (pass == 0 && kbar16) {
      if (threadIdx.x < 32) {
        float mx = 0.f;
        for (int c = threadIdx.x; c < D; c += 32) mx = fmaxf(mx, fabsf(mrow[c]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (threadIdx.x == 0) {
          const uint32_t u = __float_as_uint(mx);
          int r = 0;
          if (u != 0u && u < 0x7f800000u) {
            r = 14 - ((int)(u >> 23) - 127);
            r = r < -126 ? -126 : (r > 126 ? 126 : r);
          }
          rexp = r;
          kinv[bg * n_kb + j] = __int_as_float((127 - r) << 23);
        }
      }
      __syncthreads();
      const float sc = __int_as_float((127 + rexp) << 23);
      for (int c = threadIdx.x; c < D; c += blockDim.x) {
        const __half h = __float2half_rn(mrow[c] * sc);
        kbar16[(bg * n_kb + j) * D + c] = *reinterpret_cast<const uint16_t*>(&h);
      }
    }
  }
  if (v && threadIdx.x < 32) {
    float s = 0.f;
    for (int c = threadIdx.x; c < D; c += 32) s += vsum[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    // s = ||Vbar||^2; ln(0) = -inf contributes 0 to the additive form
    if (threadIdx.x == 0) wnorm[bg * n_kb + j] = wlog ? beta * fmaxf(0.f, logf(s)) : sqrtf(s);
  }
}

// One CTA per (b, g, key block), 256 threads as in pool_kernel: per-coordinate
// min and max over the block's keys (exact: they are input values). With mid16 given,
// also the box centre mid = (kmin+kmax)/2 and half-width rad = (kmax-kmin)/2 as fp16,
// both scaled by one power of two 2^r per block (r chosen so that the block's largest
// of |mid| and rad lands in [2^14, 2^15)), and kinv[block] = 2^-r: the operands of the
// tensor-core bounds score, where max(q a, q b) = q (a+b)/2 + |q| (b-a)/2 for b >= a.
template <typename T, int D>
__global__ void __launch_bounds__(256) pool_bounds_kernel(const T* __restrict__ k, int N, int block_k,
                                                          float* __restrict__ kmin,
                                                          float* __restrict__ kmax,
                                                          uint16_t* __restrict__ mid16,
                                                          uint16_t* __restrict__ rad16,
                                                          float* __restrict__ kinv) {
  constexpr int CPT = 8;
  constexpr int TPR = D / CPT;
  constexpr int PHASES = 256 / TPR;
  __shared__ float rmin[PHASES][D], rmax[PHASES][D];
  __shared__ float smid[D], srad[D];
  __shared__ int rexp;
  const int j = blockIdx.x;
  const size_t bg = blockIdx.y;
  const int n_kb = N / block_k;
  const int c0 = (threadIdx.x % TPR) * CPT;
  const int ph = threadIdx.x / TPR;
  const T* src = k + (bg * N + (size_t)j * block_k) * D;
  float lo[CPT], hi[CPT];
#pragma unroll
  for (int c = 0; c < CPT; ++c) { lo[c] = INFINITY; hi[c] = -INFINITY; }
  for (int r = ph; r < block_k; r += PHASES) {
    const T* row = src + (size_t)r * D + c0;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const float x = load_f32(row, c);
      lo[c] = fminf(lo[c], x);
      hi[c] = fmaxf(hi[c], x);
    }
  }
#pragma unroll
  for (int c = 0; c < CPT; ++c) { rmin[ph][c0 + c] = lo[c]; rmax[ph][c0 + c] = hi[c]; }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float a = rmin[0][c], b = rmax[0][c];
    for (int p = 1; p < PHASES; ++p) { a = fminf(a, rmin[p][c]); b = fmaxf(b, rmax[p][c]); }
    const size_t o = (bg * n_kb + j) * D + c;
    kmin[o] = a;
    kmax[o] = b;
    smid[c] = 0.5f * (a + b);
    srad[c] = 0.5f * (b - a);
  }
  if (!mid16) return;
  __syncthreads();
  if (threadIdx.x < 32) {
    float mx = 0.f;
    for (int c = threadIdx.x; c < D; c += 32) mx = fmaxf(mx, fmaxf(fabsf(smid[c]), srad[c]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (threadIdx.x == 0) {
      const uint32_t u = __float_as_uint(mx);
      int r = 0;
      if (u != 0u && u < 0x7f800000u) {
        r = 14 - ((int)(u >> 23) - 127);
        r = r < -126 ? -126 : (r > 126 ? 126 : r);
      }
      rexp = r;
      kinv[bg * n_kb + j] = __int_as_float((127 - r) << 23);
    }
  }
  __syncthreads();
  const float sc = __int_as_float((127 + rexp) << 23);
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    const size_t o = (bg * n_kb + j) * D + c;
    const __half m = __float2half_rn(smid[c] * sc), r = __float2half_rn(srad[c] * sc);
    mid16[o] = *reinterpret_cast<const uint16_t*>(&m);
    rad16[o] = *reinterpret_cast<const uint16_t*>(&r);
  }
}

cudaError_t launch_pool(const bsa_shape& s, const void* k, const void* v, float* kbar,
                        uint16_t* kbar16, float* kinv, float* wnorm, cudaStream_t st,
                        int wlog, float beta) {
  dim3 grid(s.N / s.block_k, s.B * s.Hkv);
  if (s.dtype == BSA_BF16) {
    auto kk = (const uint16_t*)k;
    auto vv = (const uint16_t*)v;
    if (s.d == 128)
      pool_kernel<uint16_t, 128><<<grid, 256, 0, st>>>(kk, vv, s.N, s.block_k, kbar, kbar16, kinv, wnorm,
                                                       wlog, beta);
    else
      pool_kernel<uint16_t, 64><<<grid, 256, 0, st>>>(kk, vv, s.N, s.block_k, kbar, kbar16, kinv, wnorm,
                                                      wlog, beta);
  } else {
    auto kk = (const float*)k;
    auto vv = (const float*)v;
    if (s.d == 128)
      pool_kernel<float, 128><<<grid, 256, 0, st>>>(kk, vv, s.N, s.block_k, kbar, kbar16, kinv, wnorm,
                                                    wlog, beta);
    else
      pool_kernel<float, 64><<<grid, 256, 0, st>>>(kk, vv, s.N, s.block_k, kbar, kbar16, kinv, wnorm,
                                                   wlog, beta);
  }
  return cudaGetLastError();
}

cudaError_t launch_pool_bounds(const bsa_shape& s, const void* k, float* kmin, float* kmax,
                               uint16_t* mid16, uint16_t* rad16, float* kinv, cudaStream_t st) {
  dim3 grid(s.N / s.block_k, s.B * s.Hkv);
#define BSA_POOLB(T, D)                                                                            \
  pool_bounds_kernel<T, D><<<grid, 256, 0, st>>>((const T*)k, s.N, s.block_k, kmin, kmax, mid16, \
                                                 rad16, kinv)
  if (s.dtype == BSA_BF16) {
    if (s.d == 128) BSA_POOLB(uint16_t, 128); else BSA_POOLB(uint16_t, 64);
  } else {
    if (s.d == 128) BSA_POOLB(float, 128); else BSA_POOLB(float, 64);
  }
#undef BSA_POOLB
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// CUDA-core score. One CTA per (query tile, b*Hq + h); the tile's rows are
// staged in shared memory as fp32, the pooled keys in chunks of 32 blocks.
// Thread (jj, rg) computes block jj of the chunk against rows rg, rg+8, ...
// BOUNDS: kbar holds kmin and kbar2 kmax; each term is max(q kmin, q kmax).
// wmode: 0 none, 1 multiply by w_j, 2 add w_j.
template <typename T, int D, bool BOUNDS>
__global__ void __launch_bounds__(256) score_simt_kernel(const T* __restrict__ q,
                                                         const float* __restrict__ kbar,
                                                         const float* __restrict__ kbar2,
                                                         const float* __restrict__ wnorm, int wmode,
                                                         float* __restrict__ scores, int N, int Hq,
                                                         int Hkv, int tile_q, int block_k) {
  extern __shared__ float sm[];
  float* qs = sm;                          // [tile_q][D]
  float* ks = qs + tile_q * D;             // [32][D+1]
  float* ks2 = ks + 32 * (D + 1);          // [32][D+1] (BOUNDS: kmax)
  __shared__ float mx[8][32];
  const int t = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / Hq, h = bh % Hq;
  const int g = h / (Hq / Hkv);
  const int n_kb = N / block_k, n_qt = N / tile_q;
  const int J = (int)(((long long)(t + 1) * tile_q - 1) / block_k);
  const T* qt = q + ((size_t)bh * N + (size_t)t * tile_q) * D;
  for (int i = threadIdx.x; i < tile_q * D; i += blockDim.x) qs[i] = load_f32(qt, i);
  const float* kb = kbar + ((size_t)b * Hkv + g) * n_kb * D;
  const float* kb2 = BOUNDS ? kbar2 + ((size_t)b * Hkv + g) * n_kb * D : nullptr;
  const float* wb = wnorm ? wnorm + ((size_t)b * Hkv + g) * n_kb : nullptr;
  float* out = scores + ((size_t)bh * n_qt + t) * n_kb;
  const int jj = threadIdx.x % 32, rg = threadIdx.x / 32;
  for (int j0 = 0; j0 <= J; j0 += 32) {
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * D; i += blockDim.x) {
      int r = i / D, c = i % D;
      ks[r * (D + 1) + c] = (j0 + r <= J) ? kb[(size_t)(j0 + r) * D + c] : 0.f;
      if (BOUNDS) ks2[r * (D + 1) + c] = (j0 + r <= J) ? kb2[(size_t)(j0 + r) * D + c] : 0.f;
    }
    __syncthreads();
    float best = -INFINITY;
    for (int r = rg; r < tile_q; r += 8) {
      float acc = 0.f;
      if (BOUNDS) {
#pragma unroll 8
        for (int c = 0; c < D; ++c) {
          const float qc = qs[r * D + c];
          acc += fmaxf(qc * ks[jj * (D + 1) + c], qc * ks2[jj * (D + 1) + c]);
        }
      } else {
#pragma unroll 8
        for (int c = 0; c < D; ++c) acc = fmaf(qs[r * D + c], ks[jj * (D + 1) + c], acc);
      }
      best = fmaxf(best, acc);
    }
    mx[rg][jj] = best;
    __syncthreads();
    if (threadIdx.x < 32 && j0 + jj <= J) {
      float m = mx[0][jj];
      for (int p = 1; p < 8; ++p) m = fmaxf(m, mx[p][jj]);
      if (wb) m = wmode == 2 ? m + wb[j0 + jj] : m * wb[j0 + jj];
      out[j0 + jj] = m;
    }
  }
  for (int j = J + 1 + threadIdx.x; j < n_kb; j += blockDim.x) out[j] = -INFINITY;
}

cudaError_t launch_score_simt(const bsa_shape& s, const void* q, const float* kbar,
                              const float* kbar2, const float* wnorm, int wmode, float* scores,
                              cudaStream_t st) {
  dim3 grid(s.N / s.tile_q, s.B * s.Hq);
  const bool bounds = kbar2 != nullptr;
  size_t smem = (size_t)s.tile_q * s.d * 4 + (bounds ? 2 : 1) * 32 * (s.d + 1) * 4;
  cudaError_t e = cudaSuccess;
#define BSA_SCORE_LAUNCH_B(T, D, BND)                                                         \
  do {                                                                                        \
    e = cudaFuncSetAttribute(score_simt_kernel<T, D, BND>,                                    \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);         \
    if (e != cudaSuccess) return e;                                                           \
    score_simt_kernel<T, D, BND><<<grid, 256, smem, st>>>((const T*)q, kbar, kbar2, wnorm,    \
                                                          wmode, scores, s.N, s.Hq, s.Hkv,    \
                                                          s.tile_q, s.block_k);               \
  } while (0)
#define BSA_SCORE_LAUNCH(T, D)                                    \
  do {                                                            \
    if (bounds) BSA_SCORE_LAUNCH_B(T, D, true);                   \
    else BSA_SCORE_LAUNCH_B(T, D, false);                         \
  } while (0)
  if (s.dtype == BSA_BF16) {
    if (s.d == 128) BSA_SCORE_LAUNCH(uint16_t, 128); else BSA_SCORE_LAUNCH(uint16_t, 64);
  } else {
    if (s.d == 128) BSA_SCORE_LAUNCH(float, 128); else BSA_SCORE_LAUNCH(float, 64);
  }
#undef BSA_SCORE_LAUNCH
#undef BSA_SCORE_LAUNCH_B
  return cudaGetLastError();
}

}  // namespace bsa
