// Key-block pooling and the CUDA-core block score.
//
// Pool ([UGS] step 1, mean-pooled keys; [Stem] Implementação, block
// downsampling): Kbar[b,g,j,:] = (1/block_k) * sum of the block's key rows,
// accumulated in fp32; for the output-aware score also
// w[b,g,j] = || (1/block_k) * sum of the block's V rows ||_2.
//
// Score ([UGS] step 2): s(t,j) = max over the tile's rows of q_i . Kbar_j
// (times w_j for the output-aware form), -inf for blocks the tile cannot see.
#include "common.cuh"
#include "kernels.h"

namespace bsa {

// One CTA per (b, g, key block). 256 threads: each thread owns 8 consecutive
// columns (one 16-byte load for bf16) and a phase of the rows.
template <typename T, int D>
__global__ void __launch_bounds__(256) pool_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                                   int N, int block_k, float* __restrict__ kbar,
                                                   uint16_t* __restrict__ kbar_hi,
                                                   uint16_t* __restrict__ kbar_lo,
                                                   float* __restrict__ wnorm) {
  constexpr int CPT = 8;                 // columns per thread
  constexpr int TPR = D / CPT;           // threads per row
  constexpr int PHASES = 256 / TPR;      // rows in flight
  __shared__ float red[PHASES][D];
  __shared__ float vsum[D];
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
        size_t o = (bg * n_kb + j) * D + c;
        kbar[o] = mean;
        if (kbar_hi) {
          uint16_t hi = f32_to_bf16_rn(mean);
          kbar_hi[o] = hi;
          kbar_lo[o] = f32_to_bf16_rn(mean - bf16_to_f32(hi));
        }
      } else {
        vsum[c] = mean * mean;
      }
    }
    __syncthreads();
  }
  if (v && threadIdx.x < 32) {
    float s = 0.f;
    for (int c = threadIdx.x; c < D; c += 32) s += vsum[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) wnorm[bg * n_kb + j] = sqrtf(s);
  }
}

cudaError_t launch_pool(const bsa_shape& s, const void* k, const void* v, float* kbar,
                        uint16_t* kbar_hi, uint16_t* kbar_lo, float* wnorm, cudaStream_t st) {
  dim3 grid(s.N / s.block_k, s.B * s.Hkv);
  if (s.dtype == BSA_BF16) {
    auto kk = (const uint16_t*)k;
    auto vv = (const uint16_t*)v;
    if (s.d == 128)
      pool_kernel<uint16_t, 128><<<grid, 256, 0, st>>>(kk, vv, s.N, s.block_k, kbar, kbar_hi, kbar_lo, wnorm);
    else
      pool_kernel<uint16_t, 64><<<grid, 256, 0, st>>>(kk, vv, s.N, s.block_k, kbar, kbar_hi, kbar_lo, wnorm);
  } else {
    auto kk = (const float*)k;
    auto vv = (const float*)v;
    if (s.d == 128)
      pool_kernel<float, 128><<<grid, 256, 0, st>>>(kk, vv, s.N, s.block_k, kbar, kbar_hi, kbar_lo, wnorm);
    else
      pool_kernel<float, 64><<<grid, 256, 0, st>>>(kk, vv, s.N, s.block_k, kbar, kbar_hi, kbar_lo, wnorm);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// CUDA-core score. One CTA per (query tile, b*Hq + h); the tile's rows are
// staged in shared memory as fp32, the pooled keys in chunks of 32 blocks.
// Thread (jj, rg) computes block jj of the chunk against rows rg, rg+8, ...
template <typename T, int D>
__global__ void __launch_bounds__(256) score_simt_kernel(const T* __restrict__ q,
                                                         const float* __restrict__ kbar,
                                                         const float* __restrict__ wnorm,
                                                         float* __restrict__ scores, int N, int Hq,
                                                         int Hkv, int tile_q, int block_k) {
  extern __shared__ float sm[];
  float* qs = sm;                          // [tile_q][D]
  float* ks = qs + tile_q * D;             // [32][D+1]
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
  const float* wb = wnorm ? wnorm + ((size_t)b * Hkv + g) * n_kb : nullptr;
  float* out = scores + ((size_t)bh * n_qt + t) * n_kb;
  const int jj = threadIdx.x % 32, rg = threadIdx.x / 32;
  for (int j0 = 0; j0 <= J; j0 += 32) {
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * D; i += blockDim.x) {
      int r = i / D, c = i % D;
      ks[r * (D + 1) + c] = (j0 + r <= J) ? kb[(size_t)(j0 + r) * D + c] : 0.f;
    }
    __syncthreads();
    float best = -INFINITY;
    for (int r = rg; r < tile_q; r += 8) {
      float acc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = fmaf(qs[r * D + c], ks[jj * (D + 1) + c], acc);
      best = fmaxf(best, acc);
    }
    mx[rg][jj] = best;
    __syncthreads();
    if (threadIdx.x < 32 && j0 + jj <= J) {
      float m = mx[0][jj];
      for (int p = 1; p < 8; ++p) m = fmaxf(m, mx[p][jj]);
      if (wb) m = m * wb[j0 + jj];
      out[j0 + jj] = m;
    }
  }
  for (int j = J + 1 + threadIdx.x; j < n_kb; j += blockDim.x) out[j] = -INFINITY;
}

cudaError_t launch_score_simt(const bsa_shape& s, const void* q, const float* kbar,
                              const float* wnorm, float* scores, cudaStream_t st) {
  dim3 grid(s.N / s.tile_q, s.B * s.Hq);
  size_t smem = (size_t)s.tile_q * s.d * 4 + 32 * (s.d + 1) * 4;
  cudaError_t e = cudaSuccess;
#define BSA_SCORE_LAUNCH(T, D)                                                              \
  do {                                                                                      \
    e = cudaFuncSetAttribute(score_simt_kernel<T, D>,                                       \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);       \
    if (e != cudaSuccess) return e;                                                         \
    score_simt_kernel<T, D><<<grid, 256, smem, st>>>((const T*)q, kbar, wnorm, scores, s.N, \
                                                     s.Hq, s.Hkv, s.tile_q, s.block_k);     \
  } while (0)
  if (s.dtype == BSA_BF16) {
    if (s.d == 128) BSA_SCORE_LAUNCH(uint16_t, 128); else BSA_SCORE_LAUNCH(uint16_t, 64);
  } else {
    if (s.d == 128) BSA_SCORE_LAUNCH(float, 128); else BSA_SCORE_LAUNCH(float, 64);
  }
#undef BSA_SCORE_LAUNCH
  return cudaGetLastError();
}

}  // namespace bsa
