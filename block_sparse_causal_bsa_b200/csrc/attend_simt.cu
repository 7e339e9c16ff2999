// Block-sparse causal attention on CUDA cores (fp32 math).
//
// O_i = sum over the keys j of the listed blocks with j <= i of
// softmax(scale * q_i . k_j) v_j ([UGS] step 5 and [Stem] Implementação:
// attention streams only the selected key blocks), evaluated FlashAttention
// style: keys arrive in chunks of 64, each chunk updates a running row max,
// the softmax denominator and the output with an online rescale.
//
// One CTA per 64 query rows of a tile (a 128-row tile takes two CTAs; both
// read the same kv_idx row). 256 threads: thread (ty, tx) owns rows
// 4*ty..4*ty+3, score columns tx + 16*c and output columns tx + 16*c.
// This is the fp32 path, and the bf16 path for shapes the tensor-core kernel
// does not cover (d = 64, key blocks of 128, query tiles of 64).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace bsa {

namespace {
constexpr int RQ = 64;   // query rows per CTA
constexpr int CK = 64;   // keys per chunk
}

template <typename T, int D>
__global__ void __launch_bounds__(256) attend_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt, int W,
    float scale_log2, T* __restrict__ out, float* __restrict__ lse, int32_t* dev_status, int N,
    int Hq, int Hkv, int tile_q, int block_k) {
  extern __shared__ float sm[];
  float* Qs = sm;                         // [RQ][D+1]
  float* Ks = Qs + RQ * (D + 1);          // [CK][D+1]
  float* Vs = Ks + CK * (D + 1);          // [CK][D]
  float* Ps = Vs + CK * D;                // [RQ][CK+1]
  const int sub = blockIdx.x;             // 64-row sub-tile index
  const int bh = blockIdx.y;
  const int b = bh / Hq, h = bh % Hq;
  const int g = h / (Hq / Hkv);
  const int n_qt = N / tile_q, n_kb = N / block_k;
  const int row0 = sub * RQ;
  const int t = row0 / tile_q;
  const int J = (int)(((long long)(t + 1) * tile_q - 1) / block_k);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;

  const T* qp = q + ((size_t)bh * N + row0) * D;
  const T* kp = k + ((size_t)b * Hkv + g) * N * D;
  const T* vp = v + ((size_t)b * Hkv + g) * N * D;
  for (int i = threadIdx.x; i < RQ * D; i += blockDim.x)
    Qs[(i / D) * (D + 1) + i % D] = load_f32(qp, i);

  float m[4], l[4], o[4][D / 16];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) o[i][c] = 0.f;
  }

  const size_t krow = (size_t)bh * n_qt + t;
  int cnt = kv_cnt[krow];
  if (cnt > W || cnt < 0) {
    if (threadIdx.x == 0) set_status(dev_status, BSA_DEV_BAD_INDEX);
    cnt = cnt < 0 ? 0 : W;
  }
  const int32_t* list = kv_idx + krow * W;
  for (int e = 0; e < cnt; ++e) {
    const int j = list[e];
    if (j < 0 || j >= n_kb || j > J) {
      if (threadIdx.x == 0) set_status(dev_status, BSA_DEV_BAD_INDEX);
      continue;
    }
    for (int ch = 0; ch < block_k / CK; ++ch) {
      const int key0 = j * block_k + ch * CK;
      if (key0 > row0 + RQ - 1) break;       // every key of the chunk is after every row
      __syncthreads();
      for (int i = threadIdx.x; i < CK * D; i += blockDim.x) {
        const int r = i / D, c = i % D;
        Ks[r * (D + 1) + c] = load_f32(kp, (size_t)(key0 + r) * D + c);
        Vs[r * D + c] = load_f32(vp, (size_t)(key0 + r) * D + c);
      }
      __syncthreads();
      float s[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) s[i][jj] = 0.f;
      for (int c = 0; c < D; ++c) {
        float qa[4], kb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) qa[i] = Qs[(4 * ty + i) * (D + 1) + c];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) kb[jj] = Ks[(tx + 16 * jj) * (D + 1) + c];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) s[i][jj] = fmaf(qa[i], kb[jj], s[i][jj]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = row0 + 4 * ty + i;
        float mx = -INFINITY;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int key = key0 + tx + 16 * jj;
          s[i][jj] = (key <= row) ? s[i][jj] * scale_log2 : -INFINITY;
          mx = fmaxf(mx, s[i][jj]);
        }
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float mn = fmaxf(m[i], mx);
        const float alpha = (mn == -INFINITY) ? 1.f : exp2f(m[i] - mn);
        float sum = 0.f;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float p = (mn == -INFINITY) ? 0.f : exp2f(s[i][jj] - mn);
          Ps[(4 * ty + i) * (CK + 1) + tx + 16 * jj] = p;
          sum += p;
        }
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        l[i] = l[i] * alpha + sum;
        m[i] = mn;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) o[i][c] *= alpha;
      }
      __syncthreads();
      for (int kk = 0; kk < CK; ++kk) {
        float pv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) pv[i] = Ps[(4 * ty + i) * (CK + 1) + kk];
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          const float vv = Vs[kk * D + tx + 16 * c];
#pragma unroll
          for (int i = 0; i < 4; ++i) o[i][c] = fmaf(pv[i], vv, o[i][c]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = row0 + 4 * ty + i;
    const float inv = l[i] > 0.f ? 1.f / l[i] : 0.f;
    T* op = out + ((size_t)bh * N + row) * D;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) store_out(op, tx + 16 * c, o[i][c] * inv);
    if (lse && tx == 0)
      lse[(size_t)bh * N + row] = l[i] > 0.f ? (m[i] + log2f(l[i])) * 0.69314718055994531f : -INFINITY;
  }
}

cudaError_t launch_attend_simt(const bsa_shape& s, const void* q, const void* k, const void* v,
                               const int32_t* kv_idx, const int32_t* kv_cnt, int W, float scale,
                               void* out, float* lse, int32_t* dev_status, cudaStream_t st) {
  dim3 grid(s.N / RQ, s.B * s.Hq);
  const float sl2 = scale * 1.4426950408889634f;
  cudaError_t e = cudaSuccess;
#define BSA_ATT_LAUNCH(T, D)                                                                    \
  do {                                                                                          \
    size_t smem = (size_t)(RQ * (D + 1) + CK * (D + 1) + CK * D + RQ * (CK + 1)) * 4;          \
    e = cudaFuncSetAttribute(attend_simt_kernel<T, D>,                                          \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);           \
    if (e != cudaSuccess) return e;                                                             \
    attend_simt_kernel<T, D><<<grid, 256, smem, st>>>(                                          \
        (const T*)q, (const T*)k, (const T*)v, kv_idx, kv_cnt, W, sl2, (T*)out, lse,            \
        dev_status, s.N, s.Hq, s.Hkv, s.tile_q, s.block_k);                                     \
  } while (0)
  if (s.dtype == BSA_BF16) {
    if (s.d == 128) BSA_ATT_LAUNCH(uint16_t, 128); else BSA_ATT_LAUNCH(uint16_t, 64);
  } else {
    if (s.d == 128) BSA_ATT_LAUNCH(float, 128); else BSA_ATT_LAUNCH(float, 64);
  }
#undef BSA_ATT_LAUNCH
  return cudaGetLastError();
}

}  // namespace bsa
