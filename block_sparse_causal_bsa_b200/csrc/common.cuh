// Internal helpers shared by the libbsa kernels (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/bsa.h"

namespace bsa {

// ---------------------------------------------------------------------------
// Tile geometry and budget. One definition, used by host validation and by the
// select / finalize kernels, so both sides agree on every slot count.
//
// Tile t covers query rows [t*tile_q, (t+1)*tile_q). Blocks f_lo..J intersect
// those rows and are always kept; blocks 0..f_lo-1 are the scored candidates
// ([UGS] step 2: selection per query tile; the diagonal block is kept for
// causal self-visibility). The budget k_t is fixed or the linear
// position-decay budget of [Stem] 2.A; expansion multiplies it by rho
// ([UGS] step 5). Both are capped at the J+1 visible blocks and never drop
// the forced ones.
struct TileSlots {
  int f_lo;     // first forced block == number of candidates
  int J;        // last visible block
  int nF;       // forced blocks
  int m;        // candidate slots at the base budget
  int M;        // candidate slots at the expanded budget
  bool cut;     // more candidates than base slots, and at least one slot
};

__host__ __device__ inline int budget_k(int t, int n_qt, int k_first, int k_last) {
  if (n_qt <= 1 || k_first == k_last) return k_first;
  // k_first >= k_last, so the quotient is non-negative and truncation is floor.
  long long num = (long long)(k_first - k_last) * (long long)t;
  return k_first - (int)(num / (long long)(n_qt - 1));
}

__host__ __device__ inline TileSlots tile_slots(int t, int n_qt, int tile_q, int block_k,
                                                int k_first, int k_last, int rho) {
  TileSlots s;
  s.f_lo = (int)(((long long)t * tile_q) / block_k);
  s.J = (int)(((long long)(t + 1) * tile_q - 1) / block_k);
  s.nF = s.J - s.f_lo + 1;
  int k = budget_k(t, n_qt, k_first, k_last);
  int vis = s.J + 1;
  int K = k < vis ? k : vis;
  if (K < s.nF) K = s.nF;
  long long kr = (long long)rho * k;
  int KM = kr < vis ? (int)kr : vis;
  if (KM < s.nF) KM = s.nF;
  s.m = K - s.nF;
  s.M = KM - s.nF;
  s.cut = (s.f_lo > s.m) && (s.m >= 1);
  return s;
}

__host__ __device__ inline int kv_width(int N, int tile_q, int block_k, int k_first, int k_last,
                                        int rho) {
  int n_kb = N / block_k;
  int f_max = tile_q / block_k;
  if (f_max < 1) f_max = 1;
  long long w = (long long)rho * (k_first > k_last ? k_first : k_last);
  if (w < f_max) w = f_max;
  if (w > n_kb) w = n_kb;
  return (int)w;
}

// ---------------------------------------------------------------------------
// Loads

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

template <typename T> __device__ __forceinline__ float load_f32(const T* p, size_t i);
template <> __device__ __forceinline__ float load_f32<float>(const float* p, size_t i) {
  return p[i];
}
template <> __device__ __forceinline__ float load_f32<uint16_t>(const uint16_t* p, size_t i) {
  return bf16_to_f32(p[i]);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

template <typename T> __device__ __forceinline__ void store_out(T* p, size_t i, float x);
template <> __device__ __forceinline__ void store_out<float>(float* p, size_t i, float x) { p[i] = x; }
template <> __device__ __forceinline__ void store_out<uint16_t>(uint16_t* p, size_t i, float x) {
  p[i] = f32_to_bf16_rn(x);
}

__device__ __forceinline__ void set_status(int32_t* st, int bit) {
  if (st) atomicOr(st, bit);
}

// One warp: copies the valid entries (0 <= j < n_blocks) of a decode visit list
// lst[0..cnt) into out[] in list order and returns their number on every lane;
// invalid entries are dropped and reported as BSA_DEV_BAD_INDEX. cnt outside
// [0, cap] is reported too and clamped.
__device__ inline int warp_compact_blocks(const int32_t* lst, int cnt, int cap, int n_blocks,
                                          uint16_t* out, int32_t* dev_status, int lane) {
  if (cnt < 0 || cnt > cap) {
    if (lane == 0) set_status(dev_status, BSA_DEV_BAD_INDEX);
    cnt = cnt < 0 ? 0 : cap;
  }
  int n = 0;
  for (int base = 0; base < cnt; base += 32) {
    const int i = base + lane;
    const int j = i < cnt ? lst[i] : -1;
    const bool valid = i < cnt && j >= 0 && j < n_blocks;
    const unsigned m = __ballot_sync(0xffffffffu, valid);
    if (__any_sync(0xffffffffu, i < cnt && !valid) && lane == 0) set_status(dev_status, BSA_DEV_BAD_INDEX);
    if (valid) out[n + __popc(m & ((1u << lane) - 1u))] = (uint16_t)j;
    n += __popc(m);
  }
  return n;
}

// Sum over a warp of fp64 terms in the order the [ART] 2.2 probe sums take here: each
// lane passes the rounded sum of its two terms (probe coordinates lane and lane + 32, zero
// where there is none); the values 16, 8, 4, 2 and 1 lanes apart are then added, each add
// rounded. Every lane returns the same sum (fp64 addition is commutative).
__device__ __forceinline__ double warp_pairwise_sum(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// Order-preserving map of an fp32 score to uint32 (larger score -> larger key).
// -0.0 is folded into +0.0 so that equal scores compare equal, as IEEE does.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace bsa
