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
// warp's shared-memory slice holds only the histogram and the short list.
//
// Bucket path. A monotone fp32 map of each score onto 256 equal-width value
// buckets between the row's min and max (x >= y implies bucket(x) >= bucket(y),
// since correctly rounded subtraction and multiplication are monotone) gives a
// histogram in one pass, and from it the bucket holding the entry of rank
// need-1, need = max(M, m+1) capped at the row length. Every entry in that bucket
// or above is copied, in block order, to a short list; the list is regrouped by
// bucket, and each entry's exact rank is the number of entries in higher buckets
// plus the number in its own bucket that beat it (a greater score, or an equal
// score at a lower block index). The ranks give the top-M list, the top-m flag
// and the operands of sigma directly.
//
// Radix path, for rows the bucket path does not take (a non-finite score, all
// scores equal, a list longer than kListCap or a bucket larger than kBucketCap):
// exact radix selection on order-preserving 32-bit keys.

constexpr uint32_t kInTopM = 0x80000000u;   // flag on a ranked entry: inside the base top-m set
constexpr int kListCap = 256;                // longest list the bucket path takes
constexpr uint32_t kBucketCap = 96;          // largest bucket its pairwise count takes

struct RadixSel {
  uint32_t v;      // key of the element at the requested rank
  int take_eq;     // how many keys equal to v (lowest indices first) are inside the top r+1
};

// Key of the (r+1)-th largest among the keys of s[0..n), n >= r+1. Digits of 8 bits,
// starting below the bits every key of the row shares (so the first histogram spreads out).
__device__ RadixSel warp_radix_select(const float* s, int n, int r, uint32_t kmin, uint32_t kmax,
                                      uint32_t* hist, int lane) {
  int want = r + 1;
  if (kmin == kmax) return {kmax, want};
  const int hb = 31 - __clz(kmin ^ kmax);
  uint32_t mask = hb == 31 ? 0u : ~((2u << hb) - 1u);
  uint32_t prefix = kmax & mask;
  int lo = hb + 1;
  while (lo > 0) {
    const int width = lo < 8 ? lo : 8;
    const int shift = lo - width;
    const uint32_t dmask = (1u << width) - 1u;
#pragma unroll
    for (int k = 0; k < 8; ++k) hist[lane * 8 + k] = 0u;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const uint32_t u = score_key(__ldg(s + i));
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    __syncwarp();
    uint32_t h8[8], s = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) { h8[k] = hist[lane * 8 + k]; s += h8[k]; }
    uint32_t incl = s;                        // sum over lanes >= this lane
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
      if (lane + off < 32) incl += y;
    }
    uint32_t c = incl - s;                    // keys whose digit lies in higher lanes' bins
    int found = -1;
    uint32_t c_at = 0;
#pragma unroll
    for (int k = 7; k >= 0; --k) {
      if (found < 0 && c < (uint32_t)want && (uint32_t)want <= c + h8[k]) { found = lane * 8 + k; c_at = c; }
      c += h8[k];
    }
    const unsigned bal = __ballot_sync(0xffffffffu, found >= 0);
    const int src = __ffs(bal) - 1;
    const int dgt = __shfl_sync(0xffffffffu, found, src);
    const uint32_t cd = __shfl_sync(0xffffffffu, c_at, src);
    prefix |= (uint32_t)dgt << shift;
    mask |= dmask << shift;
    want -= (int)cd;
    lo = shift;
    __syncwarp();
  }
  return {prefix, want};
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = max(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ uint32_t warp_min_u32(uint32_t x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = min(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ int warp_min_i32(int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = min(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_min_f32(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_max_f32(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// sigma = (s_(m-1) - s_(m)) / (s_(0) - s_(m)) with correctly rounded fp32 operations.
__device__ __forceinline__ float cut_sigma(float s0, float a, float b) {
  const float num = __fsub_rn(a, b);
  const float den = __fsub_rn(s0, b);
  return (den == 0.0f) ? 0.0f : __fdiv_rn(num, den);
}

// Radix path for the row s[0..n), ranked on order-preserving keys. Writes the top-M list
// with the top-m flag to out and returns sigma (1 when the tile has no cut).
__device__ float rank_row_radix(uint32_t* hist, int n, const TileSlots& sl, const float* s,
                                int32_t* out, int lane) {
  uint32_t kmax = 0u, kmin = 0xffffffffu;
  for (int i = lane; i < n; i += 32) {
    const uint32_t u = score_key(__ldg(s + i));
    kmax = max(kmax, u);
    kmin = min(kmin, u);
  }
  kmax = warp_max_u32(kmax);
  kmin = warp_min_u32(kmin);
  const int m = sl.m, M = sl.M;
  RadixSel selm{0u, 0}, selM{0u, 0};
  if (m > 0 && m < n) selm = warp_radix_select(s, n, m - 1, kmin, kmax, hist, lane);
  if (M > m && M < n) selM = warp_radix_select(s, n, M - 1, kmin, kmax, hist, lane);
  else if (M == m) selM = selm;
  const bool all_m = m >= n, all_M = M >= n;

  // one pass in block order: compaction of the top-M list, sigma bookkeeping
  int base_M = 0, eq_m = 0, eq_M = 0;
  int idx0 = 0x7fffffff, idx_m1 = 0x7fffffff, idx_eqnext = 0x7fffffff, idx_below = 0x7fffffff;
  uint32_t below = 0u;
  bool have_below = false;
  const unsigned lt = (1u << lane) - 1u;
  for (int b0 = 0; b0 < n; b0 += 32) {
    const int i = b0 + lane;
    const bool live = i < n;
    const uint32_t u = live ? score_key(__ldg(s + i)) : 0u;
    const bool e_m = live && !all_m && m > 0 && u == selm.v;
    const unsigned bal_m = __ballot_sync(0xffffffffu, e_m);
    const int r_m = eq_m + __popc(bal_m & lt);
    const bool in_m = live && (all_m || (m > 0 && (u > selm.v || (e_m && r_m < selm.take_eq))));
    const bool e_M = live && !all_M && u == selM.v;
    const unsigned bal_M = __ballot_sync(0xffffffffu, e_M);
    const int r_M = eq_M + __popc(bal_M & lt);
    const bool in_M = live && M > 0 && (all_M || u > selM.v || (e_M && r_M < selM.take_eq));
    const unsigned bal_in = __ballot_sync(0xffffffffu, in_M);
    if (in_M) out[base_M + __popc(bal_in & lt)] = i | (in_m ? (int)kInTopM : 0);
    base_M += __popc(bal_in);
    if (live && u == kmax) idx0 = min(idx0, i);
    if (sl.cut) {
      if (e_m && r_m == selm.take_eq - 1) idx_m1 = i;
      if (e_m && r_m == selm.take_eq) idx_eqnext = i;
      if (live && u < selm.v && (!have_below || u > below || (u == below && i < idx_below))) {
        below = u;
        idx_below = i;
        have_below = true;
      }
    }
    eq_m += __popc(bal_m);
    eq_M += __popc(bal_M);
  }
  idx0 = warp_min_i32(idx0);
  if (!sl.cut) return 1.0f;
  idx_m1 = warp_min_i32(idx_m1);
  idx_eqnext = warp_min_i32(idx_eqnext);
  // rank m: the next equal key if the top-m set left one out, else the best key below
  int idx_m = idx_eqnext;
  if (idx_m == 0x7fffffff) {
    const uint32_t bmax = warp_max_u32(have_below ? below : 0u);
    const bool mine = have_below && below == bmax;
    idx_m = warp_min_i32(mine ? idx_below : 0x7fffffff);
  }
  return cut_sigma(s[idx0], s[idx_m1], s[idx_m]);
}

// Bin b of a 256-bin histogram lives at word (b % 8) * 32 + b / 8, so lane l's
// eight bins 8l..8l+7 are read and written without bank conflicts.
__device__ __forceinline__ int hidx(int b) { return ((b & 7) << 5) | (b >> 3); }

struct BucketMap {
  float lo, inv;
  // y = (x - lo) * inv >= 0 for x >= lo; both steps are monotone, so is the bucket
  __device__ __forceinline__ int operator()(float x) const {
    return __float2int_rz(fminf(__fmul_rn(__fsub_rn(x, lo), inv), 255.0f));
  }
};

// Per-warp shared-memory slice (words): histogram, bucket starts, the list, its scores,
// and the list regrouped by bucket (scores, positions). The row itself is not staged: each
// pass reads it from global memory (the second and third passes hit L2), which keeps the
// slice small: eight CTAs (32 warps) per SM, bounded by 64 registers per thread.
constexpr int kRankSliceWords = 512 + 4 * kListCap;
constexpr int kRankWarps = 4;                // rows (warps) per CTA

// Chunk c of a row holds its elements 4c..4c+3; those at or past n read as 0 (callers
// mask them). A chunk is one 16-byte load when the row is 16-byte aligned and the chunk
// lies wholly inside [0, n); otherwise its elements are loaded one by one.
struct RowChunks {
  const float* s;
  int n;
  bool al;
  __device__ __forceinline__ float4 operator()(int c) const {
    const int i0 = 4 * c;
    if (al && i0 + 3 < n) return __ldg(reinterpret_cast<const float4*>(s) + c);
    float4 v;
    v.x = i0 < n ? __ldg(s + i0) : 0.f;
    v.y = i0 + 1 < n ? __ldg(s + i0 + 1) : 0.f;
    v.z = i0 + 2 < n ? __ldg(s + i0 + 2) : 0.f;
    v.w = i0 + 3 < n ? __ldg(s + i0 + 3) : 0.f;
    return v;
  }
};

__device__ __forceinline__ float f4_at(const float4& v, int j) {
  return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}

// Writes, per row, the top-M candidates (M = expanded slots) in ascending block
// order with kInTopM set on the top-m ones (m = base slots; top-m is a prefix of
// the same ranking, so it is a subset), and sigma from ranks 0, m-1, m.
__global__ void __launch_bounds__(kRankWarps * 32, 8) select_rank_kernel(
    const float* __restrict__ scores, int rows_bh, int n_qt, int n_kb, int tile_q, int block_k,
    int k_first, int k_last, int rho, int R, int32_t* __restrict__ ranked, float* __restrict__ sigma,
    int32_t* dev_status) {
  extern __shared__ __align__(16) uint32_t wsm[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y * kRankWarps + warp;
  if (bh >= rows_bh) return;
  const int t = n_qt - 1 - (int)blockIdx.x;          // longest rows first
  uint32_t* hist = wsm + (size_t)warp * kRankSliceWords;
  uint32_t* start = hist + 256;
  uint32_t* list = start + 256;                      // block index | bucket << 16, then | rank << 16
  float* lv = reinterpret_cast<float*>(list + kListCap);    // the list's scores
  float* sv = lv + kListCap;                         // list regrouped by bucket: scores
  uint32_t* sp = reinterpret_cast<uint32_t*>(sv + kListCap);  // ... list position | block index << 16
  const size_t row = (size_t)bh * n_qt + t;
  const TileSlots sl = tile_slots(t, n_qt, tile_q, block_k, k_first, k_last, rho);
  const int n = sl.f_lo;
  const float* s = scores + row * n_kb;
  int32_t* out = ranked + row * R;
  if (n == 0) {
    if (lane == 0) sigma[row] = 1.0f;
    return;
  }
  const RowChunks rd{s, n, (reinterpret_cast<uintptr_t>(s) & 15) == 0};
  const int nc = (n + 3) >> 2;

  // the row's min, max and finiteness (four 16-byte loads per lane in flight)
  float xmin = INFINITY, xmax = -INFINITY;
  bool bad = false;
  for (int c0 = 0; c0 < nc; c0 += 128) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + u * 32 + lane;
      v[u] = c < nc ? rd(c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + u * 32 + lane;
      if (4 * c + 3 < n) {
        xmin = fminf(fminf(xmin, v[u].x), fminf(v[u].y, fminf(v[u].z, v[u].w)));
        xmax = fmaxf(fmaxf(xmax, v[u].x), fmaxf(v[u].y, fmaxf(v[u].z, v[u].w)));
        bad |= !(isfinite(v[u].x) && isfinite(v[u].y) && isfinite(v[u].z) && isfinite(v[u].w));
      } else if (c < nc) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (4 * c + j < n) {
            const float x = f4_at(v[u], j);
            xmin = fminf(xmin, x);
            xmax = fmaxf(xmax, x);
            bad |= !isfinite(x);
          }
        }
      }
    }
  }
  xmin = warp_min_f32(xmin);
  xmax = warp_max_f32(xmax);
  bad = __any_sync(0xffffffffu, bad);

  const int m = sl.m, M = sl.M;
  const int need = min(n, max(M, m + 1));
  const unsigned lt = (1u << lane) - 1u;
  bool radix = bad || !(xmax > xmin);
  float sg = 1.0f;
  int L = 0, bcut = 0;
  BucketMap bk{xmin, fminf(__fdiv_rn(256.0f, __fsub_rn(xmax, xmin)), 3.0e38f)};
  if (!radix) {
    // histogram of the buckets
#pragma unroll
    for (int k = 0; k < 8; ++k) hist[k * 32 + lane] = 0u;
    __syncwarp();
    for (int c0 = 0; c0 < nc; c0 += 128) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u * 32 + lane;
        v[u] = c < nc ? rd(c) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = 4 * (c0 + u * 32 + lane);
        if (i < n) atomicAdd(&hist[hidx(bk(v[u].x))], 1u);
        if (i + 1 < n) atomicAdd(&hist[hidx(bk(v[u].y))], 1u);
        if (i + 2 < n) atomicAdd(&hist[hidx(bk(v[u].z))], 1u);
        if (i + 3 < n) atomicAdd(&hist[hidx(bk(v[u].w))], 1u);
      }
    }
    __syncwarp();
    uint32_t h8[8], ab[8], sum = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) { h8[k] = hist[k * 32 + lane]; sum += h8[k]; }
    uint32_t incl = sum;                             // entries in the bins of lanes >= this lane
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
      if (lane + off < 32) incl += y;
    }
    uint32_t c = incl - sum;
    int found = -1;
    uint32_t len = 0;
#pragma unroll
    for (int k = 7; k >= 0; --k) {                   // ab[k]: entries in buckets above 8*lane+k
      ab[k] = c;
      if (ab[k] < (uint32_t)need && (uint32_t)need <= ab[k] + h8[k]) { found = lane * 8 + k; len = ab[k] + h8[k]; }
      c += h8[k];
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, found >= 0)) - 1;
    bcut = __shfl_sync(0xffffffffu, found, src);
    L = (int)__shfl_sync(0xffffffffu, len, src);
    uint32_t big = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (lane * 8 + k >= bcut) big = max(big, h8[k]);
      start[k * 32 + lane] = ab[k];
      hist[k * 32 + lane] = ab[k];                   // from here on: fill cursor of each bucket
    }
    big = warp_max_u32(big);
    radix = L > kListCap || big > kBucketCap;
    __syncwarp();
  }
  if (!radix) {
    // the list: every entry in bucket bcut or above, in block order, with its score
    int base = 0;
    for (int c0 = 0; c0 < nc; c0 += 128) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u * 32 + lane;
        v[u] = c < nc ? rd(c) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i0 = 4 * (c0 + u * 32 + lane);
        const float vv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        int bj[4], cnt = 0;
        bool sj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          bj[j] = bk(vv[j]);
          sj[j] = i0 + j < n && bj[j] >= bcut;
          cnt += sj[j] ? 1 : 0;
        }
        int inc = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, inc, off);
          if (lane >= off) inc += y;
        }
        int pos = base + inc - cnt;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (sj[j]) {
            list[pos] = (uint32_t)(i0 + j) | ((uint32_t)bj[j] << 16);
            lv[pos] = vv[j];
            ++pos;
          }
        base += __shfl_sync(0xffffffffu, inc, 31);
      }
    }
    __syncwarp();
    // regroup by bucket
    for (int p = lane; p < L; p += 32) {
      const uint32_t e = list[p];
      const uint32_t idx = e & 0xffffu;
      const uint32_t slot = atomicAdd(&hist[hidx((int)(e >> 16))], 1u);
      sv[slot] = lv[p];
      sp[slot] = (uint32_t)p | (idx << 16);
    }
    __syncwarp();
    // exact ranks: entries in higher buckets, plus those of the same bucket that beat this one
    for (int q = lane; q < L; q += 32) {
      const float v = sv[q];
      const uint32_t pk = sp[q];
      const uint32_t p = pk & 0xffffu, idx = pk >> 16;
      const int hb = hidx((int)(list[p] >> 16));
      const int lo = (int)start[hb], hi = (int)hist[hb];
      int r = lo;
      for (int u = lo; u < hi; ++u) {
        const float w = sv[u];
        r += (w > v || (w == v && (sp[u] >> 16) < idx)) ? 1 : 0;
      }
      list[p] = idx | ((uint32_t)r << 16);
    }
    __syncwarp();
    // the top-M list in block order with the top-m flag; sigma's operands by rank
    int base_M = 0, i_0 = 0x7fffffff, i_m1 = 0x7fffffff, i_m = 0x7fffffff;
    for (int p0 = 0; p0 < L; p0 += 32) {
      const int p = p0 + lane;
      const bool live = p < L;
      const uint32_t e = live ? list[p] : 0u;
      const int idx = (int)(e & 0xffffu), r = (int)(e >> 16);
      const bool in_M = live && r < M;
      const unsigned bal = __ballot_sync(0xffffffffu, in_M);
      if (in_M) out[base_M + __popc(bal & lt)] = idx | (r < m ? (int)kInTopM : 0);
      base_M += __popc(bal);
      if (live && r == 0) i_0 = idx;
      if (live && r == m - 1) i_m1 = idx;
      if (live && r == m) i_m = idx;
    }
    if (sl.cut) {
      i_0 = warp_min_i32(i_0);
      i_m1 = warp_min_i32(i_m1);
      i_m = warp_min_i32(i_m);
      sg = cut_sigma(__ldg(s + i_0), __ldg(s + i_m1), __ldg(s + i_m));
    }
  } else {
    sg = rank_row_radix(hist, n, sl, s, out, lane);
  }
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
