// Exact per-row top-M ranking of block scores by one warp ([UGS] steps 2-3):
// candidates 0..n-1 ordered by (score desc, index asc), the top-M written in
// ascending block order with the top-m ones flagged, and the cut margin
// sigma = (s_(m-1) - s_(m)) / (s_(0) - s_(m)) in fp32 with correctly rounded
// operations on the scores read back by index.
//
// Shared by the standalone selection kernel (rows read from a scores array
// that is read-only for the launch: NC = true, non-coherent loads) and by the
// fused score+rank kernel (rows its own epilogue warps wrote during the launch:
// NC = false, plain coherent loads after an mbarrier acquire).
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
#pragma once

#include <math.h>

#include "common.cuh"

namespace bsa {

constexpr uint32_t kInTopM = 0x80000000u;   // flag on a ranked entry: inside the base top-m set
constexpr int kListCap = 256;                // longest list the bucket path takes
constexpr uint32_t kBucketCap = 96;          // largest bucket its pairwise count takes
// Per-warp shared-memory slice (words): histogram, bucket starts, the list, its scores,
// and the list regrouped by bucket (scores, positions).
constexpr int kRankSliceWords = 512 + 4 * kListCap;

template <bool NC>
__device__ __forceinline__ float ld_row(const float* p) {
  if constexpr (NC) return __ldg(p);
  else return *p;
}
template <bool NC>
__device__ __forceinline__ float4 ld_row4(const float* p) {
  if constexpr (NC) return __ldg(reinterpret_cast<const float4*>(p));
  else return *reinterpret_cast<const float4*>(p);
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

struct RadixSel {
  uint32_t v;      // key of the element at the requested rank
  int take_eq;     // how many keys equal to v (lowest indices first) are inside the top r+1
};

// Key of the (r+1)-th largest among the keys of s[0..n), n >= r+1. Digits of 8 bits,
// starting below the bits every key of the row shares (so the first histogram spreads out).
template <bool NC>
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
      const uint32_t u = score_key(ld_row<NC>(s + i));
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1u);
    }
    __syncwarp();
    uint32_t h8[8], sum = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) { h8[k] = hist[lane * 8 + k]; sum += h8[k]; }
    uint32_t incl = sum;                      // sum over lanes >= this lane
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, incl, off);
      if (lane + off < 32) incl += y;
    }
    uint32_t c = incl - sum;                  // keys whose digit lies in higher lanes' bins
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

// sigma = (s_(m-1) - s_(m)) / (s_(0) - s_(m)) with correctly rounded fp32 operations.
__device__ __forceinline__ float cut_sigma(float s0, float a, float b) {
  const float num = __fsub_rn(a, b);
  const float den = __fsub_rn(s0, b);
  return (den == 0.0f) ? 0.0f : __fdiv_rn(num, den);
}

// Radix path for the row s[0..n), ranked on order-preserving keys. Writes the top-M list
// with the top-m flag to out and returns sigma (1 when the tile has no cut).
template <bool NC>
__device__ float rank_row_radix(uint32_t* hist, int n, const TileSlots& sl, const float* s,
                                int32_t* out, int lane) {
  uint32_t kmax = 0u, kmin = 0xffffffffu;
  for (int i = lane; i < n; i += 32) {
    const uint32_t u = score_key(ld_row<NC>(s + i));
    kmax = max(kmax, u);
    kmin = min(kmin, u);
  }
  kmax = warp_max_u32(kmax);
  kmin = warp_min_u32(kmin);
  const int m = sl.m, M = sl.M;
  RadixSel selm{0u, 0}, selM{0u, 0};
  if (m > 0 && m < n) selm = warp_radix_select<NC>(s, n, m - 1, kmin, kmax, hist, lane);
  if (M > m && M < n) selM = warp_radix_select<NC>(s, n, M - 1, kmin, kmax, hist, lane);
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
    const uint32_t u = live ? score_key(ld_row<NC>(s + i)) : 0u;
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
  return cut_sigma(ld_row<NC>(s + idx0), ld_row<NC>(s + idx_m1), ld_row<NC>(s + idx_m));
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

// Chunk c of a row holds its elements 4c..4c+3; those at or past n read as 0 (callers
// mask them). A chunk is one 16-byte load when the row is 16-byte aligned and the chunk
// lies wholly inside [0, n); otherwise its elements are loaded one by one.
template <bool NC>
struct RowChunks {
  const float* s;
  int n;
  bool al;
  __device__ __forceinline__ float4 operator()(int c) const {
    const int i0 = 4 * c;
    if (al && i0 + 3 < n) return ld_row4<NC>(s + i0);
    float4 v;
    v.x = i0 < n ? ld_row<NC>(s + i0) : 0.f;
    v.y = i0 + 1 < n ? ld_row<NC>(s + i0 + 1) : 0.f;
    v.z = i0 + 2 < n ? ld_row<NC>(s + i0 + 2) : 0.f;
    v.w = i0 + 3 < n ? ld_row<NC>(s + i0 + 3) : 0.f;
    return v;
  }
};

__device__ __forceinline__ float f4_at(const float4& v, int j) {
  return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}

// The row's min, max and whether any entry is non-finite (four 16-byte loads per lane
// in flight); every lane receives the result.
template <bool NC>
__device__ void row_minmax(const float* s, int n, int lane, float& xmin_out, float& xmax_out,
                           bool& bad_out) {
  const RowChunks<NC> rd{s, n, (reinterpret_cast<uintptr_t>(s) & 15) == 0};
  const int nc = (n + 3) >> 2;
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
  xmin_out = warp_min_f32(xmin);
  xmax_out = warp_max_f32(xmax);
  bad_out = __any_sync(0xffffffffu, bad);
}

// Ranks the candidates s[0..n), n >= 1, of one (b, h, tile) row, given the row's min,
// max and non-finite flag (every lane must pass the same values). Writes the top-M
// entries (M = expanded slots) to out in ascending block order with kInTopM on the
// top-m ones (top-m is a prefix of the same ranking, so it is a subset), and returns
// sigma from ranks 0, m-1, m (1 for a tile with no cut). With bad set, the radix path
// runs (its order on non-finite keys is still total) and the caller reports the row.
// slice: this warp's kRankSliceWords words of shared memory.
template <bool NC>
__device__ float rank_row(const float* s, int n, const TileSlots& sl, float xmin, float xmax,
                          bool bad, uint32_t* slice, int32_t* out, int lane) {
  uint32_t* hist = slice;
  uint32_t* start = hist + 256;
  uint32_t* list = start + 256;                      // block index | bucket << 16, then | rank << 16
  float* lv = reinterpret_cast<float*>(list + kListCap);    // the list's scores
  float* sv = lv + kListCap;                         // list regrouped by bucket: scores
  uint32_t* sp = reinterpret_cast<uint32_t*>(sv + kListCap);  // ... list position | block index << 16
  const RowChunks<NC> rd{s, n, (reinterpret_cast<uintptr_t>(s) & 15) == 0};
  const int nc = (n + 3) >> 2;
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
      sg = cut_sigma(ld_row<NC>(s + i_0), ld_row<NC>(s + i_m1), ld_row<NC>(s + i_m));
    }
    __syncwarp();                                    // the slice is reused by the next row
  } else {
    sg = rank_row_radix<NC>(hist, n, sl, s, out, lane);
    __syncwarp();
  }
  return sg;
}


}  // namespace bsa
