// Vertical-slash index preparation ([VSP] Metodologia A and B.3).
//
// A query row i attends to the vertical columns j <= i and to the keys i - o of
// the slash offsets o <= i, each key once. The attention kernel works on key
// blocks of 64, so the two index lists are turned into
//   - per (b, h) two bitmaps over positions: V (bit j set for a vertical column
//     j) and S (bit o set for a slash offset o), N/64 + 1 words each (the extra
//     zero word lets a 64-bit window start anywhere);
//   - per (b, h, query tile) the ascending list of the key blocks that hold at
//     least one key of any row of the tile: the blocks with a vertical column,
//     merged with the blocks each slash diagonal crosses inside the tile
//     (rows i0..i0+127 see keys i0-o .. i0+127-o). The merge runs on a bitmap of
//     the tile's blocks, so the list comes out sorted and without duplicates.
// The attention kernel then masks each (row, key) pair with the V and S bits.
// Out-of-range entries (outside [0, N)) are dropped and reported as
// BSA_DEV_BAD_INDEX; a count outside [0, width] is reported and clamped.
#include "common.cuh"
#include "kernels.h"

namespace bsa {

namespace {

__device__ __forceinline__ int clamp_count(int c, int w, int32_t* dev_status) {
  if (c < 0 || c > w) {
    set_status(dev_status, BSA_DEV_BAD_INDEX);
    return c < 0 ? 0 : w;
  }
  return c;
}

// One CTA per (b, h): both bitmaps.
__global__ void __launch_bounds__(256) vs_bitmap_kernel(const int32_t* __restrict__ v_idx,
                                                        const int32_t* __restrict__ v_cnt, int Wv,
                                                        const int32_t* __restrict__ s_off,
                                                        const int32_t* __restrict__ s_cnt, int Ws,
                                                        int N, unsigned long long* __restrict__ vbits,
                                                        unsigned long long* __restrict__ sbits,
                                                        int32_t* dev_status) {
  const int bh = blockIdx.x;
  const int words = N / 64 + 1;
  unsigned long long* vb = vbits + (size_t)bh * words;
  unsigned long long* sb = sbits + (size_t)bh * words;
  for (int i = threadIdx.x; i < words; i += blockDim.x) {
    vb[i] = 0ull;
    sb[i] = 0ull;
  }
  __syncthreads();
  const int nv = clamp_count(v_cnt[bh], Wv, threadIdx.x == 0 ? dev_status : nullptr);
  const int ns = clamp_count(s_cnt[bh], Ws, threadIdx.x == 0 ? dev_status : nullptr);
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const int j = v_idx[(size_t)bh * Wv + i];
    if (j >= 0 && j < N) atomicOr(vb + (j >> 6), 1ull << (j & 63));
    else set_status(dev_status, BSA_DEV_BAD_INDEX);
  }
  for (int i = threadIdx.x; i < ns; i += blockDim.x) {
    const int o = s_off[(size_t)bh * Ws + i];
    if (o >= 0 && o < N) atomicOr(sb + (o >> 6), 1ull << (o & 63));
    else set_status(dev_status, BSA_DEV_BAD_INDEX);
  }
}

// One warp per (b, h, query tile): the ascending list of key blocks (of 64) that
// hold a key of some row of the tile.
__global__ void __launch_bounds__(256) vs_lists_kernel(const unsigned long long* __restrict__ vbits,
                                                       const int32_t* __restrict__ s_off,
                                                       const int32_t* __restrict__ s_cnt, int Ws,
                                                       int rows_bh, int N, int tile_q, int Wl,
                                                       int32_t* __restrict__ lists,
                                                       int32_t* __restrict__ counts) {
  extern __shared__ uint32_t tb_all[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.y * (blockDim.x / 32) + warp;
  if (bh >= rows_bh) return;
  const int t = blockIdx.x;
  const int n_qt = N / tile_q, n_kb = N / 64;
  const int nw = (n_kb + 31) / 32;
  uint32_t* tb = tb_all + (size_t)warp * nw;
  const int i0 = t * tile_q, i1 = i0 + tile_q - 1;
  const int J = i1 / 64;
  for (int w = lane; w < nw; w += 32) tb[w] = 0u;
  __syncwarp();
  // vertical: the blocks whose V word has a bit set (each block is one word)
  const unsigned long long* vb = vbits + (size_t)bh * (N / 64 + 1);
  for (int b = lane; b <= J; b += 32)
    if (vb[b] != 0ull) atomicOr(tb + (b >> 5), 1u << (b & 31));
  // slash: offset o covers keys max(0, i0-o) .. i1-o of this tile's rows
  int ns = s_cnt[bh];
  ns = ns < 0 ? 0 : (ns > Ws ? Ws : ns);
  for (int i = lane; i < ns; i += 32) {
    const int o = s_off[(size_t)bh * Ws + i];
    if (o < 0 || o >= N || o > i1) continue;
    const int lo = (i0 - o < 0 ? 0 : i0 - o) >> 6, hi = (i1 - o) >> 6;
    for (int b = lo; b <= hi; ++b) atomicOr(tb + (b >> 5), 1u << (b & 31));
  }
  __syncwarp();
  // compaction in block order
  int32_t* out = lists + ((size_t)bh * n_qt + t) * Wl;
  int n = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int b0 = 0; b0 <= J; b0 += 32) {
    const int b = b0 + lane;
    const bool set = b <= J && ((tb[b >> 5] >> (b & 31)) & 1u);
    const unsigned m = __ballot_sync(0xffffffffu, set);
    const int pos = n + __popc(m & lt);
    if (set && pos < Wl) out[pos] = b;
    n += __popc(m);
  }
  for (int p = n + lane; p < Wl; p += 32) out[p] = -1;
  if (lane == 0) counts[(size_t)bh * n_qt + t] = n < Wl ? n : Wl;
}

}  // namespace

cudaError_t launch_vs_prep(const bsa_shape& s, const int32_t* v_idx, const int32_t* v_cnt, int Wv,
                           const int32_t* s_off, const int32_t* s_cnt, int Ws, int Wl,
                           unsigned long long* vbits, unsigned long long* sbits, int32_t* lists,
                           int32_t* counts, int32_t* dev_status, cudaStream_t st) {
  const int rows_bh = s.B * s.Hq;
  vs_bitmap_kernel<<<rows_bh, 256, 0, st>>>(v_idx, v_cnt, Wv, s_off, s_cnt, Ws, s.N, vbits, sbits,
                                            dev_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n_qt = s.N / s.tile_q;
  const int nw = (s.N / 64 + 31) / 32;
  dim3 grid(n_qt, (rows_bh + 7) / 8);
  vs_lists_kernel<<<grid, 256, (size_t)8 * nw * 4, st>>>(vbits, s_off, s_cnt, Ws, rows_bh, s.N,
                                                         s.tile_q, Wl, lists, counts);
  return cudaGetLastError();
}

}  // namespace bsa
