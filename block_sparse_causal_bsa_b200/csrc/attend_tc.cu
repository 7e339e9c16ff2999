// Block-sparse causal attention on Blackwell tensor cores (tcgen05 + TMEM + TMA).
//
// O_i = sum over the keys j of the listed blocks with j <= i of
// softmax(scale * q_i . k_j) v_j -- the sparse aggregation step of [UGS]
// step 5 and [Stem] Implementação: only the blocks in kv_idx are streamed,
// with an online softmax. Shapes: bf16, d = 128, key blocks of 64, query
// tiles of 128.
//
// One CTA per (batch, query head, query tile); 352 threads in four roles:
//   warp 0 (one thread)  TMA producer: the Q tile once, then K and V tiles of
//                        128 keys = two listed blocks gathered into adjacent
//                        shared-memory rows, two stages deep.
//   warps 1, 10          MMA issuers, one thread each, one per half tile (= one
//                        listed block): S_h = Q K_h^T (N = 64) into the half's
//                        part of one of two TMEM S buffers (the next tile's S_h is
//                        issued before this tile's value product), then
//                        O_h += P_h V_h into the half's own TMEM accumulator once
//                        the half's P is written, with P_h read straight from
//                        tensor memory. The two halves run as separate pipelines.
//   warps 2-9            softmax: two warps per TMEM lane quarter; a thread owns
//                        half of one query row (the 64 keys of one listed block)
//                        and runs an independent online softmax over the blocks
//                        it sees: running max and sum of its half only, its own
//                        O_h accumulator, rescaled in TMEM only when its running
//                        max grew by more than 2^8 (exact: l and O keep the same
//                        stale max). No per-tile exchange between the halves.
//                        P_h (bf16, two per 32-bit column) is stored with
//                        tcgen05.st over the first 32 columns of the half's S
//                        region, which the softmax has just read.
//                        Epilogue: the two halves meet once, through shared
//                        memory: m = max(m0, m1), l = l0 2^(m0-m) + l1 2^(m1-m),
//                        O = (O_0 2^(m0-m) + O_1 2^(m1-m)) / l  -- the exact merge
//                        of two softmax partial sums; each half writes 64 of the
//                        128 output columns (and lse).
// Shared-memory operand layouts (128-byte swizzled, as TMA writes them):
//   Q, K: K-major [rows x 64 elements] halves; V: MN-major (rows = keys, 64
//   contiguous head dims per 128-byte row).
// TMEM: S buffers at columns 0 and 128 (half h at +64h; its P over the first 32
// of those columns once read), O_0 at 256, O_1 at 384.
// The CTA-to-work mapping walks (batch, KV head) outermost and the query heads
// of a group innermost, so CTAs running together gather from one KV head and
// reuse its blocks through L2.
// Every mbarrier wait is bounded (tc::mbar_wait); a timeout sets
// BSA_DEV_TIMEOUT, the CTA unwinds, waits for its own copies and MMAs, and
// frees its TMEM. Invalid kv_idx entries are dropped with BSA_DEV_BAD_INDEX.
// Vertical-slash variant (VS, [VSP] B.3): the block list covers the tile's
// vertical columns and slash diagonals, and each (row i, key j) pair is kept
// only if j <= i and (j is a vertical column or i - j is a slash offset), read
// from per-head bitmaps: a 64-bit word of V per key block, and a 64-bit window
// of S (bit-reversed) for the offsets i-j of the block's keys.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace bsa {

namespace {
constexpr int BQ = 128;          // query rows per tile
constexpr int BKB = 64;          // keys per listed block
constexpr int HD = 128;          // head dim
constexpr int NS = 2;            // K/V pipeline stages
constexpr int kThreads = 352;
constexpr int kSoftmaxWarps = 8;
constexpr int kMaxList = 1024;   // kv_idx entries staged per tile
constexpr uint32_t kHalf = 16384;            // [128 rows x 128 bytes]
constexpr uint32_t kTile = 2 * kHalf;        // 128 rows x 128 dims bf16
constexpr uint32_t kBoxK = 8192;             // one 64-key block half
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;                // S buffers at columns 0 and 128
constexpr uint32_t kColO = 256;              // O_0 at 256, O_1 at 384

struct __align__(8) Ctrl {
  uint64_t q_full;
  uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  uint64_t s_full[2][2];                 // [half][buffer]
  uint64_t p_full[2], o_ready[2];         // per half tile
  uint64_t done[2];
  uint64_t lbar[4];                 // per lane quarter: both halves' (m, l) written (once)
  uint32_t tmem;
  int abort_flag;
  int n_list;
  float mpart[2][128];              // [half][row] final running max of the half
  float lpart[2][128];              // [half][row] final row-sum part of the half
  int list[kMaxList];
};

constexpr size_t kSmemQ = 0;
constexpr size_t kSmemK = kSmemQ + kTile;
constexpr size_t kSmemV = kSmemK + NS * kTile;
constexpr size_t kSmemCtrl = kSmemV + NS * kTile;
constexpr size_t kSmemBytes = kSmemCtrl + sizeof(Ctrl) + 1024;   // + alignment slack

__device__ __forceinline__ bool warp_all(bool x) { return __all_sync(0xffffffffu, x); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Keys j0+u (u < 64) of block blk that row i keeps under the vertical-slash rule:
// causal (u <= i-j0) and (bit j of V, or bit i-j of S). Bitmaps have N/64+1 words.
__device__ __forceinline__ uint64_t vs_keep(const unsigned long long* __restrict__ vrow,
                                            const unsigned long long* __restrict__ srow, int i,
                                            int blk) {
  const int rel = i - blk * BKB;
  if (rel < 0) return 0ull;
  const uint64_t causal = rel >= 63 ? ~0ull : ((2ull << rel) - 1ull);
  const uint64_t v = __ldg(vrow + blk) & causal;
  // window w: bit k <-> offset base + k; key u sits on offset rel - u = base + 63 - u
  const int base = rel - 63;
  uint64_t w;
  if (base >= 0) {
    const int q = base >> 6, r = base & 63;
    const uint64_t a = __ldg(srow + q);
    w = r ? ((a >> r) | (__ldg(srow + q + 1) << (64 - r))) : a;
  } else {
    w = __ldg(srow) << (-base);                      // offsets below 0 do not exist
  }
  return v | __brevll(w);
}
}  // namespace

template <bool VS>
__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(
    const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
    const __grid_constant__ CUtensorMap tmv, const int32_t* __restrict__ kv_idx,
    const int32_t* __restrict__ kv_cnt, int W, float scale_log2, uint16_t* __restrict__ out,
    float* __restrict__ lse, int32_t* dev_status, int N, int Hq, int Hkv, int n_qt, int n_kb,
    const unsigned long long* __restrict__ vbits, const unsigned long long* __restrict__ sbits) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl& c = *reinterpret_cast<Ctrl*>(sm + kSmemCtrl);
  const uint32_t sQ = tc::smem_u32(sm + kSmemQ);
  const uint32_t sK = tc::smem_u32(sm + kSmemK);
  const uint32_t sV = tc::smem_u32(sm + kSmemV);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = Hq / Hkv;
  int x = blockIdx.x;
  const int hh = x % G;
  x /= G;
  const int t = n_qt - 1 - (x % n_qt);
  const int bgi = x / n_qt;                 // b * Hkv + g
  const int b = bgi / Hkv, g = bgi % Hkv;
  const int h = g * G + hh;
  const size_t bh = (size_t)b * Hq + h;
  const size_t krow = bh * n_qt + t;
  const int J = ((t + 1) * BQ - 1) / BKB;   // last visible block
  const int q_row0 = (int)(bh * N + (size_t)t * BQ);
  const int kv_row0 = bgi * N;

  if (threadIdx.x == 0) {
    tc::mbar_init(&c.q_full, 1);
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&c.k_full[s], 1);
      tc::mbar_init(&c.k_empty[s], 2);      // both halves' S products read the K tile
      tc::mbar_init(&c.v_full[s], 1);
      tc::mbar_init(&c.v_empty[s], 2);      // both halves' value products read the V tile
    }
    for (int i = 0; i < 2; ++i) {
      for (int bfi = 0; bfi < 2; ++bfi) tc::mbar_init(&c.s_full[i][bfi], 1);
      tc::mbar_init(&c.p_full[i], kSoftmaxWarps / 2);
      tc::mbar_init(&c.o_ready[i], 1);
      tc::mbar_init(&c.done[i], 1);
    }
    for (int q = 0; q < 4; ++q) tc::mbar_init(&c.lbar[q], 2);
    c.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&c.tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == 2) {
    // compact the valid entries of this tile's kv_idx row into shared memory
    int cnt = kv_cnt[krow];
    if (cnt < 0 || cnt > W) {
      if (lane == 0) set_status(dev_status, BSA_DEV_BAD_INDEX);
      cnt = cnt < 0 ? 0 : W;
    }
    int n = 0;
    for (int base = 0; base < cnt; base += 32) {
      const int i = base + lane;
      const int j = i < cnt ? kv_idx[krow * W + i] : -1;
      const bool valid = i < cnt && j >= 0 && j < n_kb && j <= J;
      const unsigned m = __ballot_sync(0xffffffffu, valid);
      if (__any_sync(0xffffffffu, i < cnt && !valid) && lane == 0) set_status(dev_status, BSA_DEV_BAD_INDEX);
      if (valid) c.list[n + __popc(m & ((1u << lane) - 1u))] = j;
      n += __popc(m);
    }
    if (lane == 0) c.n_list = n;
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = c.tmem;
  const int nl = c.n_list;
  const int ntiles = (nl + 1) / 2;
  volatile int* abort_flag = &c.abort_flag;
  int k_issued = 0, v_issued = 0;     // tiles whose K / V loads the producer issued
  bool mma_issued = false;

  if (warp == 0 && lane == 0 && ntiles > 0) {
    // ---------------- TMA producer ----------------
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
    tc::mbar_arrive_expect_tx(&c.q_full, kTile);
    tc::tma_load_2d(sm + kSmemQ, &tmq, 0, q_row0, &c.q_full);
    tc::tma_load_2d(sm + kSmemQ + kHalf, &tmq, 64, q_row0, &c.q_full);
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % NS;
      const int ja = c.list[2 * j];
      const int jb = (2 * j + 1 < nl) ? c.list[2 * j + 1] : ja;
      const int ra = kv_row0 + ja * BKB, rb = kv_row0 + jb * BKB;
      if (j >= NS && !tc::mbar_wait(&c.k_empty[s], ((j / NS) - 1) & 1, abort_flag, dev_status)) break;
      uint8_t* kd = sm + kSmemK + s * kTile;
      tc::mbar_arrive_expect_tx(&c.k_full[s], kTile);
      tc::tma_load_2d(kd, &tmk, 0, ra, &c.k_full[s]);
      tc::tma_load_2d(kd + kBoxK, &tmk, 0, rb, &c.k_full[s]);
      tc::tma_load_2d(kd + kHalf, &tmk, 64, ra, &c.k_full[s]);
      tc::tma_load_2d(kd + kHalf + kBoxK, &tmk, 64, rb, &c.k_full[s]);
      k_issued = j + 1;
      if (j >= NS && !tc::mbar_wait(&c.v_empty[s], ((j / NS) - 1) & 1, abort_flag, dev_status)) break;
      uint8_t* vd = sm + kSmemV + s * kTile;
      tc::mbar_arrive_expect_tx(&c.v_full[s], kTile);
      tc::tma_load_2d(vd, &tmv, 0, ra, &c.v_full[s]);
      tc::tma_load_2d(vd + kBoxK, &tmv, 0, rb, &c.v_full[s]);
      tc::tma_load_2d(vd + kHalf, &tmv, 64, ra, &c.v_full[s]);
      tc::tma_load_2d(vd + kHalf + kBoxK, &tmv, 64, rb, &c.v_full[s]);
      v_issued = j + 1;
    }
  } else if ((warp == 1 || warp == 10) && lane == 0 && ntiles > 0) {
    // ---------------- MMA issuer of one half ----------------
    const int hf = warp == 1 ? 0 : 1;
    constexpr uint32_t idS = tc::idesc_bf16_f32(128, 64, false, false);
    constexpr uint32_t idPV = tc::idesc_bf16_f32(128, 128, false, true);
    auto issue_s = [&](int j) {
      // S_h = Q (128 x d) . K_h^T, K_h = rows 64*hf .. 64*hf+63 of the K tile
      const uint32_t kb = sK + (j % NS) * kTile + hf * kBoxK;
      const uint32_t d = tmem + kColS + (j % 2) * 128 + hf * 64;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
        tc::umma_bf16(d, tc::sdesc_sw128(sQ + off, 16, 1024), tc::sdesc_sw128(kb + off, 16, 1024), idS,
                      kk > 0);
      }
      tc::umma_commit(&c.s_full[hf][j % 2]);
      tc::umma_commit(&c.k_empty[j % NS]);
    };
    bool ok = tc::mbar_wait(&c.q_full, 0, abort_flag, dev_status) &&
              tc::mbar_wait(&c.k_full[0], 0, abort_flag, dev_status);
    if (ok) {
      tc::tc_fence_after();
      issue_s(0);
      mma_issued = true;
    }
    for (int j = 0; ok && j < ntiles; ++j) {
      const int jn = j + 1;
      if (jn < ntiles) {
        // S_h(jn) overwrites the buffer of tile jn-2, whose P this half's value
        // product of tile jn-2 = j-1 reads: wait for that product to complete
        // (which also implies the softmax read S there)
        ok = tc::mbar_wait(&c.k_full[jn % NS], (jn / NS) & 1, abort_flag, dev_status) &&
             (jn < 2 || tc::mbar_wait(&c.o_ready[hf], (jn - 2) & 1, abort_flag, dev_status));
        if (!ok) break;
        tc::tc_fence_after();
        issue_s(jn);
      }
      ok = tc::mbar_wait(&c.v_full[j % NS], (j / NS) & 1, abort_flag, dev_status) &&
           tc::mbar_wait(&c.p_full[hf], j & 1, abort_flag, dev_status);
      if (!ok) break;
      tc::tc_fence_after();
      const uint32_t vb = sV + (j % NS) * kTile;
      const uint32_t pa = tmem + kColS + (j % 2) * 128 + hf * 64;    // P_h in TMEM
      // O_h += P_h (128 rows x 64 keys) . V rows of this half's block
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        tc::umma_bf16_ts(tmem + kColO + hf * 128, pa + kk * 8,
                         tc::sdesc_sw128(vb + (hf * 4 + kk) * 2048, kHalf, 1024), idPV,
                         (j > 0 || kk > 0) ? 1u : 0u);
      }
      tc::umma_commit(&c.o_ready[hf]);
      tc::umma_commit(&c.v_empty[j % NS]);
    }
  } else if (warp >= 2 && warp <= 9) {
    // ---------------- softmax warps ----------------
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;                   // 0: keys 0-63 of the tile, 1: keys 64-127
    const int r = quarter * 32 + lane;                  // row in the tile == TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t colO = kColO + half * 128;
    const int row_abs = t * BQ + r;
    const unsigned long long* vrow = VS ? vbits + bh * (size_t)(N / 64 + 1) : nullptr;
    const unsigned long long* srow = VS ? sbits + bh * (size_t)(N / 64 + 1) : nullptr;
    float m_used = -INFINITY;                           // running max of this half, scaled log2 units
    float l = 0.f;                                      // running sum of this half
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      ok = warp_all(tc::mbar_wait(&c.s_full[half][j % 2], (j / 2) & 1, abort_flag, dev_status));
      if (!ok) break;
      tc::tc_fence_after();
      float s[64];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t v[32];
        tc::tmem_ld32(tl + kColS + (j % 2) * 128 + half * 64 + cc * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(v[i]);
      }
      const bool has_b = 2 * j + 1 < nl;
      const int blk = half == 0 ? c.list[2 * j] : (has_b ? c.list[2 * j + 1] : -1);
      // mask: keys after this row, and the empty second slot of an odd tail
      const bool diag = blk < 0 || blk * BKB + BKB - 1 > t * BQ;
      float mx8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
      if (VS) {
        const uint64_t keep = blk < 0 ? 0ull : vs_keep(vrow, srow, row_abs, blk);
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          s[i] = ((keep >> i) & 1ull) ? s[i] : -INFINITY;
          mx8[i & 7] = fmaxf(mx8[i & 7], s[i]);
        }
      } else if (diag) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const bool vis = blk >= 0 && blk * BKB + i <= row_abs;
          s[i] = vis ? s[i] : -INFINITY;
          mx8[i & 7] = fmaxf(mx8[i & 7], s[i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) mx8[i & 7] = fmaxf(mx8[i & 7], s[i]);
      }
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_tile = mx * scale_log2;
      float alpha = 1.f;
      if (m_tile > m_used + 8.0f) {                     // also taken when m_used is -inf
        alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_tile);
        m_used = m_tile;
      }
      const float m_safe = (m_used == -INFINITY) ? 0.f : m_used;
      float sum0 = 0.f, sum1 = 0.f, sum2 = 0.f, sum3 = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 64; i += 4) {
        const float p0 = ex2(fmaf(s[i], scale_log2, -m_safe));
        const float p1 = ex2(fmaf(s[i + 1], scale_log2, -m_safe));
        const float p2 = ex2(fmaf(s[i + 2], scale_log2, -m_safe));
        const float p3 = ex2(fmaf(s[i + 3], scale_log2, -m_safe));
        sum0 += p0; sum1 += p1; sum2 += p2; sum3 += p3;
        __nv_bfloat162 a = __floats2bfloat162_rn(p0, p1);
        __nv_bfloat162 bq = __floats2bfloat162_rn(p2, p3);
        pk[i / 2] = *reinterpret_cast<uint32_t*>(&a);
        pk[i / 2 + 1] = *reinterpret_cast<uint32_t*>(&bq);
      }
      l = l * alpha + ((sum0 + sum1) + (sum2 + sum3));

      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // rescaling O_h: the previous value product of this half must have landed
        ok = warp_all(tc::mbar_wait(&c.o_ready[half], (j - 1) & 1, abort_flag, dev_status));
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t v[32];
          tc::tmem_ld32(tl + colO + cc * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
          tc::tmem_st32(tl + colO + cc * 32, v);
        }
      }
      // P_h -> TMEM over the first 32 columns of this half's (already read) S region
      tc::tmem_st32(tl + kColS + (j % 2) * 128 + half * 64, pk);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.p_full[half]);
    }
    // epilogue: merge the two halves' partial softmax sums, store 64 columns each
    uint16_t* orow = out + ((size_t)bh * N + (size_t)t * BQ + r) * HD + half * 64;
    bool have = ok && ntiles > 0;
    if (have) have = warp_all(tc::mbar_wait(&c.o_ready[half], (ntiles - 1) & 1, abort_flag, dev_status));
    if (ntiles > 0) {
      c.mpart[half][r] = m_used;
      c.lpart[half][r] = l;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.lbar[quarter]);
      // each half arrives only after its own last value product completed, so past
      // this barrier both O accumulators are final
      if (have) have = warp_all(tc::mbar_wait(&c.lbar[quarter], 0, abort_flag, dev_status));
    }
    if (have) {
      tc::tc_fence_after();
      const float m0 = c.mpart[0][r], m1 = c.mpart[1][r];
      const float mm = fmaxf(m0, m1);
      const float f0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - mm);
      const float f1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - mm);
      const float lt = c.lpart[0][r] * f0 + c.lpart[1][r] * f1;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float w0 = f0 * inv, w1 = f1 * inv;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t v0[32], v1[32];
        tc::tmem_ld32(tl + kColO + half * 64 + cc * 32, v0);          // O_0, this half's columns
        tc::tmem_ld32(tl + kColO + 128 + half * 64 + cc * 32, v1);    // O_1, same columns
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k0 = i + 2 * e;
            __nv_bfloat162 p = __floats2bfloat162_rn(
                __uint_as_float(v0[k0]) * w0 + __uint_as_float(v1[k0]) * w1,
                __uint_as_float(v0[k0 + 1]) * w0 + __uint_as_float(v1[k0 + 1]) * w1);
            w[e] = *reinterpret_cast<uint32_t*>(&p);
          }
          *reinterpret_cast<uint4*>(orow + cc * 32 + i) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      if (lse && half == 0)
        lse[bh * N + (size_t)t * BQ + r] = lt > 0.f ? (mm + log2f(lt)) * 0.69314718055994531f : -INFINITY;
    } else if (ntiles == 0) {
#pragma unroll
      for (int i = 0; i < 64; i += 8)
        *reinterpret_cast<uint4*>(orow + i) = make_uint4(0, 0, 0, 0);
      if (lse && half == 0) lse[bh * N + (size_t)t * BQ + r] = -INFINITY;
    }
  }

  // ---------------- teardown ----------------
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && ntiles > 0) {
    // make sure no TMA copy of this CTA is still landing in shared memory: wait for
    // the last phase issued on every stage (earlier phases completed before it)
    tc::mbar_wait_timed(&c.q_full, 0);
    for (int j = k_issued - NS < 0 ? 0 : k_issued - NS; j < k_issued; ++j)
      tc::mbar_wait_timed(&c.k_full[j % NS], (j / NS) & 1);
    for (int j = v_issued - NS < 0 ? 0 : v_issued - NS; j < v_issued; ++j)
      tc::mbar_wait_timed(&c.v_full[j % NS], (j / NS) & 1);
  }
  if ((warp == 1 || warp == 10) && lane == 0 && mma_issued) {
    // every MMA this thread issued has completed once this commit arrives
    const int hf = warp == 1 ? 0 : 1;
    tc::umma_commit(&c.done[hf]);
    tc::mbar_wait_timed(&c.done[hf], 0);
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

bool attend_tc_supported(const bsa_shape& s) {
  return s.dtype == BSA_BF16 && s.d == HD && s.block_k == BKB && s.tile_q == BQ;
}

template <bool VS>
static cudaError_t launch_attend_tc_t(const bsa_shape& s, const void* q, const void* k, const void* v,
                                      const int32_t* kv_idx, const int32_t* kv_cnt, int W, float scale,
                                      void* out, float* lse, int32_t* dev_status,
                                      const unsigned long long* vbits,
                                      const unsigned long long* sbits, cudaStream_t st) {
  if (W > kMaxList) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  const uint64_t qrows = (uint64_t)s.B * s.Hq * s.N, krows = (uint64_t)s.B * s.Hkv * s.N;
  if (!make_tmap_bf16_2d(&mq, q, qrows, HD, 64, BQ) || !make_tmap_bf16_2d(&mk, k, krows, HD, 64, BKB) ||
      !make_tmap_bf16_2d(&mv, v, krows, HD, 64, BKB))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attend_tc_kernel<VS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int n_qt = s.N / BQ;
  const long long grid = (long long)s.B * s.Hq * n_qt;
  attend_tc_kernel<VS><<<(unsigned)grid, kThreads, kSmemBytes, st>>>(
      mq, mk, mv, kv_idx, kv_cnt, W, scale * 1.4426950408889634f, (uint16_t*)out, lse, dev_status,
      s.N, s.Hq, s.Hkv, n_qt, s.N / BKB, vbits, sbits);
  return cudaGetLastError();
}

cudaError_t launch_attend_tc(const bsa_shape& s, const void* q, const void* k, const void* v,
                             const int32_t* kv_idx, const int32_t* kv_cnt, int W, float scale,
                             void* out, float* lse, int32_t* dev_status, cudaStream_t st) {
  return launch_attend_tc_t<false>(s, q, k, v, kv_idx, kv_cnt, W, scale, out, lse, dev_status, nullptr,
                                   nullptr, st);
}

cudaError_t launch_attend_tc_vs(const bsa_shape& s, const void* q, const void* k, const void* v,
                                const int32_t* lists, const int32_t* counts, int W, float scale,
                                void* out, float* lse, int32_t* dev_status,
                                const unsigned long long* vbits, const unsigned long long* sbits,
                                cudaStream_t st) {
  return launch_attend_tc_t<true>(s, q, k, v, lists, counts, W, scale, out, lse, dev_status, vbits,
                                  sbits, st);
}

}  // namespace bsa
