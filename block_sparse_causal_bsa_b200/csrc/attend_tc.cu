// Block-sparse causal attention on Blackwell tensor cores (tcgen05 + TMEM + TMA).
//
// O_i = sum over the keys j of the listed blocks with j <= i of
// softmax(scale * q_i . k_j) v_j -- the sparse aggregation step of [UGS]
// step 5 and [Stem] Implementação: only the blocks in kv_idx are streamed,
// with an online softmax. Shapes: bf16, d = 128, key blocks of 64, query
// tiles of 128.
//
// One CTA per (batch, query head, query tile), 192 threads, two CTAs per SM
// (256 TMEM columns and ~100 KB of shared memory each), so that every SM runs
// two independent pipelines of different tiles: one CTA's prologue, epilogue
// and softmax phases overlap the other's tensor-core work.
//   warp 0 (one thread)  TMA producer: the Q tile once, then the K and V rows of
//                        one listed block per stage, two stages deep.
//   warp 1 (one thread)  MMA issuer: S_j = Q K_j^T (M128 N64, 8 x K16) into one
//                        of two TMEM S buffers -- S_{j+1} is issued before the
//                        value product of block j -- then O += P_j V_j once P_j
//                        is written, P_j read straight from tensor memory (the
//                        A operand) and V as an MN-major B operand.
//   warps 2-5            softmax, one per TMEM lane quarter, a thread per query
//                        row: 64 S values from TMEM, the causal mask on the
//                        diagonal block, running max and sum, O rescaled in TMEM
//                        only when the running max grew by more than 2^8 (exact:
//                        l and O keep the same stale max), ex2 exponentials, P
//                        (bf16, two per 32-bit column) stored with tcgen05.st over
//                        the first 32 columns of the S buffer just read. O / l and
//                        lse use the sum l of the fp32 exponentials; rows of the
//                        vertical-slash variant (possibly a handful of keys) divide
//                        O by the sum of the bf16 weights as applied instead.
//                        Epilogue: O / l to bf16 in global memory, and the lse.
// Shared-memory operand layouts (128-byte swizzled, as TMA writes them):
//   Q, K: K-major [rows x 64 elements] halves; V: MN-major (rows = keys, 64
//   contiguous head dims per 128-byte row), the two 64-dim halves 8 KB apart.
// TMEM (256 columns): O at 0, S buffers at 128 and 192 (P over the first 32
// columns of a buffer once read).
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
constexpr int kThreads = 192;
constexpr int kSoftmaxWarps = 4;
constexpr int kMaxList = 1024;   // kv_idx entries staged per tile
constexpr uint32_t kQHalf = 16384;           // Q: [128 rows x 128 bytes] per 64-dim half
constexpr uint32_t kBHalf = 8192;            // K or V block: [64 rows x 128 bytes] per 64-dim half
constexpr uint32_t kBlock = 2 * kBHalf;      // one K or V block (64 keys x 128 dims)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 0;                // O accumulator
constexpr uint32_t kColS = 128;              // S buffers at 128 and 192

struct __align__(8) Ctrl {
  uint64_t q_full;
  uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  uint64_t s_full[2];
  uint64_t p_full, o_ready, done;
  uint32_t tmem;
  int abort_flag;
  int n_list;
  int list[kMaxList];
};

constexpr size_t kSmemQ = 0;
constexpr size_t kSmemK = kSmemQ + 2 * kQHalf;
constexpr size_t kSmemV = kSmemK + NS * kBlock;
constexpr size_t kSmemCtrl = kSmemV + NS * kBlock;
constexpr size_t kSmemBytes = kSmemCtrl + sizeof(Ctrl) + 1024;   // + alignment slack

__device__ __forceinline__ bool warp_all(bool x) { return __all_sync(0xffffffffu, x); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (a0, a1) += (b0, b1) as one packed fp32x2 add (sm_100), rounding as two fadds
__device__ __forceinline__ void add2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
      "add.rn.f32x2 ra, ra, rb;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
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
__global__ void __launch_bounds__(kThreads, 2) attend_tc_kernel(
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
      tc::mbar_init(&c.k_empty[s], 1);
      tc::mbar_init(&c.v_full[s], 1);
      tc::mbar_init(&c.v_empty[s], 1);
    }
    tc::mbar_init(&c.s_full[0], 1);
    tc::mbar_init(&c.s_full[1], 1);
    tc::mbar_init(&c.p_full, kSoftmaxWarps);
    tc::mbar_init(&c.o_ready, 1);
    tc::mbar_init(&c.done, 1);
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
  volatile int* abort_flag = &c.abort_flag;
  int k_issued = 0, v_issued = 0;     // blocks whose K / V loads the producer issued
  bool mma_issued = false;

  if (warp == 0 && lane == 0 && nl > 0) {
    // ---------------- TMA producer ----------------
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
    tc::mbar_arrive_expect_tx(&c.q_full, 2 * kQHalf);
    tc::tma_load_2d(sm + kSmemQ, &tmq, 0, q_row0, &c.q_full);
    tc::tma_load_2d(sm + kSmemQ + kQHalf, &tmq, 64, q_row0, &c.q_full);
    for (int j = 0; j < nl; ++j) {
      const int s = j % NS;
      const int r = kv_row0 + c.list[j] * BKB;
      if (j >= NS && !tc::mbar_wait(&c.k_empty[s], ((j / NS) - 1) & 1, abort_flag, dev_status)) break;
      uint8_t* kd = sm + kSmemK + s * kBlock;
      tc::mbar_arrive_expect_tx(&c.k_full[s], kBlock);
      tc::tma_load_2d(kd, &tmk, 0, r, &c.k_full[s]);
      tc::tma_load_2d(kd + kBHalf, &tmk, 64, r, &c.k_full[s]);
      k_issued = j + 1;
      if (j >= NS && !tc::mbar_wait(&c.v_empty[s], ((j / NS) - 1) & 1, abort_flag, dev_status)) break;
      uint8_t* vd = sm + kSmemV + s * kBlock;
      tc::mbar_arrive_expect_tx(&c.v_full[s], kBlock);
      tc::tma_load_2d(vd, &tmv, 0, r, &c.v_full[s]);
      tc::tma_load_2d(vd + kBHalf, &tmv, 64, r, &c.v_full[s]);
      v_issued = j + 1;
    }
  } else if (warp == 1 && lane == 0 && nl > 0) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idS = tc::idesc_bf16_f32(128, 64, false, false);
    constexpr uint32_t idPV = tc::idesc_bf16_f32(128, 128, false, true);
    auto issue_s = [&](int j) {
      // S_j = Q (128 x d) . K_j^T
      const uint32_t kb = sK + (j % NS) * kBlock;
      const uint32_t d = tmem + kColS + (j % 2) * 64;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t qoff = (kk >> 2) * kQHalf + (kk & 3) * 32;
        const uint32_t koff = (kk >> 2) * kBHalf + (kk & 3) * 32;
        tc::umma_bf16(d, tc::sdesc_sw128(sQ + qoff, 16, 1024), tc::sdesc_sw128(kb + koff, 16, 1024), idS,
                      kk > 0);
      }
      tc::umma_commit(&c.s_full[j % 2]);
      tc::umma_commit(&c.k_empty[j % NS]);
    };
    bool ok = tc::mbar_wait(&c.q_full, 0, abort_flag, dev_status) &&
              tc::mbar_wait(&c.k_full[0], 0, abort_flag, dev_status);
    if (ok) {
      tc::tc_fence_after();
      issue_s(0);
      mma_issued = true;
    }
    for (int j = 0; ok && j < nl; ++j) {
      const int jn = j + 1;
      if (jn < nl) {
        // S(jn) overwrites the buffer of block jn-2, whose P the value product of block
        // jn-2 = j-1 reads: wait for that product to complete (which also implies the
        // softmax read S there)
        ok = tc::mbar_wait(&c.k_full[jn % NS], (jn / NS) & 1, abort_flag, dev_status) &&
             (jn < 2 || tc::mbar_wait(&c.o_ready, (jn - 2) & 1, abort_flag, dev_status));
        if (!ok) break;
        tc::tc_fence_after();
        issue_s(jn);
      }
      ok = tc::mbar_wait(&c.v_full[j % NS], (j / NS) & 1, abort_flag, dev_status) &&
           tc::mbar_wait(&c.p_full, j & 1, abort_flag, dev_status);
      if (!ok) break;
      tc::tc_fence_after();
      const uint32_t vb = sV + (j % NS) * kBlock;
      const uint32_t pa = tmem + kColS + (j % 2) * 64;              // P_j in TMEM
      // O += P_j (128 rows x 64 keys) . V_j (64 keys x 128 dims)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        tc::umma_bf16_ts(tmem + kColO, pa + kk * 8, tc::sdesc_sw128(vb + kk * 2048, kBHalf, 1024), idPV,
                         (j > 0 || kk > 0) ? 1u : 0u);
      }
      tc::umma_commit(&c.o_ready);
      tc::umma_commit(&c.v_empty[j % NS]);
    }
  } else if (warp >= 2) {
    // ---------------- softmax warps ----------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                  // row in the tile == TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    const int row_abs = t * BQ + r;
    const unsigned long long* vrow = VS ? vbits + bh * (size_t)(N / 64 + 1) : nullptr;
    const unsigned long long* srow = VS ? sbits + bh * (size_t)(N / 64 + 1) : nullptr;
    float m_used = -INFINITY;                           // running max, scaled log2 units
    float l = 0.f;                                      // running sum of the exponentials (lse)
    float lq = 0.f;                                     // ... of their bf16 values (normalises O)
    bool ok = true;
    for (int j = 0; j < nl; ++j) {
      ok = warp_all(tc::mbar_wait(&c.s_full[j % 2], (j / 2) & 1, abort_flag, dev_status));
      if (!ok) break;
      tc::tc_fence_after();
      float s[64];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t v[32];
        tc::tmem_ld32(tl + kColS + (j % 2) * 64 + cc * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(v[i]);
      }
      const int blk = c.list[j];
      float mx8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
      if (VS) {
        const uint64_t keep = vs_keep(vrow, srow, row_abs, blk);
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          s[i] = ((keep >> i) & 1ull) ? s[i] : -INFINITY;
          mx8[i & 7] = fmaxf(mx8[i & 7], s[i]);
        }
      } else if (blk * BKB + BKB - 1 > t * BQ) {
        // the block reaches past the tile's first row: mask keys after this row
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          s[i] = blk * BKB + i <= row_abs ? s[i] : -INFINITY;
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
      float q0 = 0.f, q1 = 0.f, q2 = 0.f, q3 = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 64; i += 4) {
        const float p0 = ex2(fmaf(s[i], scale_log2, -m_safe));
        const float p1 = ex2(fmaf(s[i + 1], scale_log2, -m_safe));
        const float p2 = ex2(fmaf(s[i + 2], scale_log2, -m_safe));
        const float p3 = ex2(fmaf(s[i + 3], scale_log2, -m_safe));
        __nv_bfloat162 a = __floats2bfloat162_rn(p0, p1);
        __nv_bfloat162 bq = __floats2bfloat162_rn(p2, p3);
        const uint32_t wa = *reinterpret_cast<uint32_t*>(&a), wb = *reinterpret_cast<uint32_t*>(&bq);
        pk[i / 2] = wa;
        pk[i / 2 + 1] = wb;
        add2(sum0, sum1, p0, p1);
        add2(sum2, sum3, p2, p3);
        if (VS) {
          // vertical-slash rows may see a handful of keys: O is normalised by the sum of
          // the bf16 weights the value product uses, so the applied weights sum to one (a
          // row with one key gets exactly its value); block rows see >= 64 keys and use l
          add2(q0, q1, __uint_as_float(wa << 16), __uint_as_float(wa & 0xffff0000u));
          add2(q2, q3, __uint_as_float(wb << 16), __uint_as_float(wb & 0xffff0000u));
        }
      }
      l = l * alpha + ((sum0 + sum1) + (sum2 + sum3));
      if (VS) lq = lq * alpha + ((q0 + q1) + (q2 + q3));

      if (j > 0) {
        // the previous value product has landed: O may be rescaled, and the issuer has
        // consumed p_full(j-1), so this warp's arrival below is for phase j (a parity wait
        // cannot tell phase j-1 from j+1)
        ok = warp_all(tc::mbar_wait(&c.o_ready, (j - 1) & 1, abort_flag, dev_status));
        if (!ok) break;
        tc::tc_fence_after();
      }
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t v[32];
          tc::tmem_ld32(tl + kColO + cc * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
          tc::tmem_st32(tl + kColO + cc * 32, v);
        }
      }
      // P -> TMEM over the first 32 columns of the (already read) S buffer
      tc::tmem_st32(tl + kColS + (j % 2) * 64, pk);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.p_full);
    }
    // epilogue
    uint16_t* orow = out + ((size_t)bh * N + (size_t)t * BQ + r) * HD;
    bool have = ok && nl > 0;
    if (have) have = warp_all(tc::mbar_wait(&c.o_ready, (nl - 1) & 1, abort_flag, dev_status));
    if (have) {
      tc::tc_fence_after();
      const float ln = VS ? lq : l;
      const float inv = ln > 0.f ? 1.f / ln : 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tc::tmem_ld32(tl + kColO + cc * 32, v);
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 p = __floats2bfloat162_rn(__uint_as_float(v[i + 2 * e]) * inv,
                                                     __uint_as_float(v[i + 2 * e + 1]) * inv);
            w[e] = *reinterpret_cast<uint32_t*>(&p);
          }
          *reinterpret_cast<uint4*>(orow + cc * 32 + i) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      if (lse)
        lse[bh * N + (size_t)t * BQ + r] = l > 0.f ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
    } else if (nl == 0) {
#pragma unroll
      for (int i = 0; i < HD; i += 8)
        *reinterpret_cast<uint4*>(orow + i) = make_uint4(0, 0, 0, 0);
      if (lse) lse[bh * N + (size_t)t * BQ + r] = -INFINITY;
    }
  }

  // ---------------- teardown ----------------
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && nl > 0) {
    // make sure no TMA copy of this CTA is still landing in shared memory: wait for
    // the last phase issued on every stage (earlier phases completed before it)
    tc::mbar_wait_timed(&c.q_full, 0);
    for (int j = k_issued - NS < 0 ? 0 : k_issued - NS; j < k_issued; ++j)
      tc::mbar_wait_timed(&c.k_full[j % NS], (j / NS) & 1);
    for (int j = v_issued - NS < 0 ? 0 : v_issued - NS; j < v_issued; ++j)
      tc::mbar_wait_timed(&c.v_full[j % NS], (j / NS) & 1);
  }
  if (warp == 1) {
    if (lane == 0 && mma_issued) {
      // every MMA this thread issued has completed once this commit arrives
      tc::umma_commit(&c.done);
      tc::mbar_wait_timed(&c.done, 0);
    }
    __syncwarp();
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
