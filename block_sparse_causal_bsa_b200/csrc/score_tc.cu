// K-min/K-max block scores on Blackwell tensor cores (tcgen05 + TMEM + TMA); the
// mean-pooled backbones run in score_rank.cu.
//
// s(t,j) = max over the tile's rows i of sum_c max(q_ic kmin_jc, q_ic kmax_jc): the
// per-coordinate upper-bound backbone of [UGS] Metodologia step 1, with the tile max
// over rows of step 2; -inf for blocks j > J_t. With mid = (kmin+kmax)/2 and
// rad = (kmax-kmin)/2 >= 0 the sum is q . mid + |q| . rad, a contraction over 2d:
// each chunk of 128 blocks is two half-chunks, mid against Q and rad against |Q|,
// accumulated into the same TMEM columns, D[128 blocks x 128 rows] = [mid | rad] .
// [Q | |Q|]^T, so each TMEM lane holds one block and its thread takes the row max.
//
// Operands are fp16, one pass each: the pool kernel writes mid and rad scaled by one
// power of two 2^r per block (the block's largest of |mid| and rad lands in
// [2^14, 2^15)), and the epilogue warps convert the bf16 query tile in shared memory
// to fp16 scaled by 2^s (its largest |q| in [2^14, 2^15)) and write |Q| beside it
// (the same values with the sign cleared). Scaling by powers of two is exact; mid
// and rad round to fp16 (relative 2^-12) and the products accumulate in fp32; the
// epilogue multiplies the row max by 2^-s and 2^-r.
//
// One CTA per (batch, query head, query tile); 192 threads:
//   warp 0: TMA producer (the query tile, then the half-chunks, double-buffered);
//   warp 1: MMA issuer (8 MMAs of M128 N128 K16 per half-chunk into one of two
//           TMEM accumulators);
//   warps 2-5: convert Q and make |Q| (a thread per query row; the tile's largest
//           |q| exchanged through a bounded mbarrier), then the epilogue (TMEM ->
//           row max -> rescale -> scores row), overlapping the next chunk's MMAs.
// Every wait is bounded. Shapes: bf16, d = 128, query tile 128, key block 64 or 128.
#include <math.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace bsa {

namespace {
constexpr int TQ = 128;           // query tile rows
constexpr int HD = 128;           // head dim
constexpr int CB = 128;           // blocks per chunk (MMA M)
constexpr int kThreads = 192;
constexpr uint32_t kHalf = 16384;           // 128 rows x 128 bytes: one 64-column half
constexpr uint32_t kPart = 2 * kHalf;       // a tile or a half-chunk (128 x 128, 16-bit)
constexpr uint32_t kTmemCols = 256;         // two accumulators of 128 columns

constexpr size_t kSmemQ = 0;                // Q (bf16 from TMA, then fp16 in place)
constexpr size_t kSmemQa = kPart;           // |Q| (fp16)
constexpr size_t kSmemK = 2 * kPart;        // two half-chunk stages
constexpr size_t kSmemCtrl = kSmemK + 2 * kPart;

struct __align__(8) Ctrl {
  uint64_t q_full, qa_full, qmax_bar;
  uint64_t kb_full[2], kb_empty[2];
  uint64_t d_full[2], d_free[2];
  uint64_t done;
  uint32_t tmem;
  int abort_flag;
  uint32_t qmax_part[4];
};

__device__ __forceinline__ bool warp_all(bool x) { return __all_sync(0xffffffffu, x); }

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = max(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// 2^e as a float, e in [-126, 127]
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }
}  // namespace

__global__ void __launch_bounds__(kThreads, 1) score_bounds_kernel(
    const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmmid,
    const __grid_constant__ CUtensorMap tmrad, const float* __restrict__ kinv,
    float* __restrict__ scores, int32_t* dev_status, int N, int Hq, int Hkv, int n_qt, int n_kb,
    int block_k) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl& c = *reinterpret_cast<Ctrl*>(sm + kSmemCtrl);
  const uint32_t sQ = tc::smem_u32(sm + kSmemQ);
  const uint32_t sQa = tc::smem_u32(sm + kSmemQa);
  const uint32_t sK = tc::smem_u32(sm + kSmemK);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const int G = Hq / Hkv;
  int x = blockIdx.x;
  const int hh = x % G;
  x /= G;
  const int t = n_qt - 1 - (x % n_qt);             // longest rows first
  const int bgi = x / n_qt;
  const int b = bgi / Hkv, g = bgi % Hkv;
  const int h = g * G + hh;
  const int J = (int)(((long long)(t + 1) * TQ - 1) / block_k);
  const int nc = (J + 1 + CB - 1) / CB;
  const int kb_row0 = bgi * n_kb;

  if (threadIdx.x == 0) {
    tc::mbar_init(&c.q_full, 1);
    tc::mbar_init(&c.qa_full, 4);
    tc::mbar_init(&c.qmax_bar, 4);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&c.kb_full[i], 1);
      tc::mbar_init(&c.kb_empty[i], 1);
      tc::mbar_init(&c.d_full[i], 1);
      tc::mbar_init(&c.d_free[i], 4);
    }
    tc::mbar_init(&c.done, 1);
    c.abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&c.tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = c.tmem;
  volatile int* abort_flag = &c.abort_flag;
  int kb_issued = 0;
  bool mma_issued = false;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    tc::prefetch_tmap(&tmq);
    tc::prefetch_tmap(&tmmid);
    tc::prefetch_tmap(&tmrad);
    const int qrow = (int)(((size_t)b * Hq + h) * N + (size_t)t * TQ);
    tc::mbar_arrive_expect_tx(&c.q_full, kPart);
    tc::tma_load_2d(sm + kSmemQ, &tmq, 0, qrow, &c.q_full);
    tc::tma_load_2d(sm + kSmemQ + kHalf, &tmq, 64, qrow, &c.q_full);
    for (int u = 0; u < 2 * nc; ++u) {             // half-chunk u: chunk u/2, mid (even) or rad (odd)
      const int s = u & 1;
      if (u >= 2 && !tc::mbar_wait(&c.kb_empty[s], ((u >> 1) - 1) & 1, abort_flag, dev_status)) break;
      uint8_t* dst = sm + kSmemK + s * kPart;
      const int row = kb_row0 + (u >> 1) * CB;
      const CUtensorMap* m = (u & 1) ? &tmrad : &tmmid;
      tc::mbar_arrive_expect_tx(&c.kb_full[s], kPart);
      tc::tma_load_2d(dst, m, 0, row, &c.kb_full[s]);
      tc::tma_load_2d(dst + kHalf, m, 64, row, &c.kb_full[s]);
      kb_issued = u + 1;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idesc = tc::idesc_f16_f32(CB, TQ, false, false);
    bool ok = tc::mbar_wait(&c.qa_full, 0, abort_flag, dev_status);   // Q and |Q| converted
    for (int ch = 0; ok && ch < nc; ++ch) {
      const int db = ch & 1;
      ok = ch < 2 || tc::mbar_wait(&c.d_free[db], ((ch >> 1) - 1) & 1, abort_flag, dev_status);
      const uint32_t d = tmem + db * TQ;
      for (int part = 0; ok && part < 2; ++part) {
        const int u = ch * 2 + part;
        const int s = u & 1;
        ok = tc::mbar_wait(&c.kb_full[s], (u >> 1) & 1, abort_flag, dev_status);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t kb = sK + s * kPart;
        const uint32_t qb = part == 0 ? sQ : sQa;       // Q against mid, |Q| against rad
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          tc::umma_bf16(d, tc::sdesc_sw128(kb + off, 16, 1024), tc::sdesc_sw128(qb + off, 16, 1024), idesc,
                        (part > 0 || kk > 0) ? 1u : 0u);
        }
        mma_issued = true;
        tc::umma_commit(&c.kb_empty[s]);
      }
      if (!ok) break;
      tc::umma_commit(&c.d_full[db]);
    }
  } else if (warp >= 2) {
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                 // Q row; later: block within the chunk
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    // ---- Q (bf16) -> fp16 * 2^s in place, |Q| beside it; thread r owns row r ----
    bool ok = warp_all(tc::mbar_wait(&c.q_full, 0, abort_flag, dev_status));
    float qinv = 1.f;
    if (ok) {
      uint4 v[16];
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        // chunk order XOR-ed with the row's swizzle phase: conflict-free across the warp
        const int half = p >> 3, ck = (p & 7) ^ (r & 7);
        v[p] = *reinterpret_cast<const uint4*>(sm + kSmemQ + half * kHalf + r * 128 + ck * 16);
      }
      uint32_t mx = 0u;
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        mx = __vmaxu2(mx, v[p].x & 0x7fff7fffu);
        mx = __vmaxu2(mx, v[p].y & 0x7fff7fffu);
        mx = __vmaxu2(mx, v[p].z & 0x7fff7fffu);
        mx = __vmaxu2(mx, v[p].w & 0x7fff7fffu);
      }
      mx = warp_max_u32(max(mx & 0xffffu, mx >> 16));
      if (lane == 0) c.qmax_part[quarter] = mx;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.qmax_bar);
      ok = warp_all(tc::mbar_wait(&c.qmax_bar, 0, abort_flag, dev_status));
      if (ok) {
        const uint32_t mb = max(max(c.qmax_part[0], c.qmax_part[1]), max(c.qmax_part[2], c.qmax_part[3]));
        const uint32_t mu = (mb << 16) & 0x7fffffffu;   // the largest |q| as fp32 bits
        int se = 0;
        if (mu != 0u && mu < 0x7f800000u) {
          se = 14 - ((int)(mu >> 23) - 127);
          se = se < -126 ? -126 : (se > 126 ? 126 : se);
        }
        const float sc = exp2i(se);
        qinv = exp2i(-se);
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          uint32_t w4[4] = {v[p].x, v[p].y, v[p].z, v[p].w};
          uint32_t a4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(w4[e] << 16) * sc;
            const float hi = __uint_as_float(w4[e] & 0xffff0000u) * sc;
            const __half2 h2 = __floats2half2_rn(lo, hi);
            w4[e] = *reinterpret_cast<const uint32_t*>(&h2);
            a4[e] = w4[e] & 0x7fff7fffu;               // |q| in fp16: the sign bits cleared
          }
          const int half = p >> 3, ck = (p & 7) ^ (r & 7);
          const uint32_t off = half * kHalf + r * 128 + ck * 16;
          *reinterpret_cast<uint4*>(sm + kSmemQ + off) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          *reinterpret_cast<uint4*>(sm + kSmemQa + off) = make_uint4(a4[0], a4[1], a4[2], a4[3]);
        }
        tc::fence_proxy_async_smem();                  // generic writes -> tensor-core reads
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&c.qa_full);
      }
    }
    // ---- epilogue ----
    const float* krow = kinv + (size_t)bgi * n_kb;
    float* srow = scores + (((size_t)b * Hq + h) * n_qt + t) * n_kb;
    for (int ch = 0; ok && ch < nc; ++ch) {
      const int s = ch & 1;
      const int j = ch * CB + r;
      const float kv = j <= J ? __ldg(krow + j) : 0.f;
      if (!warp_all(tc::mbar_wait(&c.d_full[s], (ch >> 1) & 1, abort_flag, dev_status))) break;
      tc::tc_fence_after();
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t v[64];
        tc::tmem_ld64(tl + s * TQ + cc * 64, v);
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          m0 = fmaxf(m0, __uint_as_float(v[i]));
          m1 = fmaxf(m1, __uint_as_float(v[i + 1]));
        }
      }
      if (j <= J) srow[j] = (fmaxf(m0, m1) * qinv) * kv;    // exact: powers of two
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.d_free[s]);
    }
    // blocks no row of the tile can see
    for (int j = J + 1 + (threadIdx.x - 64); j < n_kb; j += 128) srow[j] = -INFINITY;
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0) {
    tc::mbar_wait_timed(&c.q_full, 0);
    for (int u = kb_issued - 2 < 0 ? 0 : kb_issued - 2; u < kb_issued; ++u)
      tc::mbar_wait_timed(&c.kb_full[u & 1], (u >> 1) & 1);
  }
  if (warp == 1) {
    if (lane == 0 && mma_issued) {
      tc::umma_commit(&c.done);
      tc::mbar_wait_timed(&c.done, 0);
    }
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

bool score_tc_supported(const bsa_shape& s) {
  return s.dtype == BSA_BF16 && s.d == HD && s.tile_q == TQ &&
         (long long)s.B * s.Hq * s.N < (1ll << 31) &&
         (long long)s.B * s.Hkv * (s.N / s.block_k) < (1ll << 31);
}

cudaError_t launch_score_tc_bounds(const bsa_shape& s, const void* q, const uint16_t* mid16,
                                   const uint16_t* rad16, const float* kinv, float* scores,
                                   int32_t* dev_status, cudaStream_t st) {
  CUtensorMap mq, mm, mr;
  const uint64_t qrows = (uint64_t)s.B * s.Hq * s.N;
  const uint64_t krows = (uint64_t)s.B * s.Hkv * (s.N / s.block_k);
  if (!make_tmap_bf16_2d(&mq, q, qrows, HD, 64, TQ) || !make_tmap_bf16_2d(&mm, mid16, krows, HD, 64, CB) ||
      !make_tmap_bf16_2d(&mr, rad16, krows, HD, 64, CB))
    return cudaErrorInvalidValue;
  const size_t smem = kSmemCtrl + sizeof(Ctrl) + 1024;
  cudaError_t e = cudaFuncSetAttribute(score_bounds_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int n_qt = s.N / TQ;
  const long long grid = (long long)s.B * s.Hq * n_qt;
  score_bounds_kernel<<<(unsigned)grid, kThreads, smem, st>>>(mq, mm, mr, kinv, scores, dev_status, s.N,
                                                             s.Hq, s.Hkv, n_qt, s.N / s.block_k, s.block_k);
  return cudaGetLastError();
}

}  // namespace bsa
