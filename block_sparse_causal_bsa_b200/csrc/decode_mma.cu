// Decode attention with run-time termination ([ART] 2.1-2.4) on warp-level
// tensor-core MMAs: the KV cache of one (batch, KV head) is streamed block by
// block, in order (or in the order of a caller's visit list, compacted into
// shared memory by warp 5 before the pipeline starts); after each block the
// normalised partial output O^(t) is probed, and from the second visit step on
// the stability test decides whether to stop.
//
// Why warp-level MMAs here: per block the contraction is skinny (N = the G <= 8
// query heads of the group), so its cost is latency, not tensor throughput. A
// single-CTA tcgen05.mma has a floor of ~80-130 cycles per instruction whatever
// N is, and a 128-key block needs 16 of them in a dependent chain (~1900 cycles),
// which set the period of the longest group's chain. An m16n8k16 mma.sync has a
// ~20-cycle latency and four warps issue one every ~2 cycles per SM, so the MMAs of
// a block cost a few hundred cycles; what bounds the chain then is the block's
// shared-memory traffic (64 KB of ldmatrix reads and the 64 KB TMA write) and the
// SM's own load bandwidth (~180-240 GB/s for one SM streaming alone).
//
// One CTA per (batch, KV head), 192 threads:
//   warp 0 (one thread)  TMA producer: K and V blocks of 128 keys (128-byte
//                        swizzled, two 64-column halves each), a ring of three
//                        64 KB stages, until told to halt.
//   warps 1-4            compute: warp w owns keys 32w..32w+31 of every block and
//                        keeps its own online-softmax state over them (running max
//                        m, row sum l, unnormalised O for all G heads):
//                          S = K Q^T   (A = K rows via ldmatrix, B = Q in registers)
//                          P = 2^(S*scale*log2e - m)  (m: the running max)
//                          O += V^T P^T (A = V^T via ldmatrix.trans, B = P^T turned
//                                        from the S accumulators by movmatrix)
//                        and after each block publishes m, l and O of the first head.
//   warp 5               decider: merges the four warps' states of block t into
//                        x^(t) = O^(t)[first head][probe dims] / l (each warp's part
//                        scaled by 2^(m_w - max m), added in warp order), then runs
//                        the stability test: in fp32 where proven margins to the
//                        defining fp64 evaluation settle it, else in fp64 (exact
//                        products, sums in a fixed pairwise order across the warp),
//                        and publishes stop / continue.
// The compute warps read the verdict on block t two blocks later, keeping their
// state as of block t-2 until then; on a stop they return that copy. After a stop
// the producer is released through a halt flag; a compute warp that waits for a
// block the producer never loads sees the halt and reads the open verdicts. All
// waits are bounded. At the end the four per-warp states are merged (the same
// scaling) and O / l is written in bf16.
// Shapes: bf16, d = 128, KV blocks of 128, Hq/Hkv in {1, 2, 4, 8}.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace bsa {

namespace {
constexpr int HD = 128;
constexpr int BKV = 128;
constexpr int GMAX = 8;
constexpr int STAGES = 3;
constexpr int kCompute = 4;               // compute warps (warps 1..4)
constexpr int kThreads = 192;
constexpr uint32_t kHalf = 16384;         // 128 rows x 128 bytes: one 64-column half
constexpr uint32_t kTile = 2 * kHalf;     // one K or V block
constexpr uint32_t kStage = 2 * kTile;    // K + V

struct __align__(16) Ctrl {
  uint64_t kv_full[STAGES], kv_empty[STAGES];
  uint64_t probe_rdy[2], decided[2];      // by block parity
  int abort_flag;                         // error: every role unwinds
  int halt;                               // producer stops issuing (normal stop or error)
  int stop_at;                            // block after which the decider stopped, or -1
  int n_steps;                            // blocks to visit
  int bad[kCompute];                      // a compute warp ended in error
  float pm[2][kCompute];                  // [block parity][warp] running max, first head
  float pl[2][kCompute];                  // [block parity][warp] row sum, first head
  float xo[2][kCompute][HD];              // [block parity][warp][head dim] O, first head
  float fm[kCompute][GMAX];               // final per-warp states: max, row sum, O
  float fl[kCompute][GMAX];
  float fo[kCompute][GMAX][HD];
  uint16_t blk[kMaxDecodeList];           // visit list (decode over a block list)
};

constexpr size_t kSmemStages = 0;
constexpr size_t kSmemCtrl = kSmemStages + STAGES * kStage;
constexpr size_t kSmemBytes = kSmemCtrl + sizeof(Ctrl) + 1024;   // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "decode_mma shared memory");

__device__ __forceinline__ bool warp_all(bool x) { return __all_sync(0xffffffffu, x); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// four 8x8 b16 matrices from shared memory (lanes 8i..8i+7 give the row addresses of
// matrix i); .trans hands each thread the transposed fragment
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
// sum over a warp of fp32 values, every lane returning the same value
__device__ __forceinline__ float warp_sum_f32(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}
// transpose of an 8x8 b16 matrix held one row fragment per thread
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// c += a (16x16, row) * b (16x8, col); bf16 operands, fp32 accumulators
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
}  // namespace

template <int G>
__global__ void __launch_bounds__(kThreads, 1) decode_mma_kernel(
    const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
    const uint16_t* __restrict__ q, const DecodeArgs a, uint16_t* __restrict__ out,
    int32_t* __restrict__ blocks_used, float* __restrict__ probe_trace, int32_t* dev_status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl& c = *reinterpret_cast<Ctrl*>(sm + kSmemCtrl);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bg = blockIdx.x;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int nb = a.L / BKV;
  const int row0 = bg * a.L;
  const uint32_t sStages = tc::smem_u32(sm + kSmemStages);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&c.kv_full[s], 1);
      tc::mbar_init(&c.kv_empty[s], kCompute);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&c.probe_rdy[i], kCompute);
      tc::mbar_init(&c.decided[i], 1);
    }
    c.abort_flag = 0;
    c.halt = 0;
    c.stop_at = -1;
    tc::fence_mbar_init();
  }
  if (warp == 5) {
    int n = nb;
    if (a.blist)
      n = warp_compact_blocks(a.blist + (size_t)bg * a.list_w, a.bcnt[bg], a.list_w, nb, c.blk,
                              dev_status, lane);
    if (lane == 0) c.n_steps = n;
  }
  __syncthreads();
  const int ns = c.n_steps;                         // visit steps
  const int tstride = a.blist ? a.list_w : nb;      // probe-trace rows per group
  volatile int* abort_flag = &c.abort_flag;
  volatile int* halt = &c.halt;
  int issued = 0;
  int used = ns;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    tc::prefetch_tmap(&tmk);
    tc::prefetch_tmap(&tmv);
    for (int t = 0; t < ns; ++t) {
      const int s = t % STAGES;
      if (t >= STAGES && !tc::mbar_wait_halt(&c.kv_empty[s], ((t / STAGES) - 1) & 1, halt, dev_status)) break;
      if (*halt) break;
      uint8_t* st = sm + kSmemStages + s * kStage;
      const int r = row0 + (a.blist ? (int)c.blk[t] : t) * BKV;
      tc::mbar_arrive_expect_tx(&c.kv_full[s], kStage);
      tc::tma_load_2d(st, &tmk, 0, r, &c.kv_full[s]);
      tc::tma_load_2d(st + kHalf, &tmk, 64, r, &c.kv_full[s]);
      tc::tma_load_2d(st + kTile, &tmv, 0, r, &c.kv_full[s]);
      tc::tma_load_2d(st + kTile + kHalf, &tmv, 64, r, &c.kv_full[s]);
      issued = t + 1;
    }
  } else if (warp >= 1 && warp <= kCompute) {
    // ---------------- compute ----------------
    const int cw = warp - 1;
    const int g8 = lane >> 2, tig = lane & 3;
    // Q^T as the B operand of S = K Q^T: column n = head g8 (zero past G), k = head dim
    uint32_t qf[8][2];
    {
      const uint16_t* qr = q + ((size_t)b * a.Hq + (size_t)g * G + (g8 < G ? g8 : 0)) * HD;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int d = 16 * kk + 8 * j + 2 * tig;
          qf[kk][j] = g8 < G ? ((uint32_t)qr[d] | ((uint32_t)qr[d + 1] << 16)) : 0u;
        }
      }
    }
    // per-lane parts of the ldmatrix row addresses inside a stage (128-byte swizzle:
    // 16-byte chunk c of row r sits at chunk c ^ (r & 7); every row used here has
    // r & 7 == lane & 7)
    const uint32_t rowK = (uint32_t)(32 * cw + (lane & 7) + ((lane >> 3) & 1) * 8) * 128u;
    const uint32_t rowV = (uint32_t)(32 * cw + (lane & 7) + (lane >> 4) * 8) * 128u;
    const uint32_t selK = (uint32_t)(lane >> 4), selV = (uint32_t)((lane >> 3) & 1);
    const uint32_t sw = (uint32_t)(lane & 7);
    // running state over this warp's keys; this thread holds heads 2 tig and 2 tig + 1
    // (h0, h1): O[d][h] for d = 16 dm + g8 (+8), m per head (equal across the 8 lanes
    // of a tig), l per head over this thread's four keys
    float o[8][4], osv[8][4];
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float msv0 = -INFINITY, msv1 = -INFINITY, lsv0 = 0.f, lsv1 = 0.f;
#pragma unroll
    for (int dm = 0; dm < 8; ++dm)
#pragma unroll
      for (int i = 0; i < 4; ++i) { o[dm][i] = 0.f; osv[dm][i] = 0.f; }
    const float sl2 = a.scale_log2;
    // after a halt seen while waiting for block t: the stop is on block t-2 or t-1 (the
    // verdicts before were read and said go on). Returns that block, or -1 (error).
    auto find_stop = [&](int t) -> int {
      for (int sb = t - 2 < 0 ? 0 : t - 2; sb < t; ++sb) {
        if (!warp_all(tc::mbar_wait(&c.decided[sb & 1], (sb >> 1) & 1, abort_flag, dev_status))) return -1;
        if (c.stop_at == sb) return sb;
      }
      return -1;
    };
    // the result for a stop on block sb: the saved state when sb = t-2, else the current
    // one (through t-1)
    auto take = [&](int sb, int t) {
      if (sb == t - 2) {
#pragma unroll
        for (int dm = 0; dm < 8; ++dm)
#pragma unroll
          for (int i = 0; i < 4; ++i) o[dm][i] = osv[dm][i];
        m0 = msv0; m1 = msv1; l0 = lsv0; l1 = lsv1;
      }
      used = sb + 1;
    };
    bool ok = true;
    for (int t = 0; t < ns; ++t) {
      const int s = t % STAGES;
      const int w = __reduce_max_sync(0xffffffffu, (unsigned)tc::mbar_wait_or_halt(
                                          &c.kv_full[s], (t / STAGES) & 1, halt, abort_flag, dev_status));
      if (w == 1) {
        // halted before block t landed: a stop was decided on block t-2 or t-1
        const int sb = find_stop(t);
        ok = sb >= 0;
        if (ok) take(sb, t);
        break;
      }
      if (w != 0) { ok = false; break; }
      const uint32_t kb = sStages + s * kStage, vb = kb + kTile;
      // S = K Q^T over this warp's 32 keys: two m16 tiles, four accumulator chains
      float sc[2][2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) sc[mt][j][i] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          uint32_t af[4];
          const uint32_t chunk = (uint32_t)(2 * (kk & 3)) + selK;
          ldsm4(kb + (uint32_t)(kk >> 2) * kHalf + rowK + (uint32_t)mt * 2048u + ((chunk ^ sw) << 4), af);
          mma16816(sc[mt][kk & 1], af, qf[kk][0], qf[kk][1]);
        }
      }
      // s[mt][i]: i = 0 / 1 key 16 mt + g8, heads h0 / h1; i = 2 / 3 key 16 mt + g8 + 8
      float sv[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sv[mt][i] = sc[mt][0][i] + sc[mt][1][i];
      // block max per head: the warp reduces it only when some score passes the running
      // max (rare after the first blocks). The max stays exact, so the largest weight is
      // 1 and its bf16 rounding is exact; a max moved only past a margin would round the
      // dominant weight and, in a peaked softmax, put its 2^-9 error on the probe.
      float bm0 = fmaxf(fmaxf(sv[0][0], sv[0][2]), fmaxf(sv[1][0], sv[1][2]));
      float bm1 = fmaxf(fmaxf(sv[0][1], sv[0][3]), fmaxf(sv[1][1], sv[1][3]));
      float mn0 = m0, mn1 = m1, al0 = 1.f, al1 = 1.f;
      if (__any_sync(0xffffffffu, bm0 * sl2 > m0 || bm1 * sl2 > m1)) {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, off));
          bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, off));
        }
        const float t0 = bm0 * sl2, t1 = bm1 * sl2;
        if (t0 > m0) { al0 = (m0 == -INFINITY) ? 0.f : ex2(m0 - t0); mn0 = t0; }
        if (t1 > m1) { al1 = (m1 == -INFINITY) ? 0.f : ex2(m1 - t1); mn1 = t1; }
      }
      float p[2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) p[mt][i] = ex2(fmaf(sv[mt][i], sl2, -((i & 1) ? mn1 : mn0)));
      const float ps0 = (p[0][0] + p[0][2]) + (p[1][0] + p[1][2]);
      const float ps1 = (p[0][1] + p[0][3]) + (p[1][1] + p[1][3]);
      // P^T as the B operand of O += V^T P^T: transposing the two 8x8 halves of each S
      // tile turns (key g8, heads 2 tig..) into (keys 2 tig.., head g8)
      uint32_t pb[2][2];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        pb[mt][0] = movm_t(pack_bf16(p[mt][0], p[mt][1]));
        pb[mt][1] = movm_t(pack_bf16(p[mt][2], p[mt][3]));
      }
      if (t >= 2) {
        // the verdict on block t-2 (it also frees that block's probe slot, reused below)
        ok = warp_all(tc::mbar_wait(&c.decided[t & 1], ((t - 2) >> 1) & 1, abort_flag, dev_status));
        if (!ok) break;
        if (c.stop_at == t - 2) {
          take(t - 2, t);
          break;
        }
      }
#pragma unroll
      for (int dm = 0; dm < 8; ++dm)
#pragma unroll
        for (int i = 0; i < 4; ++i) osv[dm][i] = o[dm][i];
      msv0 = m0; msv1 = m1; lsv0 = l0; lsv1 = l1;
      m0 = mn0; m1 = mn1;
      l0 = fmaf(l0, al0, ps0);
      l1 = fmaf(l1, al1, ps1);
      if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
        for (int dm = 0; dm < 8; ++dm) {
          o[dm][0] *= al0; o[dm][1] *= al1; o[dm][2] *= al0; o[dm][3] *= al1;
        }
      }
      float lh = l0;                    // the first head's row sum over the warp's keys
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) lh += __shfl_xor_sync(0xffffffffu, lh, off);
      // O += V^T P^T: eight m16 tiles of head dims, two k16 steps over this warp's keys
#pragma unroll
      for (int dm = 0; dm < 8; ++dm) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          uint32_t af[4];
          const uint32_t chunk = (uint32_t)(2 * (dm & 3)) + selV;
          ldsm4_t(vb + (uint32_t)(dm >> 2) * kHalf + rowV + (uint32_t)mt * 2048u + ((chunk ^ sw) << 4), af);
          mma16816(o[dm], af, pb[mt][0], pb[mt][1]);
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.kv_empty[s]);
      // publish the first head's state for the decider (lanes with tig 0 hold head 0)
      const int slot = t & 1;
      if (tig == 0) {
#pragma unroll
        for (int dm = 0; dm < 8; ++dm) {
          c.xo[slot][cw][16 * dm + g8] = o[dm][0];
          c.xo[slot][cw][16 * dm + g8 + 8] = o[dm][2];
        }
      }
      if (lane == 0) {
        c.pm[slot][cw] = m0;
        c.pl[slot][cw] = lh;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.probe_rdy[slot]);
    }
    if (ok && used == ns && ns >= 2) {
      // every block was folded; the verdict on block ns-2 is still unread (one on ns-1
      // would leave the result as it is)
      const int sb = ns - 2;
      ok = warp_all(tc::mbar_wait(&c.decided[sb & 1], (sb >> 1) & 1, abort_flag, dev_status));
      if (ok && c.stop_at == sb) take(sb, ns);
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;                  // unwind the other roles
      *halt = 1;
    }
    // final state of this warp for the merge after the teardown barrier
    float lf0 = l0, lf1 = l1;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      lf0 += __shfl_xor_sync(0xffffffffu, lf0, off);
      lf1 += __shfl_xor_sync(0xffffffffu, lf1, off);
    }
    const int h0 = 2 * tig, h1 = 2 * tig + 1;
    if (g8 == 0) {
      c.fm[cw][h0] = m0; c.fm[cw][h1] = m1;
      c.fl[cw][h0] = lf0; c.fl[cw][h1] = lf1;
    }
#pragma unroll
    for (int dm = 0; dm < 8; ++dm) {
      if (h0 < G) {
        c.fo[cw][h0][16 * dm + g8] = o[dm][0];
        c.fo[cw][h0][16 * dm + g8 + 8] = o[dm][2];
      }
      if (h1 < G) {
        c.fo[cw][h1][16 * dm + g8] = o[dm][1];
        c.fo[cw][h1][16 * dm + g8 + 8] = o[dm][3];
      }
    }
    if (lane == 0) c.bad[cw] = ok ? 0 : 1;
  } else if (warp == 5) {
    // ---------------- decider ----------------
    // Lane i owns probe coordinates i and i + 32: it merges the four warps' parts of the
    // first head for them, forms x = O / l (the fp32 divisions run in parallel) and writes
    // the trace. The sums of the test run across the warp (every lane then holds them and
    // takes the same decision); in the fp64 evaluation the products are exact (products
    // of fp32 values) and the sums take the fixed pairwise order of warp_pairwise_sum.
    const int np = a.n_probe;
    const int d0 = lane < np ? a.dims[lane] : 0;
    const int d1 = lane + 32 < np ? a.dims[lane + 32] : 0;
    float xp0 = 0.f, xp1 = 0.f;
    float sp32 = 0.f, np32 = 0.f;  // the fp32 squared norm and norm of x_{t-1}
    int run = 0;
    for (int t = 0; t < ns; ++t) {
      const int slot = t & 1;
      if (!warp_all(tc::mbar_wait(&c.probe_rdy[slot], (t >> 1) & 1, abort_flag, dev_status))) break;
      float f[kCompute];
      const float mx = fmaxf(fmaxf(c.pm[slot][0], c.pm[slot][1]), fmaxf(c.pm[slot][2], c.pm[slot][3]));
#pragma unroll
      for (int w = 0; w < kCompute; ++w) f[w] = c.pm[slot][w] == -INFINITY ? 0.f : ex2(c.pm[slot][w] - mx);
      const float lt = (c.pl[slot][0] * f[0] + c.pl[slot][1] * f[1]) + (c.pl[slot][2] * f[2] + c.pl[slot][3] * f[3]);
      const float u0 = (c.xo[slot][0][d0] * f[0] + c.xo[slot][1][d0] * f[1]) +
                       (c.xo[slot][2][d0] * f[2] + c.xo[slot][3][d0] * f[3]);
      const float u1 = (c.xo[slot][0][d1] * f[0] + c.xo[slot][1][d1] * f[1]) +
                       (c.xo[slot][2][d1] * f[2] + c.xo[slot][3][d1] * f[3]);
      const float x0 = lane < np ? __fdiv_rn(u0, lt) : 0.f;
      const float x1 = lane + 32 < np ? __fdiv_rn(u1, lt) : 0.f;
      if (probe_trace) {
        float* tr = probe_trace + ((size_t)bg * tstride + t) * np;
        if (lane < np) tr[lane] = x0;
        if (lane + 32 < np) tr[lane + 32] = x1;
      }
      // The test in fp32 first, then, only where that cannot decide, in fp64 as defined.
      // With u = 2^-24, at most 64 coordinates (each term of a sum passes at most seven
      // roundings) and both squared norms in [2^-60, 2^60], the fp32 values lie within
      //   |ds32 - ds64| <= 5u (||x|| + ||x'||) + u ds32     (each norm to 4.6u)
      //   |dd32 - dd64| <= 21u    (dot product to 7u ||x|| ||x'||, denominator to 10.2u,
      //                            the divide and the subtract; |dot| <= ||x|| ||x'||)
      // of the fp64 evaluation (whose own error is below 21 * 2^-53). The margins used
      // below, 8u (||x|| + ||x'|| + ds32) and 32u, exceed these bounds with room for the
      // rounding of the comparisons themselves, so a value outside them decides as the
      // fp64 test would.
      const float s32 = warp_sum_f32(__fadd_rn(__fmul_rn(x0, x0), __fmul_rn(x1, x1)));
      const float d32 = warp_sum_f32(__fadd_rn(__fmul_rn(x0, xp0), __fmul_rn(x1, xp1)));
      const float n32 = __fsqrt_rn(s32);
      bool stop = false;
      if (t >= 1) {
        constexpr float kU = 0x1p-24f;
        int verdict = -1;                                   // 0 / 1 decided, -1 open
        if (!(a.tau > 0.f)) {
          verdict = 0;                                      // ds >= 0 is never below it
        } else if (s32 >= 0x1p-60f && s32 <= 0x1p60f && sp32 >= 0x1p-60f && sp32 <= 0x1p60f && isfinite(d32)) {
          const float ds32 = fabsf(__fsub_rn(n32, np32));
          const float e1 = 8.f * kU * (n32 + np32 + ds32);
          if (ds32 - e1 >= a.tau) {
            verdict = 0;
          } else if (ds32 + e1 < a.tau) {
            const float dd32 = __fsub_rn(1.f, __fdiv_rn(d32, __fmul_rn(n32, np32)));
            const float e2 = 32.f * kU;
            if (dd32 + e2 < a.phi) verdict = 1;
            else if (dd32 - e2 >= a.phi) verdict = 0;
          }
        }
        if (verdict < 0) {
          // the defining fp64 evaluation: exact products, pairwise sums, rounded root,
          // product, divide and subtract
          const double sc2 = warp_pairwise_sum(
              __dadd_rn(__dmul_rn((double)x0, (double)x0), __dmul_rn((double)x1, (double)x1)));
          const double sp2 = warp_pairwise_sum(
              __dadd_rn(__dmul_rn((double)xp0, (double)xp0), __dmul_rn((double)xp1, (double)xp1)));
          const double dt = warp_pairwise_sum(
              __dadd_rn(__dmul_rn((double)x0, (double)xp0), __dmul_rn((double)x1, (double)xp1)));
          const double nc = __dsqrt_rn(sc2), npv = __dsqrt_rn(sp2);
          const double ds = fabs(__dadd_rn(nc, -npv));
          bool stable = ds < (double)a.tau;
          if (stable) {
            const double den = __dmul_rn(nc, npv);
            const double dd = (den == 0.0) ? 1.0 : __dadd_rn(1.0, -__ddiv_rn(dt, den));
            stable = dd < (double)a.phi;
          }
          verdict = stable ? 1 : 0;
        }
        run = verdict ? run + 1 : 0;
        stop = a.enable && run >= a.patience;
      }
      xp0 = x0;
      xp1 = x1;
      sp32 = s32;
      np32 = n32;
      if (lane == 0) {
        if (stop) {
          c.stop_at = t;
          *halt = 1;                    // release the producer
        }
        tc::mbar_arrive(&c.decided[slot]);
      }
      if (stop) break;
    }
  }

  // ---------------- teardown ----------------
  __syncthreads();
  if (warp == 0 && lane == 0) {
    for (int t = issued - STAGES < 0 ? 0 : issued - STAGES; t < issued; ++t)
      tc::mbar_wait_timed(&c.kv_full[t % STAGES], (t / STAGES) & 1);
  }
  if (warp >= 1 && warp <= kCompute) {
    const bool all_ok = (c.bad[0] | c.bad[1] | c.bad[2] | c.bad[3]) == 0;
    if (threadIdx.x == 32) blocks_used[bg] = all_ok ? used : 0;
    if (all_ok) {
      // merge the four warps' states: thread i writes head dim i of every head
      const int d = threadIdx.x - 32;
      uint16_t* og = out + ((size_t)b * a.Hq + (size_t)g * G) * HD;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mx = fmaxf(fmaxf(c.fm[0][h], c.fm[1][h]), fmaxf(c.fm[2][h], c.fm[3][h]));
        float f[kCompute];
#pragma unroll
        for (int w = 0; w < kCompute; ++w) f[w] = c.fm[w][h] == -INFINITY ? 0.f : ex2(c.fm[w][h] - mx);
        const float lt = (c.fl[0][h] * f[0] + c.fl[1][h] * f[1]) + (c.fl[2][h] * f[2] + c.fl[3][h] * f[3]);
        const float ov = (c.fo[0][h][d] * f[0] + c.fo[1][h][d] * f[1]) + (c.fo[2][h][d] * f[2] + c.fo[3][h][d] * f[3]);
        og[h * HD + d] = f32_to_bf16_rn(lt > 0.f ? ov / lt : 0.f);
      }
    }
  }
}

bool decode_mma_supported(const bsa_decode_shape& s) {
  const int G = s.Hq / s.Hkv;
  return s.dtype == BSA_BF16 && s.d == HD && s.block_kv == BKV && (G == 1 || G == 2 || G == 4 || G == 8) &&
         (long long)s.B * s.Hkv * s.L < (1ll << 31);
}

cudaError_t launch_decode_mma(const bsa_decode_shape& s, const DecodeArgs& a, const void* q,
                              const void* kc, const void* vc, void* out, int32_t* blocks_used,
                              float* probe_trace, int32_t* dev_status, cudaStream_t st) {
  CUtensorMap mk, mv;
  const uint64_t rows = (uint64_t)s.B * s.Hkv * s.L;
  if (!make_tmap_bf16_2d(&mk, kc, rows, HD, 64, BKV) || !make_tmap_bf16_2d(&mv, vc, rows, HD, 64, BKV))
    return cudaErrorInvalidValue;
  auto kern = decode_mma_kernel<1>;
  switch (s.Hq / s.Hkv) {
    case 1: kern = decode_mma_kernel<1>; break;
    case 2: kern = decode_mma_kernel<2>; break;
    case 4: kern = decode_mma_kernel<4>; break;
    case 8: kern = decode_mma_kernel<8>; break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<s.B * s.Hkv, kThreads, kSmemBytes, st>>>(mk, mv, (const uint16_t*)q, a, (uint16_t*)out, blocks_used,
                                                  probe_trace, dev_status);
  return cudaGetLastError();
}

}  // namespace bsa
