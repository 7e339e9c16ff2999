// Decode attention with run-time termination on Blackwell tensor cores
// ([ART] 2.1-2.4): the KV cache of one (batch, KV head) is streamed block by
// block, in order (or in the order of a caller's visit list, compacted into
// shared memory by warp 6 before the pipeline starts); after each block the
// normalised partial output O^(t) is probed, and from the second visit step on
// the stability test decides whether to stop.
//
// One CTA per (batch, KV head), 224 threads:
//   warp 0 (one thread)  TMA producer: K and V blocks of 128 keys, a ring of
//                        three stages (64 KB each), until told to halt.
//   warp 1 (one thread)  MMA issuer: S_t = K_t Q^T (M = 128 keys, N = 16: the
//                        group's query heads padded with zero rows) into one of
//                        two TMEM buffers; after the softmax warps publish P_t,
//                        D_t = V_t^T P_t^T (M = 128 head dims, V_t read as an
//                        MN-major operand straight from its TMA tile).
//   warps 2-5            softmax and fold: a thread owns TMEM lane r, i.e. key r of
//                        S_t and head dim r of D_t. Per head: the block max across
//                        the four warps (shared memory + a bounded mbarrier
//                        handshake), P_t to shared memory (bf16, 128-byte swizzle),
//                        then O[h][r] = O[h][r] * alpha_h + D_t[r][h] in registers;
//                        each warp keeps its own part of the row sums l.
//   warp 6               decider: for block t it forms the probe
//                        x^(t) = O^(t)[first head][probe dims] / l (fp32; l = the
//                        four warp parts added in a fixed order) and runs the fp64
//                        stability test (exact products, sums in a fixed pairwise
//                        order across the warp), then publishes stop / continue.
// The work is software-pipelined: the MMA issuer computes S_{t+1} before PV_t,
// and the softmax warps produce P_{t+1} (two P buffers) before they fold D_t, so
// the softmax of one block overlaps the value product of the previous one. The
// decider judges block t while the softmax warps go on with blocks t+1 and t+2;
// they read that verdict only before folding D_{t+2}, keeping a copy of O^(t)
// until then, and on a stop return that copy. After a stop the producer and MMA
// threads are released through a halt flag; the MMA issuer may then never issue
// the next S, so the softmax warps' wait for it also watches the halt flag (and
// then reads the verdicts still open), and the four warps act on one verdict
// (posted per warp and joined through the bounded `vote` mbarrier). The MMA
// issuer keeps issuing PV_t for every P_t published until the softmax warps
// leave. The CTA then waits for its own copies and MMAs and frees TMEM. All
// waits are bounded.
// Shapes: bf16, d = 128, KV blocks of 128, Hq/Hkv <= 8.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace bsa {

namespace {
constexpr int HD = 128;
constexpr int BKV = 128;
constexpr int NPAD = 16;
constexpr int GMAX = 8;
constexpr int STAGES = 3;
constexpr int kThreads = 224;
constexpr uint32_t kHalf = 16384;         // 128 rows x 128 bytes
constexpr uint32_t kTile = 2 * kHalf;     // one K or V block
constexpr uint32_t kStage = 2 * kTile;    // K + V
constexpr uint32_t kSmallHalf = 2048;     // 16 rows x 128 bytes
constexpr uint32_t kTmemCols = 64;        // S[2] at 0/16, D[2] at 32/48

struct __align__(8) Ctrl {
  uint64_t kv_full[STAGES], kv_empty[STAGES];
  uint64_t s_full[2], o_full[2];
  uint64_t p_ready[2], probe_rdy[2], decided[2], done, vote;   // probe_rdy, decided: by block parity
  uint32_t tmem;
  int abort_flag;     // error: softmax warps unwind
  int halt;           // producer / MMA stop issuing (normal stop or error)
  int sm_quit;        // the softmax warps left their loop: no further P_t will come
  int stop_at;        // block after which the decider stopped, or -1
  float rmax[2][4][GMAX];       // [block parity][warp][head]
  float lpart[2][4];            // [block parity][warp] row-sum part of the first head
  float xfull[2][HD];           // [block parity][head dim] unnormalised O of the first head
  float lfin[4][GMAX];          // [warp][head] final row-sum parts
  int swait[2][4];              // softmax warps' wait results for S_t, by t parity
  int n_steps;                  // blocks to visit
  uint16_t blk[kMaxDecodeList]; // visit list (decode over a block list)
};

constexpr size_t kSmemStages = 0;
constexpr size_t kSmemQ = kSmemStages + STAGES * kStage;
constexpr size_t kSmemP = kSmemQ + 2 * kSmallHalf;            // two P buffers of 4 KB
constexpr size_t kSmemCtrl = kSmemP + 4 * kSmallHalf;
constexpr size_t kSmemBytes = kSmemCtrl + sizeof(Ctrl) + 1024;

__device__ __forceinline__ bool warp_all(bool x) { return __all_sync(0xffffffffu, x); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// byte offset of element (row, col) in a 128-byte-swizzled K-major [rows x 128] operand
// stored as two 64-column halves of half_bytes each
__device__ __forceinline__ uint32_t sw128_off(int row, int col, uint32_t half_bytes) {
  const int half = col >> 6, c = col & 63;
  return half * half_bytes + row * 128 + ((((c >> 3) ^ (row & 7)) & 7) << 4) + (c & 7) * 2;
}
}  // namespace

template <int G>
__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(
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
  const uint32_t sQ = tc::smem_u32(sm + kSmemQ);
  const uint32_t sP = tc::smem_u32(sm + kSmemP);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&c.kv_full[s], 1);
      tc::mbar_init(&c.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&c.s_full[i], 1);
      tc::mbar_init(&c.o_full[i], 1);
    }
    tc::mbar_init(&c.vote, 4);
    tc::mbar_init(&c.p_ready[0], 4);
    tc::mbar_init(&c.p_ready[1], 4);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&c.probe_rdy[i], 4);
      tc::mbar_init(&c.decided[i], 1);
    }
    tc::mbar_init(&c.done, 1);
    c.abort_flag = 0;
    c.halt = 0;
    c.sm_quit = 0;
    c.stop_at = -1;
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&c.tmem, kTmemCols);
    tc::tmem_relinquish();
  }
  if (warp == 6) {
    int n = nb;
    if (a.blist)
      n = warp_compact_blocks(a.blist + (size_t)bg * a.list_w, a.bcnt[bg], a.list_w, nb, c.blk,
                              dev_status, lane);
    if (lane == 0) c.n_steps = n;
  }
  if (warp >= 2 && warp <= 5) {
    // Q rows of the group (zero rows up to 16) and an all-zero P, both as K-major
    // 128-byte-swizzled MMA operands
    const int tid = threadIdx.x - 64;
    uint32_t* qz = reinterpret_cast<uint32_t*>(sm + kSmemQ);
    for (int i = tid; i < (int)(6 * kSmallHalf / 4); i += 128) qz[i] = 0u;   // Q and both P buffers
    __syncwarp();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const uint16_t* qg = q + ((size_t)b * a.Hq + (size_t)g * G) * HD;
    for (int e = tid; e < G * HD; e += 128) {
      const int h = e / HD, col = e % HD;
      *reinterpret_cast<uint16_t*>(sm + kSmemQ + sw128_off(h, col, kSmallHalf)) = qg[e];
    }
    tc::fence_proxy_async_smem();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = c.tmem;
  const int ns = c.n_steps;                         // visit steps
  const int tstride = a.blist ? a.list_w : nb;      // probe-trace rows per group
  volatile int* abort_flag = &c.abort_flag;
  volatile int* halt = &c.halt;
  volatile int* sm_quit = &c.sm_quit;
  int issued = 0;
  bool mma_issued = false;
  float o_fin[G];           // softmax warps: unnormalised output of this thread's head dim
  bool out_ok = false;

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
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idS = tc::idesc_bf16_f32(128, NPAD, false, false);
    constexpr uint32_t idD = tc::idesc_bf16_f32(128, NPAD, true, false);
    auto issue_s = [&](int t) -> bool {
      const int s = t % STAGES;
      if (!tc::mbar_wait_halt(&c.kv_full[s], (t / STAGES) & 1, halt, dev_status)) return false;
      tc::tc_fence_after();
      const uint32_t kb = sStages + s * kStage;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
        const uint32_t qoff = (kk >> 2) * kSmallHalf + (kk & 3) * 32;
        tc::umma_bf16(tmem + (t & 1) * NPAD, tc::sdesc_sw128(kb + off, 16, 1024),
                      tc::sdesc_sw128(sQ + qoff, 16, 1024), idS, kk > 0);
      }
      tc::umma_commit(&c.s_full[t & 1]);
      mma_issued = true;
      return true;
    };
    bool ok = ns > 0 && issue_s(0);
    for (int t = 0; ok && t < ns; ++t) {
      // S_{t+1} first: its buffer held S_{t-1}, which the softmax warps read before P_{t-1}
      if (t + 1 < ns && !issue_s(t + 1)) break;
      // P_t comes unless the softmax warps quit first (they do after a stop is seen or on
      // an error); a halt alone must not skip PV_t once S_{t+1} is issued, since the
      // softmax warps that received S_{t+1} then wait for D_t
      if (!tc::mbar_wait_halt(&c.p_ready[t & 1], (t >> 1) & 1, sm_quit, dev_status)) break;
      tc::tc_fence_after();
      const int s = t % STAGES;
      const uint32_t vb = sStages + s * kStage + kTile;
      const uint32_t pb = sP + (t & 1) * 2 * kSmallHalf;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t poff = (kk >> 2) * kSmallHalf + (kk & 3) * 32;
        tc::umma_bf16(tmem + 32 + (t & 1) * NPAD, tc::sdesc_sw128(vb + kk * 2048, kHalf, 1024),
                      tc::sdesc_sw128(pb + poff, 16, 1024), idD, kk > 0);
      }
      tc::umma_commit(&c.o_full[t & 1]);
      tc::umma_commit(&c.kv_empty[s]);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ---------------- softmax and fold ----------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;           // key of S_t, head dim of D_t
    const uint32_t tl = tmem + ((uint32_t)(quarter * 32) << 16);
    // m, o per head; lw[0] is this warp's part of the first head's row sum (the probe needs
    // it after every block), lw[h > 0] this thread's part (reduced once, at the end)
    float m[G], lw[G], o[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { m[h] = -INFINITY; lw[h] = 0.f; o[h] = 0.f; }
    // softmax of block t: writes P_t, returns alpha_t and the block sums (ps[0]: this warp's
    // part; ps[h > 0]: this thread's key). 0: done; 1: a stop was decided before S_t arrived
    // (the MMA issuer may never issue it: it halts once the decider stops, possibly before
    // block t landed); 2: error. P_t is published (p_ready) only when 0 is returned.
    auto softmax = [&](int t, float (&alpha)[G], float (&ps)[G]) -> int {
      const int buf = t & 1;
      const int w = __reduce_max_sync(0xffffffffu, (unsigned)tc::mbar_wait_or_halt(
                                          &c.s_full[buf], (t >> 1) & 1, halt, abort_flag, dev_status));
      float sc[G];
      if (w == 0) {
        // S_t landed for this warp: its scores and, per head, the warp's block max as an
        // order-preserving key reduced in one instruction
        tc::tc_fence_after();
        uint32_t sv[16];
        tc::tmem_ld16(tl + buf * NPAD, sv);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          sc[h] = __uint_as_float(sv[h]);
          const uint32_t key = (sv[h] & 0x80000000u) ? ~sv[h] : (sv[h] | 0x80000000u);
          const uint32_t mk = __reduce_max_sync(0xffffffffu, key);
          if (lane == 0) c.rmax[buf][quarter][h] = __uint_as_float((mk & 0x80000000u) ? (mk & 0x7fffffffu) : ~mk);
        }
      }
      // one handshake for both: the four warps act on one verdict (one may see S_t land while
      // another sees the halt first) and exchange their block maxima. Each posts its result
      // (and maxima) and arrives on `vote` (phase t); a warp writes slot t&1 again only after
      // every warp arrived for t+1, i.e. read its slot-t values
      if (lane == 0) c.swait[t & 1][quarter] = w;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.vote);
      if (!warp_all(tc::mbar_wait(&c.vote, t & 1, abort_flag, dev_status))) return 2;
      const int v = max(max(c.swait[t & 1][0], c.swait[t & 1][1]), max(c.swait[t & 1][2], c.swait[t & 1][3]));
      if (v != 0) return v;
      uint8_t* pbase = sm + kSmemP + buf * 2 * kSmallHalf;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float bmax = fmaxf(fmaxf(c.rmax[buf][0][h], c.rmax[buf][1][h]),
                                 fmaxf(c.rmax[buf][2][h], c.rmax[buf][3][h]));
        const float mn = fmaxf(m[h], bmax * a.scale_log2);
        alpha[h] = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - mn);
        m[h] = mn;
        const float p = ex2(fmaf(sc[h], a.scale_log2, -mn));
        *reinterpret_cast<__nv_bfloat16*>(pbase + sw128_off(h, r, kSmallHalf)) = __float2bfloat16_rn(p);
        ps[h] = p;
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.p_ready[buf]);     // the MMA issuer may start PV_t
      float v0 = ps[0];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v0 += __shfl_xor_sync(0xffffffffu, v0, off);
      ps[0] = v0;
      return 0;
    };
    int used = ns;
    bool ok = true;
    float a_cur[G], p_cur[G], a_nxt[G], p_nxt[G];
    // O^(t-2) and its row-sum parts: the verdict on a block is read two blocks later, so
    // the decider's test runs beside the next block's softmax and fold
    float o_sv[G], l_sv[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { o_sv[h] = 0.f; l_sv[h] = 0.f; }
    // after a halt seen in block t: the stop is on block t-2 or t-1 (the verdicts before
    // were read, and said go on). Returns that block, or -1 (error).
    auto find_stop = [&](int t) -> int {
      for (int sb = t - 2 < 0 ? 0 : t - 2; sb < t; ++sb) {
        if (!warp_all(tc::mbar_wait(&c.decided[sb & 1], (sb >> 1) & 1, abort_flag, dev_status))) return -1;
        if (c.stop_at == sb) return sb;
      }
      return -1;
    };
    // the result is O^(sb) for a stop on block sb: the saved copy when sb = t-2, else the
    // current O (folded through t-1)
    auto take = [&](int sb, int t) {
      if (sb == t - 2) {
#pragma unroll
        for (int h = 0; h < G; ++h) { o[h] = o_sv[h]; lw[h] = l_sv[h]; }
      }
      used = sb + 1;
    };
    if (ns > 0) ok = softmax(0, a_cur, p_cur) == 0;  // an empty visit list leaves O = 0
    for (int t = 0; ok && t < ns; ++t) {
      const int buf = t & 1;
      if (t + 1 < ns) {
        const int rs = softmax(t + 1, a_nxt, p_nxt);  // P_{t+1} while PV_t runs
        if (rs == 1) {
          // halted before S_{t+1}: a stop was decided on block t-2 or t-1
          const int sb = find_stop(t);
          ok = sb >= 0;
          if (ok) take(sb, t);
          break;
        }
        ok = rs == 0;
        if (!ok) break;
      }
      // PV_t is issued: P_t was published, and the MMA issuer only skips it once this loop
      // has ended
      ok = warp_all(tc::mbar_wait(&c.o_full[buf], (t >> 1) & 1, abort_flag, dev_status));
      if (!ok) break;
      tc::tc_fence_after();
      uint32_t dv[16];
      tc::tmem_ld16(tl + 32 + buf * NPAD, dv);
      tc::tc_fence_before();
      if (t >= 2) {
        // the verdict on block t-2 (it also frees that block's probe slot, reused below)
        ok = warp_all(tc::mbar_wait(&c.decided[buf], ((t - 2) >> 1) & 1, abort_flag, dev_status));
        if (!ok) break;
        if (c.stop_at == t - 2) {
          take(t - 2, t);
          break;
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        o_sv[h] = o[h];
        l_sv[h] = lw[h];
        o[h] = fmaf(o[h], a_cur[h], __uint_as_float(dv[h]));
        lw[h] = fmaf(lw[h], a_cur[h], p_cur[h]);
        a_cur[h] = a_nxt[h];
        p_cur[h] = p_nxt[h];
      }
      c.xfull[buf][r] = o[0];
      if (lane == 0) c.lpart[buf][quarter] = lw[0];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&c.probe_rdy[buf]);
    }
    if (ok && used == ns && ns >= 2) {
      // every block was folded; the verdict on block ns-2 is still unread (one on ns-1
      // would leave the result as it is)
      const int sb = ns - 2;
      ok = warp_all(tc::mbar_wait(&c.decided[sb & 1], (sb >> 1) & 1, abort_flag, dev_status));
      if (ok && c.stop_at == sb) take(sb, ns);
    }
#pragma unroll
    for (int h = 1; h < G; ++h) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) lw[h] += __shfl_xor_sync(0xffffffffu, lw[h], off);
    }
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) c.lfin[quarter][h] = lw[h];
    }
    if (threadIdx.x == 64) {
      *sm_quit = 1;
      *halt = 1;                       // nothing more to stream
      blocks_used[bg] = ok ? used : 0;
    }
    // the output is written after the teardown barrier, when every warp's l part is in
    out_ok = warp_all(ok);
#pragma unroll
    for (int h = 0; h < G; ++h) o_fin[h] = o[h];
  } else if (warp == 6) {
    // ---------------- decider ----------------
    // Lane i owns probe coordinates i and i + 32: it forms x = O / l for them (the
    // fp32 divisions run in parallel), writes the trace, and the fp64 products x_t^2 and
    // x_t x_{t-1} (exact: products of fp32 values). The sums run across the warp in the
    // fixed pairwise order of warp_pairwise_sum; every lane then holds them and takes the
    // same decision. ||x_{t-1}|| is the previous block's root (the same sum of the same
    // values).
    const int np = a.n_probe;
    const int d0 = lane < np ? a.dims[lane] : 0;
    const int d1 = lane + 32 < np ? a.dims[lane + 32] : 0;
    float xp0 = 0.f, xp1 = 0.f;
    double np_prev = 0.0;          // ||x_{t-1}||
    int run = 0;
    for (int t = 0; t < ns; ++t) {
      if (!warp_all(tc::mbar_wait(&c.probe_rdy[t & 1], (t >> 1) & 1, abort_flag, dev_status))) break;
      const int buf = t & 1;
      const float lt = (c.lpart[buf][0] + c.lpart[buf][1]) + (c.lpart[buf][2] + c.lpart[buf][3]);
      const float x0 = lane < np ? __fdiv_rn(c.xfull[buf][d0], lt) : 0.f;
      const float x1 = lane + 32 < np ? __fdiv_rn(c.xfull[buf][d1], lt) : 0.f;
      if (probe_trace) {
        float* tr = probe_trace + ((size_t)bg * tstride + t) * np;
        if (lane < np) tr[lane] = x0;
        if (lane + 32 < np) tr[lane + 32] = x1;
      }
      const double sc2 = warp_pairwise_sum(
          __dadd_rn(__dmul_rn((double)x0, (double)x0), __dmul_rn((double)x1, (double)x1)));
      const double dt = warp_pairwise_sum(
          __dadd_rn(__dmul_rn((double)x0, (double)xp0), __dmul_rn((double)x1, (double)xp1)));
      xp0 = x0;
      xp1 = x1;
      const double nc = __dsqrt_rn(sc2);
      bool stop = false;
      if (t >= 1) {
        const double ds = fabs(__dadd_rn(nc, -np_prev));
        const double den = __dmul_rn(nc, np_prev);
        const double dd = (den == 0.0) ? 1.0 : __dadd_rn(1.0, -__ddiv_rn(dt, den));
        const bool stable = (ds < (double)a.tau) && (dd < (double)a.phi);
        run = stable ? run + 1 : 0;
        stop = a.enable && run >= a.patience;
      }
      np_prev = nc;
      if (lane == 0) {
        if (stop) {
          c.stop_at = t;
          *halt = 1;                    // release the producer and the MMA issuer
        }
        tc::mbar_arrive(&c.decided[t & 1]);
      }
      if (stop) break;
    }
  }

  // ---------------- teardown ----------------
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0) {
    for (int t = issued - STAGES < 0 ? 0 : issued - STAGES; t < issued; ++t)
      tc::mbar_wait_timed(&c.kv_full[t % STAGES], (t / STAGES) & 1);
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
  if (warp >= 2 && warp <= 5 && out_ok) {
    const int r = (warp & 3) * 32 + lane;
    uint16_t* og = out + ((size_t)b * a.Hq + (size_t)g * G) * HD;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float lt = (c.lfin[0][h] + c.lfin[1][h]) + (c.lfin[2][h] + c.lfin[3][h]);
      og[h * HD + r] = f32_to_bf16_rn(lt > 0.f ? o_fin[h] / lt : 0.f);
    }
  }
}

bool decode_tc_supported(const bsa_decode_shape& s) {
  const int G = s.Hq / s.Hkv;
  return s.dtype == BSA_BF16 && s.d == HD && s.block_kv == BKV && (G == 1 || G == 2 || G == 4 || G == 8) &&
         (long long)s.B * s.Hkv * s.L < (1ll << 31);
}

cudaError_t launch_decode_tc(const bsa_decode_shape& s, const DecodeArgs& a, const void* q,
                             const void* kc, const void* vc, void* out, int32_t* blocks_used,
                             float* probe_trace, int32_t* dev_status, cudaStream_t st) {
  CUtensorMap mk, mv;
  const uint64_t rows = (uint64_t)s.B * s.Hkv * s.L;
  if (!make_tmap_bf16_2d(&mk, kc, rows, HD, 64, BKV) || !make_tmap_bf16_2d(&mv, vc, rows, HD, 64, BKV))
    return cudaErrorInvalidValue;
  auto kern = decode_tc_kernel<1>;
  switch (s.Hq / s.Hkv) {
    case 1: kern = decode_tc_kernel<1>; break;
    case 2: kern = decode_tc_kernel<2>; break;
    case 4: kern = decode_tc_kernel<4>; break;
    case 8: kern = decode_tc_kernel<8>; break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<s.B * s.Hkv, kThreads, kSmemBytes, st>>>(mk, mv, (const uint16_t*)q, a, (uint16_t*)out, blocks_used,
                                                  probe_trace, dev_status);
  return cudaGetLastError();
}

}  // namespace bsa
