// Decode attention with run-time termination ([ART] 2.1-2.4), CUDA-core kernel:
// serves the shapes the tensor-core decode (decode_mma.cu) does not take
// (d = 64, KV blocks of 64).
//
// One CTA per (batch, KV head). The CTA streams the KV cache in blocks of
// block_kv keys, in order ([ART] 2.1: tile-wise streaming exposes the partial
// output O^(t)), keeping an online softmax for the G query heads of the group.
// After every block it forms the probe x^(t) = O^(t)[first head][probe_dims]
// (fp32, normalised) and, from block 1 on, tests stability in fp64:
//   d_scale = | ||x_t|| - ||x_{t-1}|| |,  d_dir = 1 - x_t.x_{t-1} / (||x_t|| ||x_{t-1}||)
// (d_dir = 1 when a norm is 0), exact products, and each sum over the probe
// coordinates taken by warp 0 in the fixed pairwise order of warp_pairwise_sum
// ([ART] 2.2). A block is stable iff d_scale < tau and d_dir < phi; the
// stream stops after `patience` consecutive stable blocks ([ART] 2.3). Block 0
// is always processed, because no test exists before block 1 ([ART] 2.4).
//
// Data movement: a three-stage ring of cp.async copies (16 bytes per thread
// per copy) brings K and V blocks into shared memory while the previous block
// is computed. K rows are stored with their 16-byte chunks XOR-swizzled by the
// row index, so the one-key-per-thread dot products read shared memory without
// bank conflicts. Waits are cp.async group waits (they complete by
// construction); no spin loops.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace bsa {

namespace {
constexpr int kStages = 3;
constexpr int kThreads = 256;

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kThreads) decode_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc,
    const uint16_t* __restrict__ vc, const DecodeArgs a, uint16_t* __restrict__ out,
    int32_t* __restrict__ blocks_used, float* __restrict__ probe_trace, int32_t* dev_status) {
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  extern __shared__ __align__(16) unsigned char smraw[];
  const int BK = a.block_kv;
  const size_t blk_bytes = (size_t)BK * D * 2;
  unsigned char* ring = smraw;                                   // kStages x (K, V)
  float* qs = reinterpret_cast<float*>(ring + kStages * 2 * blk_bytes);   // [G][D]
  float* S = qs + G * D;                                          // [G][BK]
  float* part = S + G * BK;                                       // [KQ][G][D]
  __shared__ float m_s[G], l_s[G], alpha_s[G];
  __shared__ float xcur[kMaxProbe], xprev[kMaxProbe];
  __shared__ int stop_s, run_s, nsteps_s;
  __shared__ uint16_t blk_s[kMaxDecodeList];     // visit list (decode over a block list)

  const int bg = blockIdx.x;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int nb = a.L / BK;
  const uint16_t* kbase = kc + (size_t)bg * a.L * D;
  const uint16_t* vbase = vc + (size_t)bg * a.L * D;
  const int tid = threadIdx.x;

  for (int i = tid; i < G * D; i += kThreads)
    qs[i] = bf16_to_f32(q[((size_t)b * a.Hq + (size_t)g * G) * D + i]);
  if (tid < G) { m_s[tid] = -INFINITY; l_s[tid] = 0.f; }
  if (tid == 0) { stop_s = 0; run_s = 0; }
  if (tid < 32) {
    int n = nb;
    if (a.blist)
      n = warp_compact_blocks(a.blist + (size_t)bg * a.list_w, a.bcnt[bg], a.list_w, nb, blk_s,
                              dev_status, tid);
    if (tid == 0) nsteps_s = n;
  }
  __syncthreads();
  const int ns = nsteps_s;                            // visit steps
  const int tstride = a.blist ? a.list_w : nb;        // probe-trace rows per group

  auto issue = [&](int blk) {
    if (blk < ns) {
      unsigned char* ks = ring + (size_t)(blk % kStages) * 2 * blk_bytes;
      unsigned char* vs = ks + blk_bytes;
      const size_t src = a.blist ? (size_t)blk_s[blk] : (size_t)blk;
      const unsigned char* kg = reinterpret_cast<const unsigned char*>(kbase + src * BK * D);
      const unsigned char* vg = reinterpret_cast<const unsigned char*>(vbase + src * BK * D);
      const int chunks = BK * CPR;
      for (int c = tid; c < chunks; c += kThreads) {
        const int r = c / CPR, cc = c % CPR;
        cp_async16(ks + (size_t)r * D * 2 + ((cc ^ (r % CPR)) * 16), kg + (size_t)c * 16);
        cp_async16(vs + (size_t)c * 16, vg + (size_t)c * 16);
      }
    }
    cp_async_commit();
  };

  // thread roles for the value product: (d pair, key group)
  constexpr int DP = D / 2;
  constexpr int KQ = kThreads / DP;
  const int dp = tid % DP, kq = tid / DP;
  float acc[G][2];
#pragma unroll
  for (int h = 0; h < G; ++h) { acc[h][0] = 0.f; acc[h][1] = 0.f; }

  for (int s = 0; s < kStages - 1; ++s) issue(s);
  int used = ns;
  for (int blk = 0; blk < ns; ++blk) {
    issue(blk + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncthreads();
    const unsigned char* ks = ring + (size_t)(blk % kStages) * 2 * blk_bytes;
    const uint16_t* vs = reinterpret_cast<const uint16_t*>(ks + blk_bytes);

    // scores: one key per thread, heads split over the thread groups
    const int HS = kThreads / BK;
    const int key = tid % BK, hs = tid / BK;
    {
      float dot[(G + 1) / 2 + 1];
      const int nh = (G - hs + HS - 1) / HS;
#pragma unroll
      for (int i = 0; i < (G + 1) / 2 + 1; ++i) dot[i] = 0.f;
      const unsigned char* krow = ks + (size_t)key * D * 2;
#pragma unroll 4
      for (int cc = 0; cc < CPR; ++cc) {
        uint4 u = *reinterpret_cast<const uint4*>(krow + ((cc ^ (key % CPR)) * 16));
        const uint16_t* e = reinterpret_cast<const uint16_t*>(&u);
        float kf[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) kf[x] = bf16_to_f32(e[x]);
#pragma unroll
        for (int i = 0; i < (G + 1) / 2 + 1; ++i) {
          if (i < nh) {
            const float* qh = qs + (hs + i * HS) * D + cc * 8;
#pragma unroll
            for (int x = 0; x < 8; ++x) dot[i] = fmaf(qh[x], kf[x], dot[i]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < (G + 1) / 2 + 1; ++i)
        if (i < nh) S[(hs + i * HS) * BK + key] = dot[i] * a.scale_log2;
    }
    __syncthreads();
    // online softmax: warp w handles head w
    {
      const int w = tid / 32, lane = tid % 32;
      if (w < G) {
        float mx = -INFINITY;
        for (int kk = lane; kk < BK; kk += 32) mx = fmaxf(mx, S[w * BK + kk]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float mo = m_s[w];
        const float mn = fmaxf(mo, mx);
        float sum = 0.f;
        for (int kk = lane; kk < BK; kk += 32) {
          const float p = exp2f(S[w * BK + kk] - mn);
          S[w * BK + kk] = p;
          sum += p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
          const float al = exp2f(mo - mn);     // 0 on the first block (mo = -inf)
          alpha_s[w] = al;
          l_s[w] = l_s[w] * al + sum;
          m_s[w] = mn;
        }
      }
    }
    __syncthreads();
    // value product over this thread's key group
    {
#pragma unroll
      for (int h = 0; h < G; ++h) { acc[h][0] *= alpha_s[h]; acc[h][1] *= alpha_s[h]; }
      const int kpg = BK / KQ;
      for (int kk = kq * kpg; kk < (kq + 1) * kpg; ++kk) {
        const uint32_t v2 = *reinterpret_cast<const uint32_t*>(vs + (size_t)kk * D + 2 * dp);
        const float v0 = bf16_to_f32((uint16_t)(v2 & 0xffffu));
        const float v1 = bf16_to_f32((uint16_t)(v2 >> 16));
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float p = S[h * BK + kk];
          acc[h][0] = fmaf(p, v0, acc[h][0]);
          acc[h][1] = fmaf(p, v1, acc[h][1]);
        }
      }
    }
    // probe: head 0 of the group, normalised, at the probe coordinates
    part[kq * D + 2 * dp] = acc[0][0];
    part[kq * D + 2 * dp + 1] = acc[0][1];
    __syncthreads();
    if (tid < a.n_probe) {
      const int dd = a.dims[tid];
      float s = 0.f;
      for (int p = 0; p < KQ; ++p) s = __fadd_rn(s, part[p * D + dd]);
      const float x = __fdiv_rn(s, l_s[0]);
      xcur[tid] = x;
      if (probe_trace) probe_trace[((size_t)bg * tstride + blk) * a.n_probe + tid] = x;
    }
    __syncthreads();
    if (tid < 32) {
      // lane i: coordinates i and i + 32 (zero where there is none)
      const int n = a.n_probe;
      const double a0 = tid < n ? (double)xcur[tid] : 0.0, a1 = tid + 32 < n ? (double)xcur[tid + 32] : 0.0;
      const double b0 = tid < n ? (double)xprev[tid] : 0.0, b1 = tid + 32 < n ? (double)xprev[tid + 32] : 0.0;
      if (blk >= 1) {
        const double sc = warp_pairwise_sum(__dadd_rn(__dmul_rn(a0, a0), __dmul_rn(a1, a1)));
        const double sp = warp_pairwise_sum(__dadd_rn(__dmul_rn(b0, b0), __dmul_rn(b1, b1)));
        const double dt = warp_pairwise_sum(__dadd_rn(__dmul_rn(a0, b0), __dmul_rn(a1, b1)));
        if (tid == 0) {
          const double nc = __dsqrt_rn(sc), np = __dsqrt_rn(sp);
          const double ds = fabs(__dadd_rn(nc, -np));
          const double den = __dmul_rn(nc, np);
          const double dd = (den == 0.0) ? 1.0 : __dadd_rn(1.0, -__ddiv_rn(dt, den));
          const bool stable = (ds < (double)a.tau) && (dd < (double)a.phi);
          run_s = stable ? run_s + 1 : 0;
          if (a.enable && run_s >= a.patience) stop_s = 1;
        }
      }
      __syncwarp();
      if (tid < n) xprev[tid] = xcur[tid];
      if (tid + 32 < n) xprev[tid + 32] = xcur[tid + 32];
    }
    __syncthreads();
    if (stop_s) { used = blk + 1; break; }
  }
  cp_async_wait<0>();
  __syncthreads();

  // final output: sum the key-group partials in order, normalise, store bf16
#pragma unroll
  for (int h = 0; h < G; ++h) {
    part[(kq * G + h) * D + 2 * dp] = acc[h][0];
    part[(kq * G + h) * D + 2 * dp + 1] = acc[h][1];
  }
  __syncthreads();
  for (int i = tid; i < G * D; i += kThreads) {
    const int h = i / D, dd = i % D;
    float s = 0.f;
    for (int p = 0; p < KQ; ++p) s += part[(p * G + h) * D + dd];
    const float l = l_s[h];
    out[((size_t)b * a.Hq + (size_t)g * G + h) * D + dd] = f32_to_bf16_rn(l > 0.f ? s / l : 0.f);
  }
  if (tid == 0) blocks_used[bg] = used;
}

template <int D, int G>
static cudaError_t launch_decode_t(const bsa_decode_shape& s, const DecodeArgs& a, const void* q,
                                   const void* kc, const void* vc, void* out, int32_t* blocks_used,
                                   float* probe_trace, int32_t* dev_status, cudaStream_t st) {
  const int KQ = kThreads / (D / 2);
  size_t smem = (size_t)kStages * 2 * s.block_kv * D * 2 + (size_t)G * D * 4 +
                (size_t)G * s.block_kv * 4 + (size_t)KQ * G * D * 4;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_kernel<D, G><<<s.B * s.Hkv, kThreads, smem, st>>>(
      (const uint16_t*)q, (const uint16_t*)kc, (const uint16_t*)vc, a, (uint16_t*)out, blocks_used,
      probe_trace, dev_status);
  return cudaGetLastError();
}

cudaError_t launch_decode(const bsa_decode_shape& s, const bsa_decode_params& p, const void* q,
                          const void* kc, const void* vc, float scale, void* out,
                          int32_t* blocks_used, float* probe_trace, int32_t* dev_status,
                          cudaStream_t st, const int32_t* block_list, const int32_t* list_cnt,
                          int list_w) {
  // the CUDA-core kernel below has no mbarrier waits; its only data-dependent indices
  // are visit-list entries, which it checks against the cache length
  DecodeArgs a;
  a.L = s.L; a.block_kv = s.block_kv; a.Hq = s.Hq; a.Hkv = s.Hkv;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.tau = p.tau; a.phi = p.phi; a.patience = p.patience; a.enable = p.enable;
  a.n_probe = p.n_probe;
  for (int i = 0; i < kMaxProbe; ++i) a.dims[i] = i < p.n_probe ? p.probe_dims[i] : 0;
  a.blist = block_list;
  a.bcnt = list_cnt;
  a.list_w = block_list ? list_w : 0;
  if (decode_mma_supported(s))
    return launch_decode_mma(s, a, q, kc, vc, out, blocks_used, probe_trace, dev_status, st);
  const int G = s.Hq / s.Hkv;
#define BSA_DEC(D)                                                                             \
  switch (G) {                                                                                 \
    case 1: return launch_decode_t<D, 1>(s, a, q, kc, vc, out, blocks_used, probe_trace, dev_status, st); \
    case 2: return launch_decode_t<D, 2>(s, a, q, kc, vc, out, blocks_used, probe_trace, dev_status, st); \
    case 4: return launch_decode_t<D, 4>(s, a, q, kc, vc, out, blocks_used, probe_trace, dev_status, st); \
    case 8: return launch_decode_t<D, 8>(s, a, q, kc, vc, out, blocks_used, probe_trace, dev_status, st); \
    default: return cudaErrorInvalidValue;                                                     \
  }
  if (s.d == 128) { BSA_DEC(128) } else { BSA_DEC(64) }
#undef BSA_DEC
}

}  // namespace bsa
