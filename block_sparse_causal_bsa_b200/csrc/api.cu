// C ABI of libbsa.so: argument validation, workspace layout and kernel dispatch.
// Nothing here allocates device memory; every buffer is the caller's.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace {

thread_local char g_err[512] = "";

bsa_status fail(bsa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

bsa_status ok() {
  g_err[0] = '\0';
  return BSA_OK;
}

bsa_status cuda_fail(cudaError_t e, const char* where) {
  return fail(BSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bsa_status check_shape(const bsa_shape* s) {
  if (!s) return fail(BSA_ERR_INVALID_ARG, "shape is NULL");
  if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->N < 1)
    return fail(BSA_ERR_INVALID_ARG, "B, Hq, Hkv, N must be >= 1");
  if (s->Hq % s->Hkv) return fail(BSA_ERR_INVALID_ARG, "Hq %% Hkv != 0");
  if (s->d != 64 && s->d != 128) return fail(BSA_ERR_UNSUPPORTED, "d must be 64 or 128");
  if ((s->block_k != 64 && s->block_k != 128) || (s->tile_q != 64 && s->tile_q != 128))
    return fail(BSA_ERR_UNSUPPORTED, "block_k and tile_q must be 64 or 128");
  if (s->N % s->block_k || s->N % s->tile_q)
    return fail(BSA_ERR_INVALID_ARG, "N must be a multiple of block_k and tile_q");
  if (s->dtype != BSA_BF16 && s->dtype != BSA_F32)
    return fail(BSA_ERR_INVALID_ARG, "unknown dtype");
  if ((long long)s->B * s->Hq * (s->N / s->tile_q) > (1ll << 31) - 1)
    return fail(BSA_ERR_UNSUPPORTED, "too many query tiles");
  return BSA_OK;
}

bsa_status check_params(const bsa_shape* s, const bsa_select_params* p) {
  if (!p) return fail(BSA_ERR_INVALID_ARG, "params is NULL");
  if (p->k_last < 1 || p->k_first < p->k_last)
    return fail(BSA_ERR_INVALID_ARG, "need 1 <= k_last <= k_first");
  if (p->rho < 1) return fail(BSA_ERR_INVALID_ARG, "rho must be >= 1");
  if (!(p->gate_quantile <= 1.0f))
    return fail(BSA_ERR_INVALID_ARG, "gate_quantile must be <= 1 (negative = fixed threshold)");
  if (s->N / s->block_k > bsa::kMaxCandidates)
    return fail(BSA_ERR_UNSUPPORTED, "more than %d key blocks", bsa::kMaxCandidates);
  if ((long long)s->B * (s->N / s->tile_q) > bsa::kMaxGateTiles)
    return fail(BSA_ERR_UNSUPPORTED, "B * n_qt above %d", bsa::kMaxGateTiles);
  return BSA_OK;
}

bool attend_on_tensor_cores(const bsa_shape& s, int W) {
  return bsa::attend_tc_supported(s) && W <= 1024 && (long long)s.B * s.Hq * s.N < (1ll << 31);
}

struct ScoreWs {
  float* kbar;       // pooled keys, or kmin (bounds)
  float* kbar2;      // kmax (bounds)
  uint16_t* h16;     // fp16 tensor-core operand scaled by 2^r per block: pooled keys, or mid
  uint16_t* h16b;    // bounds: rad, same scale
  float* kinv;       // 2^-r per block
  float* w;          // value-block term (output-aware kinds)
  size_t bytes;
};

bool known_kind(bsa_score_kind kind) {
  return kind == BSA_SCORE_MEAN || kind == BSA_SCORE_MEAN_VNORM || kind == BSA_SCORE_MEAN_VLOG ||
         kind == BSA_SCORE_KMINMAX;
}

ScoreWs score_ws(const bsa_shape& s, bsa_score_kind kind, void* base) {
  const size_t nk = (size_t)s.B * s.Hkv * (s.N / s.block_k);
  const bool bounds = kind == BSA_SCORE_KMINMAX;
  const bool vterm = kind == BSA_SCORE_MEAN_VNORM || kind == BSA_SCORE_MEAN_VLOG;
  ScoreWs w{};
  size_t off = 0;
  char* p = (char*)base;
  w.kbar = (float*)(p + off); off += align256(nk * s.d * 4);
  if (bounds) {
    w.kbar2 = (float*)(p + off); off += align256(nk * s.d * 4);
    w.h16b = (uint16_t*)(p + off); off += align256(nk * s.d * 2);
  }
  w.h16 = (uint16_t*)(p + off); off += align256(nk * s.d * 2);
  w.kinv = (float*)(p + off); off += align256(nk * 4);
  if (vterm) {
    w.w = (float*)(p + off); off += align256(nk * 4);
  }
  w.bytes = off;
  return w;
}

struct SelectWs {
  int32_t* ranked;
  float* sigma;
  float* sigma_bar;
  uint8_t* trigger;
  size_t bytes;
};

SelectWs select_ws(const bsa_shape& s, int W, void* base) {
  const size_t rows = (size_t)s.B * s.Hq * (s.N / s.tile_q);
  const size_t tiles = (size_t)s.B * (s.N / s.tile_q);
  SelectWs w{};
  size_t off = 0;
  char* p = (char*)base;
  w.ranked = (int32_t*)(p + off); off += align256(rows * W * 4);
  w.sigma = (float*)(p + off); off += align256(rows * 4);
  w.sigma_bar = (float*)(p + off); off += align256(tiles * 4);
  w.trigger = (uint8_t*)(p + off); off += align256(tiles);
  w.bytes = off;
  return w;
}

}  // namespace

namespace bsa {
void set_last_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}
}  // namespace bsa

extern "C" {

const char* bsa_status_string(bsa_status st) {
  switch (st) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported";
    case BSA_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* bsa_last_error(void) { return g_err; }

size_t bsa_score_workspace_bytes(const bsa_shape* s, bsa_score_kind kind) {
  if (check_shape(s) != BSA_OK || !known_kind(kind)) return 0;
  return score_ws(*s, kind, nullptr).bytes;
}

}  // extern "C"

namespace {

// Argument checks shared by bsa_score_ex and bsa_score_select; returns beta in *beta.
bsa_status check_score_args(const bsa_shape* s, bsa_score_kind kind, const bsa_score_params* prm,
                            const void* q, const void* k, const void* v, float* beta) {
  bsa_status st = check_shape(s);
  if (st != BSA_OK) return st;
  if (!known_kind(kind)) return fail(BSA_ERR_INVALID_ARG, "unknown score kind");
  if (!q || !k) return fail(BSA_ERR_INVALID_ARG, "NULL q or k");
  const bool vterm = kind == BSA_SCORE_MEAN_VNORM || kind == BSA_SCORE_MEAN_VLOG;
  if (vterm && !v) return fail(BSA_ERR_INVALID_ARG, "v is NULL for an output-aware score");
  *beta = 0.f;
  if (kind == BSA_SCORE_MEAN_VLOG) {
    if (!prm) return fail(BSA_ERR_INVALID_ARG, "BSA_SCORE_MEAN_VLOG needs params (beta)");
    *beta = prm->beta;
    if (!(*beta >= 0.f) || !(*beta < INFINITY)) return fail(BSA_ERR_INVALID_ARG, "beta must be finite and >= 0");
  }
  if (!aligned16(q) || !aligned16(k) || (v && !aligned16(v)))
    return fail(BSA_ERR_INVALID_ARG, "q/k/v need 16-byte alignment");
  return BSA_OK;
}

int wmode_of(bsa_score_kind kind) {
  return kind == BSA_SCORE_MEAN_VNORM ? 1 : (kind == BSA_SCORE_MEAN_VLOG ? 2 : 0);
}

// Pool (+ value term) and, unless ranked is given with the fused kernel, the scores.
// Launches only; the arguments are checked.
bsa_status run_score(const bsa_shape& s, bsa_score_kind kind, float beta, const void* q, const void* k,
                     const void* v, float* scores, int32_t* dev_status, const ScoreWs& w, cudaStream_t cs) {
  cudaError_t e;
  if (kind == BSA_SCORE_KMINMAX) {
    const bool tc = bsa::score_rank_supported(s);
    e = bsa::launch_pool_bounds(s, k, w.kbar, w.kbar2, tc ? w.h16 : nullptr, w.h16b, w.kinv, cs);
    if (e != cudaSuccess) return cuda_fail(e, "pool (bounds)");
    e = tc ? bsa::launch_score_rank_bounds(s, q, w.h16, w.h16b, w.kinv, scores, dev_status, cs)
           : bsa::launch_score_simt(s, q, w.kbar, w.kbar2, nullptr, 0, scores, cs);
    if (e != cudaSuccess) return cuda_fail(e, tc ? "score (tensor cores)" : "score");
    return BSA_OK;
  }
  const bool vterm = kind == BSA_SCORE_MEAN_VNORM || kind == BSA_SCORE_MEAN_VLOG;
  const bool tc = bsa::score_rank_supported(s);
  e = bsa::launch_pool(s, k, vterm ? v : nullptr, w.kbar, tc ? w.h16 : nullptr, w.kinv, w.w, cs,
                       kind == BSA_SCORE_MEAN_VLOG ? 1 : 0, beta);
  if (e != cudaSuccess) return cuda_fail(e, "pool");
  e = tc ? bsa::launch_score_rank(s, nullptr, q, w.h16, w.kinv, w.w, wmode_of(kind), scores, nullptr, 0,
                                  nullptr, nullptr, 0, dev_status, cs)
         : bsa::launch_score_simt(s, q, w.kbar, nullptr, w.w, wmode_of(kind), scores, cs);
  if (e != cudaSuccess) return cuda_fail(e, tc ? "score (tensor cores)" : "score");
  return BSA_OK;
}

// Gate and kv_idx from the ranked lists and sigma.
bsa_status run_gate_finalize(const bsa_shape& s, const bsa_select_params& p, int W, const SelectWs& w,
                             const float* sg, float* sigma_bar, uint8_t* trigger, float* theta,
                             int32_t* kv_idx, int32_t* kv_cnt, cudaStream_t cs) {
  float* sb = sigma_bar ? sigma_bar : w.sigma_bar;
  uint8_t* tr = trigger ? trigger : w.trigger;
  cudaError_t e = bsa::launch_gate(s, p, sg, sb, tr, theta, cs);
  if (e != cudaSuccess) return cuda_fail(e, "gate");
  e = bsa::launch_finalize(s, p, w.ranked, W, tr, W, kv_idx, kv_cnt, cs);
  if (e != cudaSuccess) return cuda_fail(e, "finalize");
  return BSA_OK;
}

// Workspace of bsa_score_select: the score workspace, the selection workspace, and either
// the row ring of the fused kernel or (for the shapes and kinds it does not take) a scores
// array for the unfused path.
struct ScoreSelectWs {
  ScoreWs sc;
  SelectWs sel;
  float* ring;       // fused: [kScoreRankRingCtas][kScoreRankRing][heads per unit][n_kb]
  float* scores;     // unfused: [B,Hq,n_qt,n_kb]
  size_t bytes;
};

bool fused_kind(bsa_score_kind kind) {
  return kind == BSA_SCORE_MEAN || kind == BSA_SCORE_MEAN_VNORM || kind == BSA_SCORE_MEAN_VLOG;
}

ScoreSelectWs score_select_ws(const bsa_shape& s, bsa_score_kind kind, int W, void* base) {
  ScoreSelectWs w{};
  char* p = (char*)base;
  w.sc = score_ws(s, kind, p);
  size_t off = w.sc.bytes;
  w.sel = select_ws(s, W, p ? p + off : nullptr);
  off += w.sel.bytes;
  const size_t n_kb = (size_t)(s.N / s.block_k);
  if (fused_kind(kind) && bsa::score_rank_fusable(s)) {
    w.ring = (float*)(p + off);
    off += align256((size_t)bsa::kScoreRankRingCtas * bsa::kScoreRankRing *
                    bsa::score_rank_heads_per_unit(s) * n_kb * 4);
  } else {
    w.scores = (float*)(p + off);
    off += align256((size_t)s.B * s.Hq * (s.N / s.tile_q) * n_kb * 4);
  }
  w.bytes = off;
  return w;
}

}  // namespace

extern "C" {

bsa_status bsa_score_ex(const bsa_shape* s, bsa_score_kind kind, const bsa_score_params* prm,
                        const void* q, const void* k, const void* v, float* scores,
                        int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  float beta;
  bsa_status st = check_score_args(s, kind, prm, q, k, v, &beta);
  if (st != BSA_OK) return st;
  if (!scores || !ws) return fail(BSA_ERR_INVALID_ARG, "NULL scores or workspace");
  if ((uintptr_t)ws & 255u) return fail(BSA_ERR_INVALID_ARG, "workspace needs 256-byte alignment");
  ScoreWs w = score_ws(*s, kind, ws);
  if (ws_bytes < w.bytes) return fail(BSA_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", ws_bytes, w.bytes);
  cudaStream_t cs = (cudaStream_t)stream;
  if (dev_status) {
    cudaError_t e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), cs);
    if (e != cudaSuccess) return cuda_fail(e, "clear dev_status");
  }
  st = run_score(*s, kind, beta, q, k, v, scores, dev_status, w, cs);
  return st == BSA_OK ? ok() : st;
}

bsa_status bsa_score(const bsa_shape* s, bsa_score_kind kind, const void* q, const void* k,
                     const void* v, float* scores, int32_t* dev_status, void* ws, size_t ws_bytes,
                     void* stream) {
  if (kind == BSA_SCORE_MEAN_VLOG)
    return fail(BSA_ERR_INVALID_ARG, "BSA_SCORE_MEAN_VLOG needs beta: use bsa_score_ex");
  return bsa_score_ex(s, kind, nullptr, q, k, v, scores, dev_status, ws, ws_bytes, stream);
}

int bsa_kv_idx_width(const bsa_shape* s, const bsa_select_params* p) {
  if (check_shape(s) != BSA_OK || check_params(s, p) != BSA_OK) return -1;
  return bsa::kv_width(s->N, s->tile_q, s->block_k, p->k_first, p->k_last, p->rho);
}

size_t bsa_select_workspace_bytes(const bsa_shape* s, const bsa_select_params* p) {
  if (check_shape(s) != BSA_OK || check_params(s, p) != BSA_OK) return 0;
  int W = bsa::kv_width(s->N, s->tile_q, s->block_k, p->k_first, p->k_last, p->rho);
  return select_ws(*s, W, nullptr).bytes;
}

bsa_status bsa_select(const bsa_shape* s, const bsa_select_params* p, const float* scores,
                      int32_t* kv_idx, int32_t* kv_cnt, float* sigma, float* sigma_bar,
                      uint8_t* trigger, float* theta, int32_t* dev_status, void* ws,
                      size_t ws_bytes, void* stream) {
  bsa_status st = check_shape(s);
  if (st != BSA_OK) return st;
  st = check_params(s, p);
  if (st != BSA_OK) return st;
  if (!scores || !kv_idx || !kv_cnt || !ws)
    return fail(BSA_ERR_INVALID_ARG, "NULL scores, kv_idx, kv_cnt or workspace");
  if ((uintptr_t)ws & 255u) return fail(BSA_ERR_INVALID_ARG, "workspace needs 256-byte alignment");
  const int W = bsa::kv_width(s->N, s->tile_q, s->block_k, p->k_first, p->k_last, p->rho);
  SelectWs w = select_ws(*s, W, ws);
  if (ws_bytes < w.bytes) return fail(BSA_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", ws_bytes, w.bytes);
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e;
  if (dev_status) {
    e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), cs);
    if (e != cudaSuccess) return cuda_fail(e, "clear dev_status");
  }
  float* sg = sigma ? sigma : w.sigma;
  e = bsa::launch_select_rank(*s, *p, scores, W, w.ranked, sg, dev_status, cs);
  if (e != cudaSuccess) return cuda_fail(e, "select_rank");
  st = run_gate_finalize(*s, *p, W, w, sg, sigma_bar, trigger, theta, kv_idx, kv_cnt, cs);
  return st == BSA_OK ? ok() : st;
}

size_t bsa_score_select_workspace_bytes(const bsa_shape* s, bsa_score_kind kind,
                                        const bsa_select_params* p) {
  if (check_shape(s) != BSA_OK || !known_kind(kind) || check_params(s, p) != BSA_OK) return 0;
  const int W = bsa::kv_width(s->N, s->tile_q, s->block_k, p->k_first, p->k_last, p->rho);
  return score_select_ws(*s, kind, W, nullptr).bytes;
}

bsa_status bsa_score_select(const bsa_shape* s, bsa_score_kind kind, const bsa_score_params* prm,
                            const bsa_select_params* p, const void* q, const void* k, const void* v,
                            float* scores, int32_t* kv_idx, int32_t* kv_cnt, float* sigma,
                            float* sigma_bar, uint8_t* trigger, float* theta, int32_t* dev_status,
                            void* ws, size_t ws_bytes, void* stream) {
  float beta;
  bsa_status st = check_score_args(s, kind, prm, q, k, v, &beta);
  if (st != BSA_OK) return st;
  st = check_params(s, p);
  if (st != BSA_OK) return st;
  if (!kv_idx || !kv_cnt || !ws) return fail(BSA_ERR_INVALID_ARG, "NULL kv_idx, kv_cnt or workspace");
  if ((uintptr_t)ws & 255u) return fail(BSA_ERR_INVALID_ARG, "workspace needs 256-byte alignment");
  const int W = bsa::kv_width(s->N, s->tile_q, s->block_k, p->k_first, p->k_last, p->rho);
  ScoreSelectWs w = score_select_ws(*s, kind, W, ws);
  if (ws_bytes < w.bytes) return fail(BSA_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", ws_bytes, w.bytes);
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e;
  if (dev_status) {
    e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), cs);
    if (e != cudaSuccess) return cuda_fail(e, "clear dev_status");
  }
  float* sg = sigma ? sigma : w.sel.sigma;
  if (w.ring) {
    // fused: scores are ranked inside the score kernel and written only when asked for
    const bool vterm = kind == BSA_SCORE_MEAN_VNORM || kind == BSA_SCORE_MEAN_VLOG;
    e = bsa::launch_pool(*s, k, vterm ? v : nullptr, w.sc.kbar, w.sc.h16, w.sc.kinv, w.sc.w, cs,
                         kind == BSA_SCORE_MEAN_VLOG ? 1 : 0, beta);
    if (e != cudaSuccess) return cuda_fail(e, "pool");
    e = bsa::launch_score_rank(*s, p, q, w.sc.h16, w.sc.kinv, w.sc.w, wmode_of(kind), scores, w.ring,
                               bsa::kScoreRankRingCtas, w.sel.ranked, sg, W, dev_status, cs);
    if (e != cudaSuccess) return cuda_fail(e, "score+rank (tensor cores)");
  } else {
    float* sc = scores ? scores : w.scores;
    st = run_score(*s, kind, beta, q, k, v, sc, dev_status, w.sc, cs);
    if (st != BSA_OK) return st;
    e = bsa::launch_select_rank(*s, *p, sc, W, w.sel.ranked, sg, dev_status, cs);
    if (e != cudaSuccess) return cuda_fail(e, "select_rank");
  }
  st = run_gate_finalize(*s, *p, W, w.sel, sg, sigma_bar, trigger, theta, kv_idx, kv_cnt, cs);
  return st == BSA_OK ? ok() : st;
}

bsa_status bsa_attend(const bsa_shape* s, const void* q, const void* k, const void* v,
                      const int32_t* kv_idx, const int32_t* kv_cnt, int W, float scale, void* out,
                      float* lse, int32_t* dev_status, void* stream) {
  bsa_status st = check_shape(s);
  if (st != BSA_OK) return st;
  if (!q || !k || !v || !kv_idx || !kv_cnt || !out || !dev_status)
    return fail(BSA_ERR_INVALID_ARG, "NULL q, k, v, kv_idx, kv_cnt, out or dev_status");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(BSA_ERR_INVALID_ARG, "q/k/v/out need 16-byte alignment");
  if (W < 1 || W > s->N / s->block_k) return fail(BSA_ERR_INVALID_ARG, "W out of range");
  if (!(scale > 0.0f)) return fail(BSA_ERR_INVALID_ARG, "softmax_scale must be > 0");
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), cs);
  if (e != cudaSuccess) return cuda_fail(e, "clear dev_status");
  // tensor-core path for its shapes (bf16, d 128, blocks 64, tiles 128); CUDA cores otherwise
  if (attend_on_tensor_cores(*s, W)) {
    e = bsa::launch_attend_tc(*s, q, k, v, kv_idx, kv_cnt, W, scale, out, lse, dev_status, cs);
    if (e != cudaSuccess) return cuda_fail(e, "attend (tensor cores)");
  } else {
    e = bsa::launch_attend_simt(*s, q, k, v, kv_idx, kv_cnt, W, scale, out, lse, dev_status, cs);
    if (e != cudaSuccess) return cuda_fail(e, "attend");
  }
  return ok();
}

// ---- vertical-slash attention ----------------------------------------------------------

static int vs_list_width(const bsa_shape& s, int Wv, int Ws) {
  const long long w = (long long)Wv + 3ll * Ws;        // a slash diagonal crosses <= 3 blocks per tile
  const int n_kb = s.N / 64;
  return (int)(w < n_kb ? w : n_kb);
}

struct VsWs {
  unsigned long long* vbits;
  unsigned long long* sbits;
  int32_t* lists;
  int32_t* counts;
  size_t bytes;
};

static VsWs vs_ws(const bsa_shape& s, int Wl, void* base) {
  const size_t bh = (size_t)s.B * s.Hq;
  const size_t words = (size_t)s.N / 64 + 1;
  const size_t rows = bh * (s.N / s.tile_q);
  VsWs w{};
  size_t off = 0;
  char* p = (char*)base;
  w.vbits = (unsigned long long*)(p + off); off += align256(bh * words * 8);
  w.sbits = (unsigned long long*)(p + off); off += align256(bh * words * 8);
  w.lists = (int32_t*)(p + off); off += align256(rows * Wl * 4);
  w.counts = (int32_t*)(p + off); off += align256(rows * 4);
  w.bytes = off;
  return w;
}

static bsa_status check_vs(const bsa_shape* s, int Wv, int Ws) {
  bsa_status st = check_shape(s);
  if (st != BSA_OK) return st;
  if (!bsa::attend_tc_supported(*s) || (long long)s->B * s->Hq * s->N >= (1ll << 31))
    return fail(BSA_ERR_UNSUPPORTED, "vertical-slash attention takes bf16, d 128, key blocks of 64, tiles of 128");
  if (Wv < 1 || Ws < 1) return fail(BSA_ERR_INVALID_ARG, "Wv and Ws must be >= 1");
  if (vs_list_width(*s, Wv, Ws) > 1024)
    return fail(BSA_ERR_UNSUPPORTED, "min(n_kb, Wv + 3*Ws) must be <= 1024");
  return BSA_OK;
}

size_t bsa_attend_vs_workspace_bytes(const bsa_shape* s, int Wv, int Ws) {
  if (check_vs(s, Wv, Ws) != BSA_OK) return 0;
  return vs_ws(*s, vs_list_width(*s, Wv, Ws), nullptr).bytes;
}

bsa_status bsa_attend_vs(const bsa_shape* s, const void* q, const void* k, const void* v,
                         const int32_t* v_idx, const int32_t* v_cnt, int Wv, const int32_t* s_off,
                         const int32_t* s_cnt, int Ws, float scale, void* out, float* lse,
                         int32_t* dev_status, void* ws, size_t ws_bytes, void* stream) {
  bsa_status st = check_vs(s, Wv, Ws);
  if (st != BSA_OK) return st;
  if (!q || !k || !v || !v_idx || !v_cnt || !s_off || !s_cnt || !out || !dev_status || !ws)
    return fail(BSA_ERR_INVALID_ARG, "NULL input, index list, count, out, dev_status or workspace");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || ((uintptr_t)ws & 255u))
    return fail(BSA_ERR_INVALID_ARG, "q/k/v/out need 16-byte and workspace 256-byte alignment");
  if (!(scale > 0.0f)) return fail(BSA_ERR_INVALID_ARG, "softmax_scale must be > 0");
  const int Wl = vs_list_width(*s, Wv, Ws);
  VsWs w = vs_ws(*s, Wl, ws);
  if (ws_bytes < w.bytes) return fail(BSA_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", ws_bytes, w.bytes);
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), cs);
  if (e != cudaSuccess) return cuda_fail(e, "clear dev_status");
  e = bsa::launch_vs_prep(*s, v_idx, v_cnt, Wv, s_off, s_cnt, Ws, Wl, w.vbits, w.sbits, w.lists, w.counts,
                          dev_status, cs);
  if (e != cudaSuccess) return cuda_fail(e, "vertical-slash lists");
  e = bsa::launch_attend_tc_vs(*s, q, k, v, w.lists, w.counts, Wl, scale, out, lse, dev_status, w.vbits,
                               w.sbits, cs);
  if (e != cudaSuccess) return cuda_fail(e, "vertical-slash attend");
  return ok();
}

static bsa_status check_decode(const bsa_decode_shape* s, const bsa_decode_params* p, const void* q,
                               const void* kc, const void* vc, float scale, const void* out,
                               const int32_t* blocks_used, const int32_t* dev_status) {
  if (!s || !p) return fail(BSA_ERR_INVALID_ARG, "shape or params is NULL");
  if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->L < 1 || s->Hq % s->Hkv)
    return fail(BSA_ERR_INVALID_ARG, "bad B/Hq/Hkv/L");
  const int G = s->Hq / s->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return fail(BSA_ERR_UNSUPPORTED, "Hq/Hkv must be 1, 2, 4 or 8");
  if (s->d != 64 && s->d != 128) return fail(BSA_ERR_UNSUPPORTED, "d must be 64 or 128");
  if (s->block_kv != 64 && s->block_kv != 128) return fail(BSA_ERR_UNSUPPORTED, "block_kv must be 64 or 128");
  if (s->L % s->block_kv) return fail(BSA_ERR_INVALID_ARG, "L must be a multiple of block_kv");
  if ((long long)s->B * s->Hkv * s->L >= (1ll << 31))
    return fail(BSA_ERR_UNSUPPORTED, "B * Hkv * L must be below 2^31 (cache rows are int32 coordinates)");
  if (s->dtype != BSA_BF16) return fail(BSA_ERR_UNSUPPORTED, "decode takes bf16 only");
  if (p->patience < 1) return fail(BSA_ERR_INVALID_ARG, "patience must be >= 1");
  if (p->n_probe < 1 || p->n_probe > bsa::kMaxProbe || !p->probe_dims)
    return fail(BSA_ERR_INVALID_ARG, "n_probe must be 1..%d with probe_dims given", bsa::kMaxProbe);
  for (int i = 0; i < p->n_probe; ++i)
    if (p->probe_dims[i] < 0 || p->probe_dims[i] >= s->d)
      return fail(BSA_ERR_INVALID_ARG, "probe_dims[%d] out of range", i);
  if (!(p->tau >= 0.0f) || !(p->phi >= 0.0f)) return fail(BSA_ERR_INVALID_ARG, "tau and phi must be >= 0");
  if (!q || !kc || !vc || !out || !blocks_used || !dev_status)
    return fail(BSA_ERR_INVALID_ARG, "NULL q, caches, out, blocks_used or dev_status");
  if (!aligned16(q) || !aligned16(kc) || !aligned16(vc) || !aligned16(out))
    return fail(BSA_ERR_INVALID_ARG, "q/caches/out need 16-byte alignment");
  if (!(scale > 0.0f)) return fail(BSA_ERR_INVALID_ARG, "softmax_scale must be > 0");
  return BSA_OK;
}

bsa_status bsa_decode(const bsa_decode_shape* s, const bsa_decode_params* p, const void* q,
                      const void* kc, const void* vc, float scale, void* out, int32_t* blocks_used,
                      float* probe_trace, int32_t* dev_status, void* stream) {
  bsa_status st = check_decode(s, p, q, kc, vc, scale, out, blocks_used, dev_status);
  if (st != BSA_OK) return st;
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), cs);
  if (e != cudaSuccess) return cuda_fail(e, "clear dev_status");
  e = bsa::launch_decode(*s, *p, q, kc, vc, scale, out, blocks_used, probe_trace, dev_status, cs);
  if (e != cudaSuccess) return cuda_fail(e, "decode");
  return ok();
}

bsa_status bsa_decode_list(const bsa_decode_shape* s, const bsa_decode_params* p, const void* q,
                           const void* kc, const void* vc, const int32_t* block_list,
                           const int32_t* list_cnt, int list_width, float scale, void* out,
                           int32_t* blocks_used, float* probe_trace, int32_t* dev_status,
                           void* stream) {
  bsa_status st = check_decode(s, p, q, kc, vc, scale, out, blocks_used, dev_status);
  if (st != BSA_OK) return st;
  if (!block_list || !list_cnt) return fail(BSA_ERR_INVALID_ARG, "NULL block_list or list_cnt");
  if (list_width < 1 || list_width > bsa::kMaxDecodeList)
    return fail(BSA_ERR_UNSUPPORTED, "list_width must be 1..%d", bsa::kMaxDecodeList);
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(dev_status, 0, sizeof(int32_t), cs);
  if (e != cudaSuccess) return cuda_fail(e, "clear dev_status");
  e = bsa::launch_decode(*s, *p, q, kc, vc, scale, out, blocks_used, probe_trace, dev_status, cs,
                         block_list, list_cnt, list_width);
  if (e != cudaSuccess) return cuda_fail(e, "decode_list");
  return ok();
}

// ---- which kernels a call runs ----------------------------------------------------------

int bsa_attend_path(const bsa_shape* s, int W) {
  if (check_shape(s) != BSA_OK || W < 1 || W > s->N / s->block_k) return -1;
  return attend_on_tensor_cores(*s, W) ? BSA_PATH_TENSOR_CORES : BSA_PATH_CUDA_CORES;
}

int bsa_score_path(const bsa_shape* s, bsa_score_kind kind) {
  if (check_shape(s) != BSA_OK || !known_kind(kind)) return -1;
  const bool tc = bsa::score_rank_supported(*s);
  return tc ? BSA_PATH_TENSOR_CORES : BSA_PATH_CUDA_CORES;
}

int bsa_decode_path(const bsa_decode_shape* s) {
  // the shape checks of bsa_decode (check_decode), without the pointers and parameters
  if (!s || s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->L < 1 || s->Hq % s->Hkv) return -1;
  const int G = s->Hq / s->Hkv;
  if ((G != 1 && G != 2 && G != 4 && G != 8) || (s->d != 64 && s->d != 128) ||
      (s->block_kv != 64 && s->block_kv != 128) || s->L % s->block_kv ||
      (long long)s->B * s->Hkv * s->L >= (1ll << 31) || s->dtype != BSA_BF16)
    return -1;
  return bsa::decode_mma_supported(*s) ? BSA_PATH_TENSOR_CORES : BSA_PATH_CUDA_CORES;
}

}  // extern "C"
