// Internal launchers behind the C ABI (host side). Each returns cudaError_t of the launch.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bsa.h"

namespace bsa {

// Pooled keys (+ value-block term). kbar fp32 [B,Hkv,n_kb,d]; kbar16 fp16 [B,Hkv,n_kb,d]
// scaled per block by 2^r and kinv [B,Hkv,n_kb] = 2^-r (both may be null); wnorm
// [B,Hkv,n_kb] (only when v != null): ||Vbar|| (wlog 0) or beta * max(0, ln ||Vbar||^2)
// (wlog 1).
cudaError_t launch_pool(const bsa_shape& s, const void* k, const void* v, float* kbar,
                        uint16_t* kbar16, float* kinv, float* wnorm, cudaStream_t st,
                        int wlog = 0, float beta = 0.f);

// Per-coordinate key bounds: kmin, kmax fp32 [B,Hkv,n_kb,d]; for the tensor-core score
// (pointers may be null) mid = (kmin+kmax)/2 and rad = (kmax-kmin)/2 as fp16 scaled by
// 2^r per block, and kinv [B,Hkv,n_kb] = 2^-r.
cudaError_t launch_pool_bounds(const bsa_shape& s, const void* k, float* kmin, float* kmax,
                               uint16_t* mid16, uint16_t* rad16, float* kinv, cudaStream_t st);

// Block scores on CUDA cores (fp32). kbar2 != null selects the bounds backbone (kbar =
// kmin, kbar2 = kmax). wmode: 0 none, 1 times wnorm, 2 plus wnorm.
cudaError_t launch_score_simt(const bsa_shape& s, const void* q, const float* kbar,
                              const float* kbar2, const float* wnorm, int wmode, float* scores,
                              cudaStream_t st);

// Mean-pooled block scores on tcgen05 (fp16 operands with power-of-two scales), persistent,
// optionally fused with the ranking of the selection. kbar16/kinv from launch_pool.
// ranked == null: scores only (scores required). ranked != null: also the top-M lists
// [B*Hq*n_qt][W] and sigma; scores may then be null, and the rows go through
// ring [ring_ctas][kScoreRankRing][heads per unit][n_kb] instead (the grid is capped at
// ring_ctas).
bool score_rank_supported(const bsa_shape& s);
// The K-min/K-max backbone in the same persistent kernel (one head per unit, two passes per
// chunk: mid against Q, rad against |Q|); mid16, rad16, kinv from launch_pool_bounds.
cudaError_t launch_score_rank_bounds(const bsa_shape& s, const void* q, const uint16_t* mid16,
                                     const uint16_t* rad16, const float* kinv, float* scores,
                                     int32_t* dev_status, cudaStream_t st);
bool score_rank_fusable(const bsa_shape& s);          // the ranking too
int score_rank_heads_per_unit(const bsa_shape& s);
constexpr int kScoreRankRingCtas = 256;
constexpr int kScoreRankRing = 8;
cudaError_t launch_score_rank(const bsa_shape& s, const bsa_select_params* p, const void* q,
                              const uint16_t* kbar16, const float* kinv, const float* wnorm, int wmode,
                              float* scores, float* ring, int ring_ctas, int32_t* ranked, float* sigma,
                              int W, int32_t* dev_status, cudaStream_t st);

// Selection: ranked candidate lists + sigma, then the gate, then kv_idx.
cudaError_t launch_select_rank(const bsa_shape& s, const bsa_select_params& p, const float* scores,
                               int R, int32_t* ranked, float* sigma, int32_t* dev_status,
                               cudaStream_t st);
cudaError_t launch_gate(const bsa_shape& s, const bsa_select_params& p, const float* sigma,
                        float* sigma_bar, uint8_t* trigger, float* theta, cudaStream_t st);
cudaError_t launch_finalize(const bsa_shape& s, const bsa_select_params& p, const int32_t* ranked,
                            int R, const uint8_t* trigger, int W, int32_t* kv_idx, int32_t* kv_cnt,
                            cudaStream_t st);

// Sparse attend on CUDA cores (fp32 math; bf16 or fp32 I/O).
cudaError_t launch_attend_simt(const bsa_shape& s, const void* q, const void* k, const void* v,
                               const int32_t* kv_idx, const int32_t* kv_cnt, int W, float scale,
                               void* out, float* lse, int32_t* dev_status, cudaStream_t st);

// Sparse attend on tcgen05 tensor cores (bf16, d = 128, block_k = 64, tile_q = 128).
bool attend_tc_supported(const bsa_shape& s);

// Vertical-slash: bitmaps V and S per (b, h) (N/64+1 words each) and the per-tile key-block
// lists (width Wl, ascending, -1 padded) with their counts; then the masked tensor-core attend.
cudaError_t launch_vs_prep(const bsa_shape& s, const int32_t* v_idx, const int32_t* v_cnt, int Wv,
                           const int32_t* s_off, const int32_t* s_cnt, int Ws, int Wl,
                           unsigned long long* vbits, unsigned long long* sbits, int32_t* lists,
                           int32_t* counts, int32_t* dev_status, cudaStream_t st);
cudaError_t launch_attend_tc_vs(const bsa_shape& s, const void* q, const void* k, const void* v,
                                const int32_t* lists, const int32_t* counts, int W, float scale,
                                void* out, float* lse, int32_t* dev_status,
                                const unsigned long long* vbits, const unsigned long long* sbits,
                                cudaStream_t st);
cudaError_t launch_attend_tc(const bsa_shape& s, const void* q, const void* k, const void* v,
                             const int32_t* kv_idx, const int32_t* kv_cnt, int W, float scale,
                             void* out, float* lse, int32_t* dev_status, cudaStream_t st);

// Limits of this build (checked on the host).
constexpr int kMaxCandidates = 8192;     // n_kb limit of the selection (the range its tests cover)
constexpr int kMaxGateTiles = 16384;     // B * n_qt for the single-CTA gate sort
constexpr int kMaxProbe = 64;
constexpr int kMaxGroup = 8;             // Hq / Hkv in decode
constexpr int kMaxDecodeList = 4096;     // visit-list width in decode over a block list

// Decode kernel arguments (passed by value).
struct DecodeArgs {
  int L, block_kv, Hq, Hkv;
  float scale_log2;
  float tau, phi;
  int patience, enable, n_probe;
  int dims[kMaxProbe];
  // decode over a block list: blist [B, Hkv, list_w] (visit order), bcnt [B, Hkv];
  // blist == nullptr streams blocks 0, 1, ... in order
  const int32_t* blist;
  const int32_t* bcnt;
  int list_w;
};

// Decode with run-time termination on warp-level tensor-core MMAs (mma.sync; bf16, d 128,
// KV blocks of 128, Hq/Hkv in {1, 2, 4, 8}).
bool decode_mma_supported(const bsa_decode_shape& s);
cudaError_t launch_decode_mma(const bsa_decode_shape& s, const DecodeArgs& a, const void* q,
                              const void* kc, const void* vc, void* out, int32_t* blocks_used,
                              float* probe_trace, int32_t* dev_status, cudaStream_t st);

// Decode with run-time termination (dispatches to the tensor-core kernel where it applies).
cudaError_t launch_decode(const bsa_decode_shape& s, const bsa_decode_params& p, const void* q,
                          const void* kc, const void* vc, float scale, void* out,
                          int32_t* blocks_used, float* probe_trace, int32_t* dev_status,
                          cudaStream_t st, const int32_t* block_list = nullptr,
                          const int32_t* list_cnt = nullptr, int list_w = 0);

// Sets the text bsa_last_error() returns on this thread.
void set_last_error(const char* fmt, ...);

}  // namespace bsa
