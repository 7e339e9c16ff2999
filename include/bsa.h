/*
 * bsa.h -- C ABI of libbsa.so: block-sparse causal attention on NVIDIA B200 (sm_100a).
 *
 * Pages the operations follow (cited by title and section):
 *   [UGS]  "Resumo Técnico: Seleção com Portão de Incerteza para Atenção de
 *          Esparsidade em Blocos", Metodologia steps 1-5.
 *   [Stem] "Stem: Rethinking Causal Information Flow in Sparse Attention",
 *          Resumo técnico, 2. Metodologia A (TPD), B (OAM), Implementação.
 *   [ART]  "Resumo Técnico: ART (Attention Run-time Termination)", 2. Metodologia 2.1-2.4.
 *   [VSP]  "VSPrefill: Vertical-Slash Sparse Attention with Lightweight Indexing for
 *          Long-Context Prefilling", 2. Metodologia A (vertical-slash pattern), B.3 (fused kernel).
 *
 * The problem as those pages frame it: block scores -> per-tile top-k list
 * kv_idx -> sparse attention that streams only the listed blocks ([UGS] steps
 * 2 and 5); and for decode: stream KV blocks in order and stop once the
 * partial output is stable ([ART] 2.2, 2.3).
 *
 * Conventions shared by every call
 *   Layout     Q [B,Hq,N,d], K and V [B,Hkv,N,d], O like Q; contiguous, d innermost.
 *              Query head h reads KV head h / (Hq/Hkv).
 *   Tiles      query tile t = rows [t*tile_q, (t+1)*tile_q); key block j = keys
 *              [j*block_k, (j+1)*block_k); n_qt = N/tile_q, n_kb = N/block_k.
 *              Causal: query i sees keys 0..i. J_t = ((t+1)*tile_q-1)/block_k is
 *              the last block tile t can see; blocks (t*tile_q)/block_k .. J_t
 *              intersect the tile's own rows and are always kept ("forced").
 *   Memory     Every tensor argument is a DEVICE pointer owned by the caller,
 *              unless a comment says "host". The library never allocates or
 *              frees; workspace is caller-provided and sized by the *_bytes calls.
 *   Streams    `stream` is a cudaStream_t (NULL = legacy default stream). All
 *              compute calls only enqueue work and return; results are ready
 *              after the stream is synchronised.
 *   Errors     Argument errors are detected on the host before anything is
 *              enqueued and return BSA_ERR_INVALID_ARG / BSA_ERR_UNSUPPORTED;
 *              launch failures return BSA_ERR_CUDA. bsa_last_error() gives a
 *              one-line reason (per thread). Problems only the device can see
 *              (an out-of-range kv_idx entry, a non-finite candidate score, a
 *              wait that ran out) are OR-ed into *dev_status as BSA_DEV_* bits;
 *              the call clears *dev_status first, the offending work is
 *              skipped, and the kernel never traps.
 *   Precision  bf16 inputs, fp32 accumulation and softmax; BSA_F32 inputs run
 *              an fp32 CUDA-core path, and so do a few bf16 shapes (see the
 *              bsa_*_path queries below, which report the choice).
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, workspace too small, ... */
  BSA_ERR_UNSUPPORTED = 2,   /* valid but outside what this build implements */
  BSA_ERR_CUDA = 3           /* a CUDA launch or runtime call failed */
} bsa_status;

/* Bits OR-ed into *dev_status by the device. */
enum {
  BSA_DEV_OK = 0,
  BSA_DEV_BAD_INDEX = 1,     /* kv_idx entry >= n_kb, > J_t, or a count > W */
  BSA_DEV_TIMEOUT = 2,       /* a bounded wait on an mbarrier ran out */
  BSA_DEV_BAD_SCORE = 4      /* a candidate block score was NaN or infinite */
};

typedef enum { BSA_BF16 = 0, BSA_F32 = 1 } bsa_dtype;

/* Block score backbone.
 *   BSA_SCORE_MEAN        s(t,j) = max over the tile's rows i of q_i . mean(K block j)
 *                         ([UGS] steps 1-2: mean-pooled keys, tile max over rows).
 *   BSA_SCORE_MEAN_VNORM  the same max times || mean(V block j) ||_2, an output-aware
 *                         weighting of the block (motivated by [Stem] 2.B: value
 *                         magnitude enters the selection metric).
 *   BSA_SCORE_MEAN_VLOG   the same max plus beta * max(0, ln || mean(V block j) ||^2):
 *                         [Stem] 2.B's additive Output-Aware Metric at block level, the
 *                         block's mean value vector standing for V_j (bsa_score_ex only,
 *                         beta from bsa_score_params).
 *   BSA_SCORE_KMINMAX     s(t,j) = max over the tile's rows i of
 *                         sum_c max(q_ic kmin_jc, q_ic kmax_jc), kmin/kmax the per-
 *                         coordinate minimum/maximum of block j's keys: the K-min/K-max
 *                         upper-bound backbone named in [UGS] Metodologia step 1. */
typedef enum {
  BSA_SCORE_MEAN = 0,
  BSA_SCORE_MEAN_VNORM = 1,
  BSA_SCORE_MEAN_VLOG = 2,
  BSA_SCORE_KMINMAX = 3
} bsa_score_kind;

/* Extra score parameters (bsa_score_ex). beta: weight of the value term of
 * BSA_SCORE_MEAN_VLOG (in the units of the unscaled q . k). */
typedef struct {
  float beta;
} bsa_score_params;

/* Prefill problem. d in {64,128}; block_k, tile_q in {64,128}; N a multiple of both. */
typedef struct {
  int B, Hq, Hkv, N, d, block_k, tile_q;
  bsa_dtype dtype;
} bsa_shape;

/* Selection parameters.
 *   k_first, k_last  budget in blocks, counting the forced blocks. Equal = fixed
 *                    top-k ([UGS] step 2). Otherwise the Token Position-Decay budget
 *                    of [Stem] 2.A, read as the linear decay
 *                    k_t = k_first - floor((k_first-k_last)*t/(n_qt-1)).
 *                    Requires 1 <= k_last <= k_first. Every budget is capped at the
 *                    J_t+1 blocks the tile can see and never drops the forced blocks.
 *   rho              expansion factor for triggered tiles: top-rho*k instead of
 *                    top-k ([UGS] step 5). rho = 1 disables the gate.
 *   gate_quantile    q in [0,1]: theta = linear-interpolation empirical q-quantile of
 *                    the head-mean sigma over the cut tiles of this call (one call =
 *                    one layer, [UGS] step 4). A negative value selects the fixed
 *                    gate_threshold instead.
 *   gate_threshold   fixed theta when gate_quantile < 0. */
typedef struct {
  int k_first, k_last;
  int rho;
  float gate_quantile;
  float gate_threshold;
} bsa_select_params;

/* Decode problem: one query token per sequence, KV cache of length L.
 * d in {64,128}; block_kv in {64,128}; L a multiple of block_kv; Hq/Hkv in {1,2,4,8};
 * B*Hkv*L < 2^31. */
typedef struct {
  int B, Hq, Hkv, L, d, block_kv;
  bsa_dtype dtype;           /* BSA_BF16 only */
} bsa_decode_shape;

/* Run-time termination ([ART] 2.2-2.4).
 *   tau, phi     thresholds: block t >= 1 is stable iff |‖x_t‖-‖x_{t-1}‖| < tau and
 *                1 - cos(x_t, x_{t-1}) < phi (1 when a norm is 0), computed in fp64
 *                on the fp32 probe values: exact products, each sum over the
 *                coordinates in one fixed pairwise order (coordinate i with i + 32,
 *                zero where absent, then values 16, 8, 4, 2, 1 apart).
 *   patience     stop after `patience` consecutive stable blocks (>= 1) ([ART] 2.3).
 *   enable       0 = never stop (probes are still recorded when asked for).
 *   n_probe      number of probe coordinates (1..64).
 *   probe_dims   HOST array of n_probe coordinates in [0,d): the probe x^(t) is the
 *                normalised partial output O^(t) of the KV group's first query head
 *                at these coordinates ([ART] 2.2 names a register fragment of the
 *                leading thread; this build fixes a layout-free coordinate set). */
typedef struct {
  float tau, phi;
  int patience;
  int enable;
  int n_probe;
  const int* probe_dims;
} bsa_decode_params;

/* ---- scoring ([UGS] steps 1-2; [Stem] 2.B, Implementação) ------------------------ */

/* Workspace bytes bsa_score needs (pooled keys and the value-block norms). */
size_t bsa_score_workspace_bytes(const bsa_shape* shape, bsa_score_kind kind);

/* scores [B,Hq,n_qt,n_kb] fp32: s(t,j) for j <= J_t, -inf for j > J_t.
 * No 1/sqrt(d) factor (a common positive factor changes neither the ranking nor sigma;
 * for BSA_SCORE_MEAN_VLOG the caller's beta carries the relative weight).
 * The tile max runs over all tile_q rows, unmasked.
 * q, k: inputs of `shape->dtype`; v is read only for the output-aware kinds (VNORM, VLOG;
 * else may be NULL).
 * dev_status: device int32 or NULL (BSA_DEV_TIMEOUT if a bounded wait ran out).
 * bsa_score takes every kind but BSA_SCORE_MEAN_VLOG (which needs beta: INVALID_ARG).
 * Precision: bf16 inputs with d = 128 and query tiles of 128 score the mean-pooled
 * kinds on tensor cores with fp16 operands: each query tile and each pooled-key block
 * is scaled by a power of two (exact) so that its largest magnitude lands in
 * [2^14, 2^15); the pooled keys are then rounded to fp16 (relative 2^-12), the query
 * values convert exactly unless they lie more than 2^-24 below the tile's largest, and
 * the products accumulate in fp32. BSA_SCORE_KMINMAX on tensor cores carries the box
 * centre and half-width as bf16 hi/lo pairs (about 2^-17 relative). */
bsa_status bsa_score(const bsa_shape* shape, bsa_score_kind kind,
                     const void* q, const void* k, const void* v,
                     float* scores, int32_t* dev_status, void* workspace, size_t workspace_bytes,
                     void* stream);

/* bsa_score with parameters: params may be NULL except for BSA_SCORE_MEAN_VLOG, which
 * needs a finite beta >= 0. */
bsa_status bsa_score_ex(const bsa_shape* shape, bsa_score_kind kind, const bsa_score_params* params,
                        const void* q, const void* k, const void* v,
                        float* scores, int32_t* dev_status, void* workspace, size_t workspace_bytes,
                        void* stream);

/* ---- selection ([UGS] steps 2-5; [Stem] 2.A) -------------------------------------- */

/* kv_idx row width W = min(n_kb, max(rho*max(k_first,k_last), forced blocks per tile)).
 * Depends only on the parameters, never on data ([UGS] step 5: uniform dispatch shape).
 * Returns -1 on invalid arguments. */
int bsa_kv_idx_width(const bsa_shape* shape, const bsa_select_params* params);

size_t bsa_select_workspace_bytes(const bsa_shape* shape, const bsa_select_params* params);

/* From scores (as written by bsa_score, same stream) to kv_idx.
 *   kv_idx   [B,Hq,n_qt,W] int32: the forced blocks plus the best m_t (or, for a
 *            triggered tile, M_t) candidate blocks, ranked by (score desc, index asc),
 *            written in ascending order and padded with -1 ([UGS] steps 2, 5).
 *   kv_cnt   [B,Hq,n_qt] int32: number of valid entries.
 *   sigma    [B,Hq,n_qt] fp32 or NULL: (s_(m-1)-s_(m))/(s_(0)-s_(m)) over the ranked
 *            candidates with m = m_t, fp32 ([UGS] step 3); 1 for a tile with no cut.
 *   sigma_bar[B,n_qt] fp32 or NULL: fp32 head sum in head order, / Hq ([UGS] step 4).
 *   trigger  [B,n_qt] uint8 or NULL: cut tile and sigma_bar < theta (strict).
 *   theta    device fp32 scalar or NULL (NaN when undefined).
 *   dev_status device int32 or NULL: BSA_DEV_BAD_SCORE on a non-finite candidate.
 * Limits: n_kb <= 8192 and B * n_qt <= 16384 (the gate sorts one layer's tiles in one
 * CTA); beyond them BSA_ERR_UNSUPPORTED and nothing is launched. */
bsa_status bsa_select(const bsa_shape* shape, const bsa_select_params* params,
                      const float* scores, int32_t* kv_idx, int32_t* kv_cnt,
                      float* sigma, float* sigma_bar, uint8_t* trigger, float* theta,
                      int32_t* dev_status, void* workspace, size_t workspace_bytes,
                      void* stream);

/* ---- scoring and selection in one call ([UGS] steps 1-5; [Stem] 2.A, 2.B) -------- */

/* Workspace bytes bsa_score_select needs (0 on invalid arguments). */
size_t bsa_score_select_workspace_bytes(const bsa_shape* shape, bsa_score_kind kind,
                                        const bsa_select_params* params);

/* bsa_score followed by bsa_select, with the same arguments and results, in one call:
 * the pages' framing of scores -> per-tile top-k -> kv_idx ([UGS] steps 2-5; its
 * Contribuições 3 runs selection and expansion in one fused code path).
 *   scores   [B,Hq,n_qt,n_kb] fp32 or NULL. NULL: the scores are not written out.
 *   kv_idx, kv_cnt, sigma, sigma_bar, trigger, theta, dev_status: as bsa_select
 *            (dev_status also collects bsa_score's device bits).
 *   params   score parameters as bsa_score_ex (NULL except for BSA_SCORE_MEAN_VLOG).
 * For bf16 inputs with d = 128 and query tiles of 128, and the mean-pooled kinds
 * (BSA_SCORE_MEAN, _VNORM, _VLOG), the ranking runs inside the tensor-core score
 * kernel: each (batch, head, tile) row is ranked by a warp of the score kernel
 * right after it is complete, from L2, and the scores never make a round trip
 * through DRAM unless asked for. Other shapes and BSA_SCORE_KMINMAX run the two
 * calls one after the other (the scores then pass through the workspace when the
 * scores pointer is NULL). Results are identical either way given the same scores.
 * Workspace: bsa_score_select_workspace_bytes() bytes, 256-byte aligned. Errors,
 * limits and stream semantics as bsa_score and bsa_select. */
bsa_status bsa_score_select(const bsa_shape* shape, bsa_score_kind kind,
                            const bsa_score_params* score_params, const bsa_select_params* params,
                            const void* q, const void* k, const void* v, float* scores,
                            int32_t* kv_idx, int32_t* kv_cnt, float* sigma, float* sigma_bar,
                            uint8_t* trigger, float* theta, int32_t* dev_status, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ---- sparse attend ([UGS] step 5; [Stem] Implementação) ------------------------- */

/* O_i = sum over keys j in the listed blocks with j <= i of softmax(scale * q_i.k_j) v_j.
 *   kv_idx/kv_cnt as written by bsa_select (entries beyond kv_cnt ignored; order free).
 *   out  like Q, of `shape->dtype`.  lse [B,Hq,N] fp32 or NULL: natural log of the
 *        softmax denominator (-inf for a row that sees no key; its output row is 0).
 *   dev_status  device int32, required. */
bsa_status bsa_attend(const bsa_shape* shape, const void* q, const void* k, const void* v,
                      const int32_t* kv_idx, const int32_t* kv_cnt, int W, float softmax_scale,
                      void* out, float* lse, int32_t* dev_status, void* stream);

/* ---- vertical-slash sparse attention ([VSP] Metodologia A, B.3) ------------------- */

/* Query row i of head (b, h) attends to the union, each key once, of the vertical
 * columns j <= i and the keys i - o of the slash offsets o <= i:
 *   O_i = sum over those keys j of softmax(scale * q_i.k_j) v_j.
 *   v_idx [B,Hq,Wv] int32, device: vertical key positions (any order), the first
 *         v_cnt[b,h] used;  s_off [B,Hq,Ws] int32, device: slash offsets (any order),
 *         the first s_cnt[b,h] used. Entries outside [0, N) are skipped and reported
 *         as BSA_DEV_BAD_INDEX; counts outside [0, width] are reported and clamped.
 *   out like Q (bf16); lse [B,Hq,N] fp32 or NULL (-inf, with output 0, for a row
 *         with no key).  dev_status device int32, required.
 * The two index lists are merged per query tile into the ascending list of the key
 * blocks that hold a kept key, and the attention masks every (row, key) pair by the
 * rule above ([VSP] B.3 merges the vertical and diagonal indices in the kernel).
 * Shapes: bf16, d 128, block_k 64, tile_q 128; Wv, Ws >= 1 and min(N/64, Wv + 3*Ws)
 * <= 1024 (else BSA_ERR_UNSUPPORTED). Workspace: bsa_attend_vs_workspace_bytes()
 * bytes, 256-byte aligned (0 for an unsupported shape). */
size_t bsa_attend_vs_workspace_bytes(const bsa_shape* shape, int Wv, int Ws);
bsa_status bsa_attend_vs(const bsa_shape* shape, const void* q, const void* k, const void* v,
                         const int32_t* v_idx, const int32_t* v_cnt, int Wv,
                         const int32_t* s_off, const int32_t* s_cnt, int Ws, float softmax_scale,
                         void* out, float* lse, int32_t* dev_status, void* workspace,
                         size_t workspace_bytes, void* stream);

/* ---- decode with run-time termination ([ART] 2.1-2.4) ----------------------------- */

/* q [B,Hq,d], k_cache/v_cache [B,Hkv,L,d] bf16. Per (batch, KV head) the blocks
 * 0,1,2,... are streamed in order with an online softmax for the group's query heads;
 * block 0 is always processed ([ART] 2.4); after each block t >= 1 the stability test
 * runs and streaming stops after `patience` consecutive stable blocks.
 *   out          [B,Hq,d] bf16: normalised output over the processed blocks.
 *   blocks_used  [B,Hkv] int32.
 *   probe_trace  [B,Hkv,L/block_kv,n_probe] fp32 or NULL: x^(t) for every processed
 *                block (later entries untouched).
 *   dev_status   device int32, required. */
bsa_status bsa_decode(const bsa_decode_shape* shape, const bsa_decode_params* params,
                      const void* q, const void* k_cache, const void* v_cache,
                      float softmax_scale, void* out, int32_t* blocks_used,
                      float* probe_trace, int32_t* dev_status, void* stream);

/* Decode over a block list: the same stream, test and stop rule as bsa_decode, but
 * each (batch, KV head) visits the blocks of its list in list order -- for example a
 * selector's kv_idx visited first block first, then most important or most recent
 * first. [ART] 2.4: a full pass does not depend on the visiting order; the first
 * listed block is always processed (no test before the second visit step).
 *   block_list  [B,Hkv,list_width] int32, device: block numbers (0 <= j < L/block_kv)
 *               in visiting order; entries at or beyond list_cnt are ignored. An
 *               out-of-range entry is skipped and reported as BSA_DEV_BAD_INDEX; a
 *               block listed twice is visited twice (the caller lists each once).
 *   list_cnt    [B,Hkv] int32, device: entries used (clamped to 0..list_width, with
 *               BSA_DEV_BAD_INDEX when outside). An empty list gives out = 0,
 *               blocks_used = 0.
 *   list_width  1..4096 (BSA_ERR_UNSUPPORTED beyond).
 *   blocks_used [B,Hkv] int32: visit steps processed.
 *   probe_trace [B,Hkv,list_width,n_probe] fp32 or NULL: x^(t) per visit step.
 * Other arguments, layouts and errors as bsa_decode. */
bsa_status bsa_decode_list(const bsa_decode_shape* shape, const bsa_decode_params* params,
                           const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_list, const int32_t* list_cnt, int list_width,
                           float softmax_scale, void* out, int32_t* blocks_used,
                           float* probe_trace, int32_t* dev_status, void* stream);

/* ---- selection without a caller-provided workspace -------------------------------- */

/* The pages have no counterpart to this call; it exists for callers that cannot
 * allocate device memory (for example a plugin whose host process owns all device
 * memory through its own pool, or a serving loop where a cudaMalloc could
 * synchronise the device). It does exactly what bsa_select does, with the same
 * arguments minus the workspace, and allocates nothing: its scratch is a static
 * array of bsa_select_noalloc_max_bytes() bytes (32 MiB) in device memory that
 * every GPU loading libbsa.so keeps until the process exits.
 *   - Shapes whose bsa_select_workspace_bytes() exceed that size are rejected with
 *     BSA_ERR_UNSUPPORTED (bsa_last_error() says why); nothing is launched.
 *   - Every call looks up the array's device address in the current device's
 *     current context. The first call on a device also loads the library's device
 *     code there; make that first call before any stream capture.
 *   - All calls share the one array. Calls that overlap on the GPU (other streams,
 *     other host threads on the same device) race on it: the caller must order them.
 *     The array keeps the last call's contents; no entry has to start at zero. */
size_t bsa_select_noalloc_max_bytes(void);
bsa_status bsa_select_noalloc(const bsa_shape* shape, const bsa_select_params* params,
                              const float* scores, int32_t* kv_idx, int32_t* kv_cnt,
                              float* sigma, float* sigma_bar, uint8_t* trigger, float* theta,
                              int32_t* dev_status, void* stream);

/* ---- self-test of the bounded device waits ------------------------------------------ */

/* The pages have no counterpart to this call. It exercises, on the GPU, the bounded
 * mbarrier wait that every tensor-core kernel of this library uses for its pipeline
 * stages (the device-side "wait timeout" error of the calls above):
 *   mode 0: two waits on barriers nothing completes. The first gives up after the
 *           library's wait limit (1 s), ORs BSA_DEV_TIMEOUT into *dev_status and raises
 *           the CTA's abort flag; the second then gives up through that flag.
 *           completed[0] = completed[1] = 0.
 *   mode 1: both barriers are completed first; both waits succeed, *dev_status = 0,
 *           completed[0] = completed[1] = 1.
 * dev_status: device int32, zeroed by the call. completed: device int32[2].
 * Asynchronous on stream; the kernel never traps or spins without a bound, and the
 * context stays usable afterwards. Returns BSA_ERR_INVALID_ARG for another mode or a
 * null pointer, BSA_ERR_CUDA if the launch fails. */
bsa_status bsa_selftest_wait(int mode, int32_t* dev_status, int32_t* completed, void* stream);

/* ---- which kernels a call runs ------------------------------------------------------ */

/* The compute calls pick their kernels from the shape alone. These queries return the
 * choice without launching anything: BSA_PATH_TENSOR_CORES (tcgen05/TMEM/TMA kernels for
 * scoring and attention; for decode, TMA-fed warp-level mma.sync, whose per-instruction
 * latency suits the few query heads of a KV head),
 * BSA_PATH_CUDA_CORES (fp32 CUDA-core kernels, about an order of magnitude slower on
 * large problems), or -1 for arguments the call itself would reject.
 *   bsa_score_path   tensor cores for bf16 inputs with d = 128 and query tiles of 128
 *                    (any key block); CUDA cores for BSA_F32 inputs, d = 64 or query tiles
 *                    of 64. The same holds for bsa_score_select, which ranks inside the
 *                    tensor-core score kernel for the mean-pooled kinds.
 *   bsa_attend_path  tensor cores for bf16, d = 128, key blocks of 64, query tiles of 128,
 *                    W <= 1024 and B*Hq*N < 2^31; CUDA cores for every other shape
 *                    (BSA_F32, d = 64, key blocks of 128, query tiles of 64, W > 1024).
 *   bsa_decode_path  tensor cores for d = 128 and block_kv = 128; CUDA cores for d = 64
 *                    or block_kv = 64 (decode takes bf16 caches, Hq/Hkv in {1, 2, 4, 8}
 *                    and B*Hkv*L < 2^31 only; -1 otherwise).
 * bsa_attend_vs always runs on tensor cores (other shapes are rejected). */
enum { BSA_PATH_CUDA_CORES = 0, BSA_PATH_TENSOR_CORES = 1 };
int bsa_score_path(const bsa_shape* shape, bsa_score_kind kind);
int bsa_attend_path(const bsa_shape* shape, int W);
int bsa_decode_path(const bsa_decode_shape* shape);

/* ---- misc --------------------------------------------------------------------------- */

const char* bsa_status_string(bsa_status status);
/* Reason for the last non-OK status returned on this thread ("" if none). */
const char* bsa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */
