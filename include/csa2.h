/*
 * csa2.h - C ABI of libcsa2, the B200 (sm_100a) decode hot path of Compressed
 * Sparse Attention 2 (CSA2) with an FP4 main-KV cache, as described on the
 * DeepSeek V4.1 Flash KV-cache pages:
 *
 *  [G] "DeepSeek V4.1 Flash KV Cache: 890 Bytes per Token Explained",
 *      sections on CSA2 modes, the hierarchical sparse indexer and FP4 storage.
 *  [N] "DeepSeek-V4.1-Flash: 890 Bytes Per Token, 437x Smaller KV Cache",
 *      sections "CSA2: Sharing Main KV, Indexer K, and Top-K Indices Across
 *      Layers", "FP4 KV Quantization and Cache Lifetime Management" and
 *      "Causal Encoder-Decoder and Prefill Halving".
 *  [T] "890 bytes per token: how DeepSeek V4.1-Flash's KV cache works",
 *      "Mechanism 4: the hierarchical sparse indexer".
 *
 * Conventions shared by every call:
 *  - Every data pointer is DEVICE memory owned by the caller; the library
 *    never allocates, frees or keeps a pointer after the call returns.
 *    Scratch space comes in through (ws, ws_bytes); the *_workspace_size
 *    functions give the bytes needed.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream). The return value reports host-side argument checks and
 *    launch errors only (cudaGetLastError after the launches).
 *  - Return value: CSA2_OK or a negative csa2_status. On error nothing has
 *    been launched, except CSA2_ERR_CUDA, which reports a failed launch.
 *  - Kernels never trap: an out-of-range position found on the device is
 *    skipped, not written; a wait inside a kernel that runs out its time or
 *    iteration bound records it in a device flag and the kernel returns
 *    (csa2_device_status reads the flags).
 *  - bf16 tensors are IEEE bfloat16 bit patterns; fp32 is IEEE binary32.
 *  - Layouts are row-major with the listed dimensions, densely packed.
 *  - Selection order everywhere: score descending, then position ascending.
 *    Index outputs are listed in ascending order, padded with -1.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSA2_ABI_VERSION 1

/* Constants the pages fix ([G] indexer section, [N] CSA2 and CED sections). */
#define CSA2_POOL_BLOCKS 2048 /* candidate pool: up to 2,048 blocks ...      */
#define CSA2_BLOCK_TOKENS 8   /* ... of 8 tokens (16,384 positions)          */
#define CSA2_TOPK 512         /* each query keeps its best 512 candidates    */
#define CSA2_N_WIN 128        /* sliding window: the last 128 tokens         */
#define CSA2_FP4_GROUP 16     /* one E4M3 scale per 16 channels              */

typedef enum csa2_status {
    CSA2_OK = 0,
    CSA2_ERR_NULL = -1,      /* a required pointer is NULL                    */
    CSA2_ERR_SHAPE = -2,     /* a size is outside the supported range         */
    CSA2_ERR_ALIGN = -3,     /* a pointer or row size breaks the alignment rule */
    CSA2_ERR_RANGE = -4,     /* a host-side value is out of range             */
    CSA2_ERR_WORKSPACE = -5, /* ws is NULL or smaller than required           */
    CSA2_ERR_CUDA = -6,      /* a kernel launch failed                        */
    CSA2_ERR_DEVICE_TIMEOUT = -7 /* a kernel gave up a bounded wait (device flag) */
} csa2_status;

/* CSA2 layer modes ([N] CSA2 section). */
typedef enum csa2_mode {
    CSA2_MODE_FULL = 0,    /* score the whole context, build the pool, fresh top-512 */
    CSA2_MODE_REINDEX = 1, /* rescore the pool with the layer's own indexer Q        */
    CSA2_MODE_REUSE = 2    /* attend the indices of the nearest Full/Reindex layer   */
} csa2_mode;

/* Human-readable text for a status code (static storage). */
const char *csa2_status_string(int status);

/* CSA2_ABI_VERSION of the loaded library. */
int csa2_abi_version(void);

/* Device-side error status of the current device: CSA2_ERR_DEVICE_TIMEOUT if
 * any kernel of the library gave up a bounded wait since the flags were last
 * cleared, else CSA2_OK (CSA2_ERR_CUDA if the flags cannot be read). With
 * clear != 0 the flags are reset after reading. Synchronizes the device. The
 * outputs of a call whose kernel gave up are unspecified; the CUDA context
 * stays usable. */
int csa2_device_status(int clear);

/* Self-test of that path: launches one CTA whose wait on an mbarrier that
 * nothing completes gives up after limit_us microseconds (1..1,000,000) and
 * records the timeout, as a kernel of the library would. */
int csa2_selftest_wait_timeout(int limit_us, void *stream);

/* Per-call error word. The workspaces of csa2_sparse_attn_decode(_mxfp4) and
 * csa2_decode_stack start with the call's error word: the call clears it on
 * `stream` before its kernels run, and a kernel of that call that gives up a
 * bounded wait sets it (besides the library flags above), so a timeout can be
 * told apart from other calls on other streams. csa2_workspace_status reads
 * the word at the start of ws on `stream` and synchronizes that stream:
 * CSA2_ERR_DEVICE_TIMEOUT if it is set, else CSA2_OK; with clear != 0 a set
 * word is reset (on the stream). CSA2_ERR_NULL for a NULL ws, CSA2_ERR_CUDA if
 * the word cannot be read. csa2_decode_stack_noalloc keeps its word inside
 * the library: use csa2_device_status for it. */
int csa2_workspace_status(const void *ws, int clear, void *stream);

/* Self-test of the per-call word: as csa2_selftest_wait_timeout, and the
 * timeout also sets the error word at the start of ws (device memory of at
 * least 4 bytes; the call does not clear it first). */
int csa2_selftest_workspace_timeout(int limit_us, void *ws, void *stream);

/* ------------------------------------------------------------------------
 * FP4 append: quantize-and-pack new main-KV rows into the cache.
 * [G] FP4 section and [N] FP4 section: E2M1 elements, one E4M3 scale per 16
 * channels, NVFP4 without its global scale; quantized when written.
 *
 * For token row (b, i), i < n_new, written at position p = start_pos[b] + i:
 *   for each 16-channel group g:  s = E4M3_rn_satfinite(amax_g / 6)  (fp32 div)
 *     element c: code = E2M1_rn_satfinite(x_c / s) (fp32 div), +0 if s == 0
 *   kv_fp4[b][p][c/2]: byte holds channel 2j in its low nibble, 2j+1 high
 *   kv_sf[b][p][g]  : the E4M3 scale code
 *
 *  kv_bf16   [B][n_new][C] bf16, 16-byte aligned
 *  start_pos [B] int64 (device); rows with p outside [0, cap) are skipped
 *  kv_fp4    [B][cap][C/2] uint8, 8-byte aligned
 *  kv_sf     [B][cap][C/16] uint8 (E4M3)
 *  C % 16 == 0, 16 <= C <= 8192.
 * ------------------------------------------------------------------------ */
int csa2_kv_append_fp4(const void *kv_bf16, int B, int n_new, int C, const int64_t *start_pos,
                       int64_t cap, uint8_t *kv_fp4, uint8_t *kv_sf, void *stream);

/* ------------------------------------------------------------------------
 * MXFP4 variant of the append ([T] mechanism 3 calls the cache format MXFP4
 * and gives no detail; read as the OCP Microscaling format): E2M1 elements,
 * one E8M0 scale per 32 channels.
 * For token row (b, i) at p = start_pos[b] + i, per 32-channel block g:
 *   e = clamp(floor(log2(amax_g)) - 2, -127, 127)   (-127 when amax_g = 0)
 *   element c: code = E2M1_rn_satfinite(x_c * 2^-e)   (an exact scaling)
 *   kv_fp4[b][p][c/2]: as csa2_kv_append_fp4;  kv_sf[b][p][g] = e + 127
 *  kv_sf [B][cap][C/32] uint8 (E8M0); C % 32 == 0, 32 <= C <= 8192; other
 *  arguments and errors as csa2_kv_append_fp4.
 * ------------------------------------------------------------------------ */
int csa2_kv_append_mxfp4(const void *kv_bf16, int B, int n_new, int C, const int64_t *start_pos,
                         int64_t cap, uint8_t *kv_fp4, uint8_t *kv_sf, void *stream);

/* ------------------------------------------------------------------------
 * Full-mode indexer scan ([N] CSA2 section: a Full layer projects indexer K
 * and scores the context; [G] indexer section: 8-token blocks).
 *
 * Query (b, i) sees positions t < V(b, i), where V = ctx_len[b] when q_pos is
 * NULL (decode: the query sees the whole context) and
 * V = min(q_pos[b][i] + 1, ctx_len[b]) otherwise (causal prefill).
 *   S[t]      = sum_{h,d} q_idx[b][i][h][d] * k_idx[b][t][h][d]   (exact int32)
 *   tok[t]    = fp32_rn(S[t]) * k_scale[b][t]                     (one fp32 mul)
 *   blk[j]    = max_{t in [8j, 8j+8), t < V} tok[t],  j < ceil(V/8)
 *
 *  q_idx     [B][Nq][H][D] int8
 *  k_idx     [B][cap][H][D] int8, 16-byte aligned; H*D % 16 == 0, H*D <= 65536
 *  k_scale   [B][cap] fp32
 *  ctx_len   [B] int64 (device), 0 <= ctx_len <= cap
 *  q_pos     [B][Nq] int64 (device) or NULL
 *  tok_score [B][Nq][cap] fp32 or NULL; entries t >= V are not written
 *  blk_score [B][Nq][ceil(cap/8)] fp32; entries j >= ceil(V/8) are not written
 *  n_blk     [B][Nq] int32 or NULL: receives ceil(V/8)
 * ------------------------------------------------------------------------ */
int csa2_index_full(const int8_t *q_idx, const int8_t *k_idx, const float *k_scale,
                    const int64_t *ctx_len, const int64_t *q_pos, int B, int Nq, int H, int D,
                    int64_t cap, float *tok_score, float *blk_score, int32_t *n_blk, void *stream);

/* ------------------------------------------------------------------------
 * Top-k selection ([G] indexer section: the pool keeps the best 2,048 blocks
 * and each query its best 512 candidates; [N] CSA2 section: fresh top-512 in
 * Full and Reindex layers).
 *
 * Row r has candidates i < n_valid[r] (all n when n_valid is NULL) with score
 * score[r][i] and position cand_pos[r][i] (i itself when cand_pos is NULL);
 * candidates with a negative position are skipped. The best min(k, #valid)
 * under (score desc, position asc) are written to out[r] in ascending
 * position order, then -1 up to k entries. -0.0 ranks equal to +0.0.
 *
 *  score    [R][n] fp32 (no NaN)
 *  cand_pos [R][n] int32 or NULL
 *  n_valid  [R] int32 (device) or NULL
 *  out      [R][k] int32
 *  1 <= k <= 4096, 1 <= n < 2^31.
 *  ws/ws_bytes: at least csa2_topk_workspace_size(R, n, k) bytes (may be 0,
 *  in which case ws may be NULL).
 * ------------------------------------------------------------------------ */
size_t csa2_topk_workspace_size(int R, int64_t n, int k);
int csa2_topk(const float *score, const int32_t *cand_pos, const int32_t *n_valid, int R,
              int64_t n, int k, int32_t *out, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Pool gather for the Full layer's own top-512: list the pooled positions of
 * query (b, i) with the token scores the scan already produced ([G] indexer
 * section: each query keeps its best 512 of the pool).
 *   slot s*8 + r:  position p = 8*pool[b][i][s] + r,
 *                  pool_pos = p and pool_score = tok_score[b][i][p] if the pool
 *                  entry is >= 0 and p < V(b, i) (as in csa2_index_full),
 *                  else pool_pos = -1.
 *  tok_score  [B][Nq][cap] fp32
 *  pool       [B][Nq][P] int32 block ids (-1 = empty slot)
 *  pool_score [B][Nq][8P] fp32, pool_pos [B][Nq][8P] int32
 * ------------------------------------------------------------------------ */
int csa2_pool_gather(const float *tok_score, const int32_t *pool, const int64_t *ctx_len,
                     const int64_t *q_pos, int B, int Nq, int P, int64_t cap, float *pool_score,
                     int32_t *pool_pos, void *stream);

/* ------------------------------------------------------------------------
 * Full-layer selection in one call: the pool and the top-K of each query from
 * the scan's outputs ([G] indexer section: the pool keeps the best 2,048
 * blocks of 8 tokens and each query its best 512 candidates of the pool;
 * [N] CSA2 section: a Full layer builds the pool and selects a fresh top-512).
 * For query (b, i), with V = V(b, i) as in csa2_index_full and
 * nb = clamp(n_blk[b][i], 0, ceil(cap/8)):
 *   pool[b][i] = the best min(P, nb) of blk_score[b][i][0..nb) by (score desc,
 *                block id asc), block ids ascending, then -1;
 *   top[b][i]  = the best min(K, #) positions p = 8 j + r with j in the pool
 *                and p < V, by (tok_score[b][i][p] desc, p asc), ascending,
 *                then -1.
 * The result equals csa2_topk (k = P, n_valid = n_blk), csa2_pool_gather and
 * csa2_topk (k = K) in sequence, bit for bit; no intermediate buffer is
 * needed. One CTA per query holds a row in shared memory, hence the limits.
 * Precondition (as csa2_index_full writes them): blk_score[j] is the maximum
 * of tok_score over the visible positions of block j. The best K tokens then
 * lie in the best min(K, P) blocks, and only those blocks' tokens are read.
 *  blk_score [B][Nq][ceil(cap/8)] fp32, n_blk [B][Nq] int32
 *  tok_score [B][Nq][cap] fp32 (no NaN)
 *  ctx_len   [B] int64 (device); q_pos [B][Nq] int64 (device) or NULL
 *  pool      [B][Nq][P] int32, top [B][Nq][K] int32
 *  1 <= P <= 2048, 1 <= K <= 8 P, ceil(cap/8) <= 16384 and 8 P <= 16384;
 *  CSA2_ERR_SHAPE otherwise (the three calls have no such limits).
 * ------------------------------------------------------------------------ */
int csa2_full_select(const float *blk_score, const int32_t *n_blk, const float *tok_score,
                     const int64_t *ctx_len, const int64_t *q_pos, int B, int Nq, int64_t cap,
                     int P, int K, int32_t *pool, int32_t *top, void *stream);

/* ------------------------------------------------------------------------
 * Reindex rescoring ([N] CSA2 section: a Reindex layer reuses the main KV and
 * indexer K of the preceding Full layer and rescores the candidate pool with
 * its own indexer Q; [G] indexer section: later layers search only the pool).
 * Same slot layout as csa2_pool_gather, with the score computed as in
 * csa2_index_full from this layer's q_idx.
 *  q_idx [B][Nq][H][D] int8; k_idx, k_scale, ctx_len, q_pos as in csa2_index_full
 *  pool  [B][Nq][P] int32 block ids (-1 = empty slot)
 *  pool_score [B][Nq][8P] fp32, pool_pos [B][Nq][8P] int32
 * ------------------------------------------------------------------------ */
int csa2_index_reindex(const int8_t *q_idx, const int8_t *k_idx, const float *k_scale,
                       const int32_t *pool, const int64_t *ctx_len, const int64_t *q_pos, int B,
                       int Nq, int H, int D, int64_t cap, int P, float *pool_score,
                       int32_t *pool_pos, void *stream);

/* ------------------------------------------------------------------------
 * Sparse attention ([T] mechanism 4: attention runs only over the selected
 * candidates; [N] CED and CSA2 sections: every layer has its own main Q and
 * SWA KV, and the window is the last 128 tokens).
 *
 * For query (b, i) at position p (q_pos[b][i], or the position of the last
 * SWA row, swa_pos0[b] + swa_rows - 1, when q_pos is NULL) and head h, the
 * keys are the selected main-KV rows topk[b][i][0..K) (entries < 0 skipped),
 * dequantized as e2m1(code) * e4m3(scale), followed by the SWA rows whose
 * positions lie in [max(0, p - n_win + 1), p] (row r holds position
 * swa_pos0[b] + r). K = V = the row (one shared KV head). Then
 *   out[b][i][h] = sum_j softmax_j(softmax_scale * q[b][i][h] . key_j) key_j.
 * A query with no keys gets a zero output.
 *
 *  q_bf16   [B][Nq][Hq][C] bf16, 16-byte aligned
 *  kv_fp4   [B][cap][C/2] uint8, kv_sf [B][cap][C/16] uint8 (as written by
 *           csa2_kv_append_fp4)
 *  topk     [B][Nq][K] int32 positions (< cap)
 *  swa_bf16 [B][swa_rows][C] bf16, 16-byte aligned; swa_pos0 [B] int64 (device)
 *  out      [B][Nq][Hq][C] fp32
 *  C % 32 == 0, 32 <= C <= 1024; 1 <= Hq <= 256; 0 <= K <= 4096; 0 <= n_win <= 4096.
 *  ws/ws_bytes: at least csa2_sparse_attn_workspace_size(...) bytes (0 for
 *           shapes whose kernel has no bounded wait and no scratch: then ws
 *           may be NULL), 16-byte aligned (CSA2_ERR_ALIGN otherwise; device
 *           allocations are). It starts with the call's error word (read with
 *           csa2_workspace_status); the rest is the kernels' exchange space.
 * ------------------------------------------------------------------------ */
size_t csa2_sparse_attn_workspace_size(int B, int Nq, int Hq, int C, int K, int n_win);
int csa2_sparse_attn_decode(const void *q_bf16, const uint8_t *kv_fp4, const uint8_t *kv_sf,
                            int64_t cap, const int32_t *topk, int K, const void *swa_bf16,
                            const int64_t *swa_pos0, int swa_rows, const int64_t *q_pos,
                            int n_win, int B, int Nq, int Hq, int C, float softmax_scale,
                            float *out, void *ws, size_t ws_bytes, void *stream);

/* The same attention over an MXFP4 cache (csa2_kv_append_mxfp4): kv_sf is
 * [B][cap][C/32] E8M0, a row's value is e2m1(code) * 2^(e - 127); C % 32 == 0.
 * Everything else, including the workspace size, as csa2_sparse_attn_decode. */
int csa2_sparse_attn_decode_mxfp4(const void *q_bf16, const uint8_t *kv_fp4, const uint8_t *kv_sf,
                                  int64_t cap, const int32_t *topk, int K, const void *swa_bf16,
                                  const int64_t *swa_pos0, int swa_rows, const int64_t *q_pos,
                                  int n_win, int B, int Nq, int Hq, int C, float softmax_scale,
                                  float *out, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * One decode step of a CSA2 layer stack ([N] CSA2 section: static per-layer
 * modes; decoder groups 1 Full + 3 Reuse, then 1 Reindex + 3 Reuse).
 *
 * Runs, in layer order: Full -> csa2_index_full, pool selection (top
 * min(2048, nblk) blocks), csa2_pool_gather and the top-512; Reindex ->
 * csa2_index_reindex over the most recent Full layer's pool and the top-512;
 * Reuse -> nothing; then, for every layer, csa2_sparse_attn_decode with the
 * indices of the most recent Full/Reindex layer. One query per sequence
 * (Nq = 1) at position ctx_len[b] - 1, seeing the whole context.
 * With 512 channels, 64 heads and fewer than 64 sequences, the attention of a
 * Full or Reindex layer and the Reuse layers after it (up to 8 layers) runs as
 * one kernel launch: layer l + 1 of a sequence starts once layer l of that
 * sequence is written (per-sequence counters in the workspace; sequences are
 * independent and never wait for each other).
 * When kv_new_bf16 ([B][C] bf16, 16-byte aligned) is not NULL, the step first
 * appends that row to the FP4 cache at position ctx_len[b] - 1 (as
 * csa2_kv_append_fp4 does); the new token's indexer key is expected to be in
 * k_idx/k_scale already.
 *
 * Per layer (csa2_layer):
 *  mode   csa2_mode
 *  q_idx  [B][H][D] int8 for Full/Reindex layers, ignored for Reuse
 *  q      [B][Hq][C] bf16 main Q
 *  swa    [B][swa_rows][C] bf16 sliding-window KV (row r = position swa_pos0[b] + r)
 *  out    [B][Hq][C] fp32 attention output
 *  topk   [B][512] int32, written by Full/Reindex layers, ignored for Reuse
 * Shared:
 *  pool   [B][2048] int32, written by Full layers (the pool Reindex layers use)
 *  pool_ready: 1 if `pool` already holds the pool of a Full layer run by an
 *         earlier call (a stack that starts with a Reindex group), else 0;
 *         with 0 the first non-Reuse layer must be Full.
 *  softmax_scale as given (1/sqrt(C) in the pages' reading).
 *  scan_events: NULL, or two cudaEvent_t that are recorded on `stream` right
 *         before and right after the step's first indexer kernel: the first
 *         Full layer's scan, or, in a stack without a Full layer, the first
 *         Reindex rescoring (to time that kernel inside the step).
 *  ws/ws_bytes: at least csa2_decode_stack_workspace_size(...) bytes,
 *         16-byte aligned (CSA2_ERR_ALIGN otherwise; device allocations
 *         are); it starts with the call's error word (csa2_workspace_status),
 *         cleared by the call.
 *  Errors: CSA2_ERR_RANGE if a Reuse layer has no preceding Full/Reindex
 *  layer or a Reindex layer has no pool; nothing is launched then.
 * ------------------------------------------------------------------------ */
typedef struct csa2_layer {
    int mode;
    const int8_t *q_idx;
    const void *q;
    const void *swa;
    float *out;
    int32_t *topk;
} csa2_layer;

size_t csa2_decode_stack_workspace_size(int B, int Hq, int C, int H, int D, int64_t cap);
int csa2_decode_stack(const csa2_layer *layers, int n_layers, const void *kv_new_bf16,
                      const int8_t *k_idx, const float *k_scale, uint8_t *kv_fp4, uint8_t *kv_sf,
                      int64_t cap, const int64_t *ctx_len, const int64_t *swa_pos0, int swa_rows,
                      int B, int Hq, int C, int H, int D, float softmax_scale, int32_t *pool,
                      int pool_ready, void *const *scan_events, void *ws, size_t ws_bytes,
                      void *stream);

/* ------------------------------------------------------------------------
 * csa2_decode_stack_noalloc: csa2_decode_stack for callers that cannot
 * allocate device memory. The pages have no counterpart; this is a service of
 * this library.
 *
 * Who needs it: code that runs while a stream is being captured into a CUDA
 * graph (allocation is not allowed there), plugin hosts that pass a kernel only
 * its input and output buffers and own every allocation, and latency-critical
 * loops that cannot pay for the device-wide synchronisation cudaMalloc/cudaFree
 * may cause. They cannot provide the workspace csa2_decode_stack asks for.
 *
 * Arguments and results: as csa2_decode_stack, minus scan_events, ws and
 * ws_bytes. The scratch space is a file-scope device array of
 * CSA2_NOALLOC_SCRATCH_BYTES inside the library. Every GPU that loads the
 * library holds it until the process exits. The call allocates nothing.
 * Limit: problems whose csa2_decode_stack_workspace_size exceeds
 * CSA2_NOALLOC_SCRATCH_BYTES are rejected with CSA2_ERR_WORKSPACE before
 * anything is launched. (B = 4 sequences of 1,048,576 tokens need 18.5 MiB.)
 * Set-up: the first call on each device, with that device current, looks up
 * the array's device address (cudaGetSymbolAddress) and keeps it. Make that
 * first call before any stream capture. A failed look-up returns CSA2_ERR_CUDA.
 * The kept address belongs to the device's current CUDA context: after
 * cudaDeviceReset (or anything else that destroys that context) it no longer
 * names the array, so a process that resets a device must not call this entry
 * point on that device again.
 * Sharing: every call uses the same array, which keeps the last call's
 * contents. Calls that overlap on the GPU (other streams, other host threads)
 * race and must be serialised by the caller. No part of the array has to
 * start at zero.
 * ------------------------------------------------------------------------ */
#define CSA2_NOALLOC_SCRATCH_BYTES (24u << 20)
int csa2_decode_stack_noalloc(const csa2_layer *layers, int n_layers, const void *kv_new_bf16,
                              const int8_t *k_idx, const float *k_scale, uint8_t *kv_fp4,
                              uint8_t *kv_sf, int64_t cap, const int64_t *ctx_len,
                              const int64_t *swa_pos0, int swa_rows, int B, int Hq, int C, int H,
                              int D, float softmax_scale, int32_t *pool, int pool_ready,
                              void *stream);

/* ------------------------------------------------------------------------
 * csa2_attn_resident_clusters: how many 8-CTA clusters of the tensor-core
 * attention kernel can be resident at once on the current device when each
 * cluster takes heads_per_cluster (16, 32 or 64) of the 64 query heads. The
 * decode stack splits the heads as finely as the (query row, head group)
 * items still fit in that many clusters. An introspection aid for callers
 * sizing batches; the pages have no counterpart. Returns the count (at least
 * 1; the library's upper bound of 18 when the occupancy query fails), or
 * CSA2_ERR_RANGE for another heads_per_cluster. Needs a current device.
 * ------------------------------------------------------------------------ */
int csa2_attn_resident_clusters(int heads_per_cluster);

#ifdef __cplusplus
}
#endif

#endif /* CSA2_H */
