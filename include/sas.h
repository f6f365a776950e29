/*
 * sas.h -- C ABI of the SAS gated block-sparse causal attention library
 * (libsas.so, CUDA kernels for sm_100a).
 *
 * The method (SAS close reading, liuzhao09.github.io, sections 2.1, 2.2 and
 * 2.4; SAS reproduction note, daiwk.github.io, core formula):
 *   - the sequence is cut into contiguous blocks of b = 64 tokens;
 *   - each history block m has a summary kbar_m (the mean of its 64 keys);
 *   - a selector scores the C causally visible history blocks,
 *     s_m = scale * qbar . kbar_m, scale = 1/sqrt(d) by default;
 *   - the gate is g = softmax(s) over those C blocks, g0 = 1 for the current
 *     block, log g_m = s_m - LSE(s);
 *   - I = TopK(s, k) (ties go to the lower block index), S = B0 + I, with B0
 *     the current block, always kept and causally masked;
 *   - o = softmax(q K_S^T * scale + log g_S) V_S;
 *   - the backward pass returns dQ, dK, dV and, per selected block, d(log g):
 *     the sum of the logit gradients inside that block.
 *
 * Conventions shared by every call
 *   - Every tensor pointer is a DEVICE pointer, allocated and owned by the
 *     caller. The library never allocates, frees or synchronises (apart from
 *     the two diagnostic calls at the end of this file); all work is enqueued
 *     on `stream` (NULL = the legacy default stream) and the call returns as
 *     soon as it is enqueued.
 *   - Layouts are dense row-major ("HND"): q, o, dO, dq [B][Hq][N][d];
 *     k, v, dk, dv [B][Hkv][N][d]; decode q/o [B][Hq][d]; caches
 *     [B][Hkv][Lmax][d]; block summaries [B][Hkv][N/64][d] fp32 (bf16 too
 *     through the *_ex and sas_block_summary_last calls).
 *     Selection rows: prefill idx/logg/dlogg [B][Hkv][T][topk] and cnt
 *     [B][Hkv][T] with T = ceil(N/64); decode idx [B][Hkv][topk].
 *     idx lists the kept history blocks in ascending order, padded with -1;
 *     cnt = min(topk, C).
 *   - Element type of q/k/v/o/dO/dq/dk/dv/caches: SAS_BF16 or SAS_F32, the
 *     same for all of them in one call. Scores, gates and lse are fp32,
 *     summaries fp32 unless a call says otherwise; accumulation is fp32.
 *   - Supported: d in {64, 128}; block size 64 (fixed); Hq % Hkv == 0;
 *     Hq/Hkv <= 8; 1 <= topk <= 128 (topk = 0 is accepted where stated);
 *     every pointer 16-byte aligned. Other shapes return SAS_ERR_UNSUPPORTED.
 *   - scale <= 0 selects the default 1/sqrt(d).
 *   - Invalid arguments are rejected on the host before any launch, with
 *     SAS_ERR_INVALID_ARG and a message in sas_last_error_message().
 *   - Workspace: each call that needs scratch memory states its size through
 *     a *_workspace_size() function; pass a caller-owned device buffer of at
 *     least that many bytes (16-byte aligned) as ws/ws_bytes. Contents need
 *     not be initialised. Calls that share a workspace must not overlap.
 *   - Calls are stateless apart from the workspace and may be captured in a
 *     CUDA graph.
 */
#ifndef SAS_H
#define SAS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* sas_stream_t;

typedef enum sas_status {
  SAS_OK = 0,
  SAS_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or argument      */
  SAS_ERR_UNSUPPORTED = 2,  /* valid but not implemented (d, group, topk)    */
  SAS_ERR_CUDA = 3,         /* a CUDA launch or runtime call failed          */
  SAS_ERR_TIMEOUT = 4,      /* a bounded device wait gave up (see below)     */
  SAS_ERR_INTERNAL = 5      /* an internal consistency check failed          */
} sas_status;

typedef enum sas_dtype { SAS_F32 = 0, SAS_BF16 = 1 } sas_dtype;
typedef enum sas_mode { SAS_PREFILL = 0, SAS_DECODE = 1 } sas_mode;

/* Static text for a status code. */
const char* sas_strerror(sas_status status);
/* Detail of the last failing call on this host thread ("" if none). */
const char* sas_last_error_message(void);
/* Library version, major*10000 + minor*100 + patch. */
int sas_version(void);

/*
 * Block summaries (SAS close reading, section 2.1: a block summary compresses
 * the block's adjacent keys; here the mean of the 64 keys).
 *   k     [B][H][N][d] (dt)              input
 *   lens  [B] int32 or NULL              valid length per sequence; blocks
 *                                        not complete within lens[b] get 0
 *   ksum  [B][H][N/64][d] fp32           output, ksum[b,h,m] = mean of keys
 *                                        64m .. 64m+63
 * No workspace. N/64 == 0 is a no-op.
 */
sas_status sas_block_summary(const void* k, sas_dtype dt, int B, int H, int N, int d,
                             const int32_t* lens, float* ksum, sas_stream_t stream);

/*
 * Selector scores, normalised gate and Top-K (SAS close reading, sections 2.1
 * and 2.2: s = R(q, {K_Bm}), I = TopK(s, k), g = softmax(s), log g = s - LSE).
 * The selector is parameter-free: s_m = scale * qbar . ksum_m.
 *   mode SAS_PREFILL: q [B][Hq][N][d]; one row per (b, kv group r, query
 *     block t), qbar = mean of q over the group's Hq/Hkv heads and the query
 *     block's tokens, C = t. Outputs idx/logg [B][Hkv][T][topk], cnt
 *     [B][Hkv][T]. lens must be NULL.
 *   mode SAS_DECODE: q [B][Hq][d] (one token per sequence at position
 *     lens[b]-1); one row per (b, r), qbar = mean over the group's heads,
 *     C = (lens[b]-1)/64. N is Lmax. Outputs idx/logg [B][Hkv][topk], cnt
 *     [B][Hkv]. lens [B] int32 device, 1 <= lens[b] <= N.
 *   ksum  [B][Hkv][N/64][d] fp32 (from sas_block_summary)
 *   logg  log g of each kept block (padding slots 0)
 *   scores_out  fp32 or NULL: the raw selector scores s_m of every row,
 *     prefill [B][Hkv][T][T] (row (b, r, t), column m) and decode
 *     [B][Hkv][N/64]; entries m >= C hold -inf. Written only when non-NULL
 *     (16-byte aligned); nothing on the attention path reads them.
 *   topk >= 0; topk = 0 gives cnt = 0.
 * Workspace: sas_select_workspace_size().
 */
size_t sas_select_workspace_size(int B, int Hq, int Hkv, int N, int d, int topk, sas_mode mode);
sas_status sas_select(const void* q, sas_dtype dt, const float* ksum, int B, int Hq, int Hkv,
                      int N, int d, int topk, sas_mode mode, const int32_t* lens, float scale,
                      int32_t* idx, int32_t* cnt, float* logg, float* scores_out, void* ws,
                      size_t ws_bytes, sas_stream_t stream);

/*
 * Prefill selection that allocates nothing and takes no workspace. The paper
 * has no counterpart: this is an interface variant of sas_select(SAS_PREFILL)
 * for callers that cannot allocate device memory when they call, such as a
 * host runtime that hands a kernel library only its input and output
 * buffers and forbids device allocation after start-up (cudaMalloc can
 * synchronise the device and has no latency bound).
 *   Same arguments, layouts and results as sas_select in SAS_PREFILL mode
 *   (without scores_out).
 *   Its scratch (the fp32 query summary of every (b, kv group, query block),
 *   B*Hkv*ceil(N/64)*d*4 bytes) lives in a fixed device array inside the
 *   library of sas_select_prefill_noalloc_capacity() bytes (4 MiB), which
 *   every GPU that loads the library keeps until the process exits. Larger
 *   problems are rejected with SAS_ERR_UNSUPPORTED and a message.
 *   The first call on each device looks up the array's device address once
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   All calls share the array; each call overwrites what it reads, and calls
 *   that overlap on the GPU (other streams, other threads) race on it.
 *   Calls no cudaMalloc, cudaFree or allocating library routine.
 */
size_t sas_select_prefill_noalloc_capacity(void);
sas_status sas_select_prefill_noalloc(const void* q, sas_dtype dt, const float* ksum, int B,
                                      int Hq, int Hkv, int N, int d, int topk, float scale,
                                      int32_t* idx, int32_t* cnt, float* logg,
                                      sas_stream_t stream);

/*
 * Gated sparse attention forward for prefill/training (SAS close reading,
 * sections 2.2 and 2.4; reproduction note, core formula):
 *   o_i = sum_j softmax_j(z_ij) v_j,  lse_i = log sum_j exp(z_ij),
 *   z_ij = scale * q_i . k_j + logg[slot(j)] for keys of kept history blocks,
 *   z_ij = scale * q_i . k_j for keys j <= i of the current block.
 * Unselected blocks are skipped, never masked.
 *   q [B][Hq][N][d], k, v [B][Hkv][N][d]     inputs (dt)
 *   idx, cnt, logg                           prefill selection rows (any
 *     selection is accepted: ascending distinct indices < t, -1 padded)
 *   o [B][Hq][N][d] (dt), lse [B][Hq][N] fp32 outputs
 * Workspace: sas_attn_fwd_workspace_size() (may be 0).
 */
size_t sas_attn_fwd_workspace_size(int B, int Hq, int Hkv, int N, int d, int topk, sas_dtype dt);
sas_status sas_attn_fwd(const void* q, const void* k, const void* v, sas_dtype dt, int B, int Hq,
                        int Hkv, int N, int d, const int32_t* idx, const int32_t* cnt,
                        const float* logg, int topk, float scale, void* o, float* lse, void* ws,
                        size_t ws_bytes, sas_stream_t stream);

/*
 * Backward of the forward above for L with dL/do = dO (SAS close reading,
 * section 2.4 and eq. 5): with p recomputed from lse,
 *   D_i = dO_i . o_i, dp_ij = dO_i . v_j, dz_ij = p_ij (dp_ij - D_i),
 *   dq_i = scale sum_j dz_ij k_j, dk_j = scale sum_i dz_ij q_i,
 *   dv_j = sum_i p_ij dO_i,
 *   dlogg[b,r,t,slot] = sum over the group's heads, the rows of query block t
 *     and the slot's 64 keys of dz.
 *   o, lse: the forward's outputs for the same inputs.
 *   dq [B][Hq][N][d], dk, dv [B][Hkv][N][d] (dt), dlogg [B][Hkv][T][topk]
 *   fp32 outputs; padding slots of dlogg are 0. Outputs are overwritten.
 * Workspace: sas_attn_bwd_workspace_size().
 */
size_t sas_attn_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d, int topk, sas_dtype dt);
sas_status sas_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, sas_dtype dt, int B, int Hq, int Hkv, int N, int d,
                        const float* lse, const int32_t* idx, const int32_t* cnt,
                        const float* logg, int topk, float scale, void* dq, void* dk, void* dv,
                        float* dlogg, void* ws, size_t ws_bytes, sas_stream_t stream);

/*
 * One decode step (SAS close reading, section 2.4 serving path: GQA groups
 * share one block set; section 2.1: the current block is always kept):
 * selection as sas_select(SAS_DECODE), then for every head h of group r
 *   o_h = softmax(scale * q_h K_S^T + bias) V_S over the kept blocks and the
 *   lens[b]-64t tokens of the current block t = (lens[b]-1)/64, with
 *   bias = logg of the key's block when gated = 1 and 0 when gated = 0
 *   (the inference-time "Algorithm 2" reading, section 2.1).
 *   q [B][Hq][d], kc, vc [B][Hkv][Lmax][d] (dt), lens [B] int32 device
 *   ksum [B][Hkv][Lmax/64][d] fp32 summaries of the cache
 *   o [B][Hq][d] (dt) output; idx_out [B][Hkv][topk] int32 or NULL
 * One launch: a thread-block cluster per (b, kv group) selects, attends and
 * combines through distributed shared memory. Workspace:
 * sas_decode_workspace_size() returns 0; ws may be NULL.
 */
size_t sas_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int d, int topk);
sas_status sas_decode(const void* q, const void* kc, const void* vc, sas_dtype dt, int B, int Hq,
                      int Hkv, int Lmax, int d, const int32_t* lens, const float* ksum, int topk,
                      int gated, float scale, void* o, int32_t* idx_out, void* ws,
                      size_t ws_bytes, sas_stream_t stream);

/*
 * Decode attention for a given selection: the attention half of sas_decode,
 * with idx/cnt/logg as inputs (layouts of sas_select(SAS_DECODE)), so that any
 * selection and any gate can be applied. Same definition as sas_decode
 * (SAS close reading, sections 2.1, 2.2 and 2.4).
 *   idx [B][Hkv][topk] int32 (ascending, < (lens[b]-1)/64), cnt [B][Hkv],
 *   logg [B][Hkv][topk] fp32; o [B][Hq][d] (dt) output.
 * Workspace: sas_decode_attend_workspace_size().
 */
size_t sas_decode_attend_workspace_size(int B, int Hq, int Hkv, int Lmax, int d, int topk);
sas_status sas_decode_attend(const void* q, const void* kc, const void* vc, sas_dtype dt, int B,
                             int Hq, int Hkv, int Lmax, int d, const int32_t* lens,
                             const int32_t* idx, const int32_t* cnt, const float* logg, int topk,
                             int gated, float scale, void* o, void* ws, size_t ws_bytes,
                             sas_stream_t stream);

/*
 * Summaries in bf16, for cheaper long-context selection (SAS close reading,
 * liuzhao09.github.io, section 2.4: the selector still scans every history
 * block summary, so at very long contexts ranking, not attention I/O, sets
 * the decode cost; bf16 halves the bytes of that scan).
 * sas_block_summary_ex writes the summaries in sum_dt: SAS_F32 as
 * sas_block_summary, or SAS_BF16, the fp32 mean rounded to nearest even.
 * sas_decode_ex is sas_decode reading summaries of type sum_dt; the scores
 * are computed from the stored (rounded) summaries. Same arguments, layouts
 * and errors as sas_block_summary / sas_decode otherwise; sum_dt outside
 * {SAS_F32, SAS_BF16} is SAS_ERR_INVALID_ARG.
 */
sas_status sas_block_summary_ex(const void* k, sas_dtype dt, int B, int H, int N, int d,
                                const int32_t* lens, void* ksum, sas_dtype sum_dt,
                                sas_stream_t stream);
sas_status sas_decode_ex(const void* q, const void* kc, const void* vc, sas_dtype dt, int B,
                         int Hq, int Hkv, int Lmax, int d, const int32_t* lens, const void* ksum,
                         sas_dtype sum_dt, int topk, int gated, float scale, void* o,
                         int32_t* idx_out, sas_stream_t stream);

/*
 * Summary upkeep during decode (SAS close reading, section 2.4: serving keeps
 * the block summaries beside the cache). For every (sequence b, head h),
 * writes the summary of block C - 1, C = (lens[b] - 1) / 64: the last
 * complete block before the current one, which completed when the current
 * block began. Rows with C = 0 are left alone. Calling it once per decode
 * step keeps the summaries current as long as at most 64 tokens are appended
 * between calls (sas_block_summary rebuilds all of them otherwise).
 *   block_table NULL: k [B][H][N][d] (dt), ksum [B][H][N/64][d] (sum_dt).
 *   block_table [B][N/64] int32: k is the page pool [npages][H][64][d] and
 *     ksum the page summaries [npages][H][d]; the block's page is
 *     block_table[b][C - 1]. An entry outside [0, npages) skips the row and
 *     is reported by sas_device_status (kernel k_summary_last).
 *   lens [B] int32 device, 1 <= lens[b] <= N; N a multiple of 64.
 *   sum_dt SAS_F32 or SAS_BF16 (the fp32 mean rounded to nearest even).
 */
sas_status sas_block_summary_last(const void* k, sas_dtype dt, int B, int H, int N, int d,
                                  const int32_t* lens, void* ksum, sas_dtype sum_dt,
                                  const int32_t* block_table, int npages, sas_stream_t stream);

/*
 * Per-token selection prefill (SAS close reading, section 2.4: the fused
 * kernel masks, per query, the blocks below that query's gate threshold and
 * skips key tiles no query selected). Each query token i of kv group r has
 * its own row: qbar_i = the mean of the group's heads at token i, C_i = i/64
 * history blocks, s_m = scale * qbar_i . ksum_m, log g = s - LSE(s), Top-K
 * with ties to the lower block index; every head of the group attends over
 * its token's set and the causal part of the token's own block.
 *   Selection rows: idx/logg [B][Hkv][N][topk] (ascending, -1 / 0 padding),
 *   cnt [B][Hkv][N]; dlogg has the layout of logg.
 *   sas_select_tokens: q [B][Hq][N][d] (dt), ksum [B][Hkv][N/64][d] fp32.
 *   sas_attn_fwd_tokens / sas_attn_bwd_tokens: as sas_attn_fwd /
 *   sas_attn_bwd with per-token rows; the backward's workspace is
 *   sas_attn_bwd_tokens_workspace_size() bytes.
 *   sas_select_bwd_tokens: the selector's gradient for per-token rows (eq. 8,
 *   section 2.3, as sas_select_bwd): for token i of group r with C = i/64,
 *   ds_m = dlogg[slot of m] [m in I_i] - g_m sum_{l in I_i} dlogg[slot of l];
 *   each head of the group gets scale * sum_m ds_m ksum_m / G ADDED into dq
 *   at token i, and each of block m's 64 keys gets
 *   scale * sum_i ds_im qbar_i / 64 ADDED into dk. Its workspace is
 *   sas_select_bwd_tokens_workspace_size() bytes (fp32 summary gradients).
 *   N <= 32832 (512 history blocks per query block); larger N returns
 *   SAS_ERR_UNSUPPORTED. CUDA-core kernels (fp32 arithmetic).
 */
sas_status sas_select_tokens(const void* q, sas_dtype dt, const float* ksum, int B, int Hq,
                             int Hkv, int N, int d, int topk, float scale, int32_t* idx,
                             int32_t* cnt, float* logg, sas_stream_t stream);
sas_status sas_attn_fwd_tokens(const void* q, const void* k, const void* v, sas_dtype dt, int B,
                               int Hq, int Hkv, int N, int d, const int32_t* idx,
                               const int32_t* cnt, const float* logg, int topk, float scale,
                               void* o, float* lse, sas_stream_t stream);
size_t sas_attn_bwd_tokens_workspace_size(int B, int Hq, int Hkv, int N, int d);
size_t sas_select_bwd_tokens_workspace_size(int B, int Hq, int Hkv, int N, int d);
sas_status sas_select_bwd_tokens(const void* q, sas_dtype dt, const float* ksum, int B, int Hq,
                                 int Hkv, int N, int d, int topk, float scale, const int32_t* idx,
                                 const int32_t* cnt, const float* dlogg, void* dq, void* dk,
                                 void* ws, size_t ws_bytes, sas_stream_t stream);
sas_status sas_attn_bwd_tokens(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, sas_dtype dt, int B, int Hq, int Hkv, int N,
                               int d, const float* lse, const int32_t* idx, const int32_t* cnt,
                               const float* logg, int topk, float scale, void* dq, void* dk,
                               void* dv, float* dlogg, void* ws, size_t ws_bytes,
                               sas_stream_t stream);

/*
 * One decode step from and to host memory. When q_host is page-locked host
 * memory (cudaHostAlloc / cudaMallocHost), the step reads q straight from
 * it over the bus and q_dev is not touched; otherwise the copy of q_host
 * ([B][Hq][d], dt) into q_dev is enqueued on `stream` first. Likewise, when
 * o_host is page-locked the step writes o straight into it and o_dev is not
 * touched; otherwise it writes o_dev and a copy into o_host follows. The
 * caches, lens and summaries are device memory as in sas_decode. Returns
 * once the work is enqueued; o_host is valid after the stream reaches that
 * point, and q_host may be rewritten only after that point too.
 */
sas_status sas_decode_host(const void* q_host, void* q_dev, const void* kc, const void* vc,
                           sas_dtype dt, int B, int Hq, int Hkv, int Lmax, int d,
                           const int32_t* lens, const float* ksum, int topk, int gated,
                           float scale, void* o_dev, void* o_host, int32_t* idx_out,
                           sas_stream_t stream);

/*
 * Decode over a paged cache (the serving layout of the pages' SGLang /
 * FlashInfer setting; SAS close reading, section 2.4): as sas_decode, but
 * the caches are pools of 64-token pages, one page per (block, kv head):
 *   kpool, vpool  [npages][Hkv][64][d], dt
 *   kspool        [npages][Hkv][d] fp32: the summary (mean of the 64 keys) of
 *                 every full page; sas_block_summary over the pools viewed as
 *                 [npages][Hkv][64][d] (B = npages, N = 64) computes it, and
 *                 a serving loop refreshes it when a page fills
 *   block_table   [B][max_blocks] int32: page of each logical 64-token block
 *                 of sequence b (entries past ceil(lens[b]/64) unused;
 *                 out-of-range ids are replaced by page 0 and flagged, see
 *                 sas_device_status)
 *   lens          [B] int32, 1 <= lens[b] <= 64 max_blocks
 * idx_out holds logical block indices. Pages may be shared between
 * sequences (read only). Needs no workspace.
 */
sas_status sas_decode_paged(const void* q, const void* kpool, const void* vpool,
                            const float* kspool, sas_dtype dt, int B, int Hq, int Hkv, int npages,
                            int d, const int32_t* block_table, int max_blocks,
                            const int32_t* lens, int topk, int gated, float scale, void* o,
                            int32_t* idx_out, sas_stream_t stream);
/*
 * sas_decode_paged with the page summaries kspool [npages][Hkv][d] of type
 * sum_dt: SAS_F32 (as sas_decode_paged) or SAS_BF16 (the bf16 summaries of
 * sas_decode_ex: half the bytes of the summary scan; sas_block_summary_ex and
 * sas_block_summary_last with a block table write them). The scores are
 * computed from the stored summaries. sum_dt outside {SAS_F32, SAS_BF16} is
 * SAS_ERR_INVALID_ARG; arguments, layouts and errors as sas_decode_paged
 * otherwise.
 */
sas_status sas_decode_paged_ex(const void* q, const void* kpool, const void* vpool,
                               const void* kspool, sas_dtype sum_dt, sas_dtype dt, int B, int Hq,
                               int Hkv, int npages, int d, const int32_t* block_table,
                               int max_blocks, const int32_t* lens, int topk, int gated,
                               float scale, void* o, int32_t* idx_out, sas_stream_t stream);

/*
 * Selector backward (SAS close reading, section 2.3, eq. 8, sparse scope),
 * prefill rows: the gradient that reaches q and k through the selector,
 * ADDED into dq and dk (typically the outputs of sas_attn_bwd, so the two
 * calls give the full gradient). For each (b, r, t) with C = t visible
 * history blocks, kept set I (idx, cnt) and g = softmax(s):
 *   ds_m = dlogg[slot of m] [m in I] - g_m * sum_{l in I} dlogg[slot of l],
 * then with s_m = scale * qbar_t . kbar_m (the parameter-free selector of
 * sas_select): every row of block t and head of group r gets
 * scale * sum_m ds_m kbar_m / (G n_t), and every key of block m gets
 * scale * sum_t ds_tm qbar_t / 64.
 *   q      [B][Hq][N][d], dt          ksum  [B][Hkv][N/64][d] fp32 (summaries)
 *   idx, cnt, dlogg                   as sas_select / sas_attn_bwd (prefill rows)
 *   dq     [B][Hq][N][d], dt (in/out) dk    [B][Hkv][N][d], dt (in/out)
 *   ws     sas_select_bwd_workspace_size() bytes (query means and ds rows)
 * topk = 0 or N <= 64 leave dq and dk unchanged.
 */
size_t sas_select_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d);
sas_status sas_select_bwd(const void* q, sas_dtype dt, const float* ksum, int B, int Hq, int Hkv,
                          int N, int d, int topk, float scale, const int32_t* idx,
                          const int32_t* cnt, const float* dlogg, void* dq, void* dk, void* ws,
                          size_t ws_bytes, sas_stream_t stream);

/*
 * Device status. Kernels never trap: every wait on an mbarrier is bounded in
 * wall-clock time (200 ms); a wait that gives up, or a selection index out of
 * range (replaced by the current block), sets a bit in a per-kernel error
 * word in device memory, and the launch runs to completion with unspecified
 * results for the affected rows.
 *
 * sas_device_status synchronises `stream`, reads every kernel's error word
 * (they are per process and device, shared by all streams) and returns
 * SAS_ERR_TIMEOUT if any wait gave up, SAS_ERR_INTERNAL if only an index was
 * out of range, SAS_OK otherwise; sas_last_error_message() names the
 * kernels. clear != 0 resets the words afterwards (the status returned is
 * the one read before clearing). This call and sas_debug_wait_timeout are
 * the only ones that synchronise; they are for diagnostics and tests.
 */
sas_status sas_device_status(int clear, sas_stream_t stream);

/*
 * Test hook for the failure path: enqueues a one-warp kernel whose barrier
 * nothing completes. It gives up after the wait limit (200 ms), records a
 * timeout in its error word and exits; nothing hangs or faults. A following
 * sas_device_status returns SAS_ERR_TIMEOUT naming k_wait_selftest.
 */
sas_status sas_debug_wait_timeout(sas_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SAS_H */
