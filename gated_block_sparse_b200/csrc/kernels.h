// Host-side launchers of the SAS kernels (internal; the public ABI is sas.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sas {

// 3-D bf16 TMA tensor map over a row-major [planes][rows_per_plane][d] tensor
// ({64, 64, 1} box, 128-byte swizzle, zero fill); false when encoding fails.
bool make_tma_map_bf16_3d(CUtensorMap* map, const void* base, int d, int rows_per_plane,
                          int planes);
// 3-D fp32 TMA tensor map with a {box_d, box_rows, 1} box, no swizzle.
bool make_tma_map_f32_3d(CUtensorMap* map, const void* base, int d, int rows_per_plane,
                         int planes, int box_d, int box_rows);

// Block summaries: ksum[b,h,m] = mean of keys 64m..64m+63.
cudaError_t launch_block_summary(const void* k, int bf16, int B, int H, int N, int d,
                                 const int32_t* lens, float* ksum, cudaStream_t st);
// The same, summaries stored in bf16 (the fp32 mean rounded to nearest even).
cudaError_t launch_block_summary_bf16(const void* k, int bf16, int B, int H, int N, int d,
                                      const int32_t* lens, void* ksum, cudaStream_t st);
// Summary of each (sequence, head)'s last complete block, (lens[b]-1)/64 - 1
// (nothing when there is none); paged when bt != nullptr.
cudaError_t launch_summary_last(const void* k, int bf16, int B, int H, int N, int d,
                                const int32_t* lens, void* ksum, int sum_bf16,
                                const int32_t* bt, int max_blocks, int npages,
                                cudaStream_t st);
uint32_t* summary_error_word();

// Per-token selection prefill (k_tokens.cu): selection rows per query token,
// idx/logg [B][Hkv][N][topk], cnt [B][Hkv][N]; N <= tokens_max_n().
int tokens_max_n();
cudaError_t launch_select_tokens(const void* q, int bf16, const float* ksum, int B, int Hq,
                                 int Hkv, int N, int d, int topk, float scale, int32_t* idx,
                                 int32_t* cnt, float* logg, cudaStream_t st);
cudaError_t launch_attn_fwd_tokens(const void* q, const void* k, const void* v, int bf16, int B,
                                   int Hq, int Hkv, int N, int d, const int32_t* idx,
                                   const int32_t* cnt, const float* logg, int topk, float scale,
                                   void* o, float* lse, cudaStream_t st);
size_t attn_bwd_tokens_ws_bytes(int B, int Hkv, int N, int d);
cudaError_t launch_attn_bwd_tokens(const void* q, const void* k, const void* v, const void* o,
                                   const void* dout, int bf16, int B, int Hq, int Hkv, int N,
                                   int d, const float* lse, const int32_t* idx,
                                   const int32_t* cnt, const float* logg, int topk, float scale,
                                   void* dq, void* dk, void* dv, float* dlogg, void* ws,
                                   cudaStream_t st);
// Selector backward for per-token rows (eq. 8), added into dq and dk; ws
// holds the fp32 block-summary gradients [B][Hkv][N/64][d].
size_t select_bwd_tokens_ws_bytes(int B, int Hkv, int N, int d);
cudaError_t launch_select_bwd_tokens(const void* q, int bf16, const float* ksum, int B, int Hq,
                                     int Hkv, int N, int d, int topk, float scale,
                                     const int32_t* idx, const int32_t* cnt, const float* dlogg,
                                     void* dq, void* dk, void* ws, cudaStream_t st);
uint32_t* tokens_error_word();

// ---- selection
// Shared layout of one row's per-chunk partial results (decode scratch).
struct SelectPlan {
  int rows;       // number of selection rows
  int chunk;      // history blocks per chunk
  int nchunk;     // chunks per row
  int topk;
};
SelectPlan plan_decode_select(int B, int Hkv, int Lmax, int topk);
size_t decode_select_ws_bytes(const SelectPlan& p);

// scores (nullable): raw selector scores [B][Hkv][T][T], -inf at m >= t.
cudaError_t launch_select_prefill(const void* q, int bf16, const float* ksum, int B, int Hq,
                                  int Hkv, int N, int d, int topk, float scale, int32_t* idx,
                                  int32_t* cnt, float* logg, float* scores, void* ws,
                                  cudaStream_t st);
size_t select_prefill_ws_bytes(int B, int Hkv, int N, int d);
// Query means of the prefill selector, qbar [B][Hkv][T][d] fp32.
cudaError_t launch_qbar_prefill(const void* q, int bf16, int B, int Hq, int Hkv, int N, int d,
                                float* qbar, cudaStream_t st);

// ---- selector backward (k_select_bwd.cu)
// Adds the gradient that reaches q and k through the selector (eq. 8 of the
// gate, then s = scale qbar . kbar) into dq and dk. ws: qbar and the ds rows.
size_t select_bwd_ws_bytes(int B, int Hkv, int N, int d);
cudaError_t launch_select_bwd(const void* q, int bf16, const float* ksum, int B, int Hq, int Hkv,
                              int N, int d, int topk, float scale, const int32_t* idx,
                              const int32_t* cnt, const float* dlogg, void* dq, void* dk,
                              void* ws, cudaStream_t st);
// Prefill selection with its query-summary scratch in a fixed device array
// of the library (no workspace argument); capacity in fp32 values.
size_t select_prefill_static_capacity();
cudaError_t launch_select_prefill_static(const void* q, int bf16, const float* ksum, int B,
                                         int Hq, int Hkv, int N, int d, int topk, float scale,
                                         int32_t* idx, int32_t* cnt, float* logg,
                                         cudaStream_t st);

// Decode selection. `counters` holds one int per row and must be zero on
// entry (the kernel leaves it zero); `ws` holds the plan's partials.
// scores (nullable): raw selector scores [B][Hkv][Lmax/64], -inf at m >= C.
cudaError_t launch_select_decode(const void* q, int bf16, const float* ksum, int B, int Hq,
                                 int Hkv, int Lmax, int d, int topk, const int32_t* lens,
                                 float scale, int32_t* idx, int32_t* cnt, float* logg,
                                 float* scores, const SelectPlan& plan, int* counters, void* ws,
                                 cudaStream_t st);

// ---- decode attention
size_t decode_attend_ws_bytes(int B, int Hq, int Hkv, int topk, int d);
cudaError_t launch_decode_attend(const void* q, const void* kc, const void* vc, int bf16, int B,
                                 int Hq, int Hkv, int Lmax, int d, const int32_t* lens,
                                 const int32_t* idx, const int32_t* cnt, const float* logg,
                                 int topk, int gated, float scale, void* o, int* counters,
                                 void* ws, cudaStream_t st, bool pdl);
uint32_t* decode_error_word();

// One-launch decode step: selection + attention + combine, one thread-block
// cluster per (sequence, kv group); needs no workspace.
cudaError_t launch_decode_fused(const void* q, const void* kc, const void* vc, int bf16, int B,
                                int Hq, int Hkv, int Lmax, int d, const int32_t* lens,
                                const float* ksum, int topk, int gated, float scale, void* o,
                                int32_t* idx_out, cudaStream_t st);
// The same with the summaries' element type chosen: fp32 (sum_bf16 = 0) or
// bf16 (half the bytes of the summary scan).
cudaError_t launch_decode_fused_ex(const void* q, const void* kc, const void* vc, int bf16, int B,
                                   int Hq, int Hkv, int Lmax, int d, const int32_t* lens,
                                   const void* ksum, int sum_bf16, int topk, int gated,
                                   float scale, void* o, int32_t* idx_out, cudaStream_t st);
// Paged caches: kpool, vpool [npages][Hkv][64][d], kspool [npages][Hkv][d]
// (the summary of each page; fp32, or bf16 with sum_bf16 = 1), block_table
// [B][max_blocks] page ids.
cudaError_t launch_decode_paged(const void* q, const void* kpool, const void* vpool, int bf16,
                                int B, int Hq, int Hkv, int npages, int d,
                                const int32_t* block_table, int max_blocks, const int32_t* lens,
                                const void* kspool, int sum_bf16, int topk, int gated,
                                float scale, void* o, int32_t* idx_out, cudaStream_t st);
uint32_t* decode_fused_error_word();
uint32_t* attn_simt_error_word();

// ---- prefill attention (SIMT path: fp32 or bf16 inputs, any GPU of sm_100a)
cudaError_t launch_attn_fwd_simt(const void* q, const void* k, const void* v, int bf16, int B,
                                 int Hq, int Hkv, int N, int d, const int32_t* idx,
                                 const int32_t* cnt, const float* logg, int topk, float scale,
                                 void* o, float* lse, cudaStream_t st);
// Tensor-core forward (tcgen05 + TMEM + TMA): bf16, d = 128, even group size.
bool attn_fwd_tc_supported(int bf16, int d, int Hq, int Hkv);
cudaError_t launch_attn_fwd_tc(const void* q, const void* k, const void* v, int B, int Hq,
                               int Hkv, int N, const int32_t* idx, const int32_t* cnt,
                               const float* logg, int topk, float scale, void* o, float* lse,
                               cudaStream_t st);
// The same kernel with per-token selection rows (idx/logg [B][Hkv][N][topk],
// cnt [B][Hkv][N]): units are the union of the query block's tokens' blocks;
// N <= 64 * 513.
cudaError_t launch_attn_fwd_tc_tokens(const void* q, const void* k, const void* v, int B, int Hq,
                                      int Hkv, int N, const int32_t* idx, const int32_t* cnt,
                                      const float* logg, int topk, float scale, void* o,
                                      float* lse, cudaStream_t st);
uint32_t* attn_fwd_tc_error_word();
// Tensor-core backward (same support as the forward); ws as attn_bwd_simt.
cudaError_t launch_attn_bwd_tc(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, int B, int Hq, int Hkv, int N,
                               const float* lse, const int32_t* idx, const int32_t* cnt,
                               const float* logg, int topk, float scale, void* dq, void* dk,
                               void* dv, float* dlogg, void* ws, cudaStream_t st);
// The same kernel with per-token selection rows (layouts as the per-token
// forward; dlogg [B][Hkv][N][topk]); ws as launch_attn_bwd_tc.
cudaError_t launch_attn_bwd_tc_tokens(const void* q, const void* k, const void* v,
                                      const void* o, const void* dout, int B, int Hq, int Hkv,
                                      int N, const float* lse, const int32_t* idx,
                                      const int32_t* cnt, const float* logg, int topk,
                                      float scale, void* dq, void* dk, void* dv, float* dlogg,
                                      void* ws, cudaStream_t st);
uint32_t* attn_bwd_tc_error_word();

// Self-test of the bounded wait (k_status.cu): one warp waits on a barrier
// that nothing completes; after the wait limit it records kErrWaitTimeout in
// its own error word.
cudaError_t launch_wait_selftest(cudaStream_t st);
uint32_t* selftest_error_word();
size_t attn_bwd_simt_ws_bytes(int B, int Hkv, int N, int d);
cudaError_t launch_attn_bwd_simt(const void* q, const void* k, const void* v, const void* o,
                                 const void* dout, int bf16, int B, int Hq, int Hkv, int N, int d,
                                 const float* lse, const int32_t* idx, const int32_t* cnt,
                                 const float* logg, int topk, float scale, void* dq, void* dk,
                                 void* dv, float* dlogg, void* ws, cudaStream_t st);

}  // namespace sas
