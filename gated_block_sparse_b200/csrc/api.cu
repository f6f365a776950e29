// C ABI of libsas (declared in include/sas.h): argument validation, workspace
// carving and kernel launches. Host code only; the kernels live in k_*.cu.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <string>

#include "../../include/sas.h"
#include "kernels.h"
#include "ptx.cuh"

namespace {

thread_local std::string g_last_error;

sas_status fail(sas_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

sas_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return SAS_OK;
  return fail(SAS_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE(cond, st, ...) \
  do {                         \
    if (!(cond)) return fail(st, __VA_ARGS__); \
  } while (0)

#define REQUIRE_PTR(p)                                                                   \
  do {                                                                                   \
    if ((p) == nullptr) return fail(SAS_ERR_INVALID_ARG, "%s must not be NULL", #p);     \
    if (!aligned16(p)) return fail(SAS_ERR_INVALID_ARG, "%s must be 16-byte aligned", #p); \
  } while (0)

sas_status check_common(sas_dtype dt, int B, int Hq, int Hkv, int N, int d, int topk) {
  REQUIRE(dt == SAS_F32 || dt == SAS_BF16, SAS_ERR_INVALID_ARG, "dtype must be SAS_F32 or SAS_BF16");
  REQUIRE(B >= 0 && N >= 0, SAS_ERR_INVALID_ARG, "B and N must be >= 0 (B=%d N=%d)", B, N);
  REQUIRE(Hq >= 1 && Hkv >= 1, SAS_ERR_INVALID_ARG, "head counts must be >= 1 (Hq=%d Hkv=%d)", Hq, Hkv);
  REQUIRE(Hq % Hkv == 0, SAS_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  REQUIRE(Hq / Hkv <= 8, SAS_ERR_UNSUPPORTED, "at most 8 query heads per kv head (got %d)", Hq / Hkv);
  REQUIRE(d == 64 || d == 128, SAS_ERR_UNSUPPORTED, "head dim must be 64 or 128 (got %d)", d);
  REQUIRE(topk >= 0, SAS_ERR_INVALID_ARG, "topk must be >= 0 (got %d)", topk);
  REQUIRE(topk <= 128, SAS_ERR_UNSUPPORTED, "topk must be <= 128 (got %d)", topk);
  return SAS_OK;
}

float resolve_scale(float scale, int d) { return scale > 0.f ? scale : 1.0f / sqrtf((float)d); }

size_t a16(size_t x) { return (x + 15) & ~(size_t)15; }

}  // namespace

extern "C" {

const char* sas_strerror(sas_status s) {
  switch (s) {
    case SAS_OK: return "ok";
    case SAS_ERR_INVALID_ARG: return "invalid argument";
    case SAS_ERR_UNSUPPORTED: return "unsupported configuration";
    case SAS_ERR_CUDA: return "CUDA error";
    case SAS_ERR_TIMEOUT: return "device wait timed out";
    case SAS_ERR_INTERNAL: return "internal error";
  }
  return "unknown status";
}

const char* sas_last_error_message(void) { return g_last_error.c_str(); }

int sas_version(void) { return 100; }

sas_status sas_block_summary(const void* k, sas_dtype dt, int B, int H, int N, int d,
                             const int32_t* lens, float* ksum, sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_common(dt, B, H, H, N, d, 0);
  if (s != SAS_OK) return s;
  if (B == 0 || N / 64 == 0) return SAS_OK;
  REQUIRE_PTR(k);
  REQUIRE_PTR(ksum);
  if (lens) REQUIRE(aligned16(lens), SAS_ERR_INVALID_ARG, "lens must be 16-byte aligned");
  return cuda_status(sas::launch_block_summary(k, dt == SAS_BF16, B, H, N, d, lens, ksum,
                                               (cudaStream_t)stream),
                     "sas_block_summary launch");
}

sas_status sas_block_summary_ex(const void* k, sas_dtype dt, int B, int H, int N, int d,
                                const int32_t* lens, void* ksum, sas_dtype sum_dt,
                                sas_stream_t stream) {
  g_last_error.clear();
  REQUIRE(sum_dt == SAS_F32 || sum_dt == SAS_BF16, SAS_ERR_INVALID_ARG,
          "summary dtype must be SAS_F32 or SAS_BF16");
  if (sum_dt == SAS_F32)
    return sas_block_summary(k, dt, B, H, N, d, lens, static_cast<float*>(ksum), stream);
  sas_status s = check_common(dt, B, H, H, N, d, 0);
  if (s != SAS_OK) return s;
  if (B == 0 || N / 64 == 0) return SAS_OK;
  REQUIRE_PTR(k);
  REQUIRE_PTR(ksum);
  if (lens) REQUIRE(aligned16(lens), SAS_ERR_INVALID_ARG, "lens must be 16-byte aligned");
  return cuda_status(sas::launch_block_summary_bf16(k, dt == SAS_BF16, B, H, N, d, lens, ksum,
                                                    (cudaStream_t)stream),
                     "sas_block_summary_ex launch");
}

sas_status sas_block_summary_last(const void* k, sas_dtype dt, int B, int H, int N, int d,
                                  const int32_t* lens, void* ksum, sas_dtype sum_dt,
                                  const int32_t* block_table, int npages, sas_stream_t stream) {
  g_last_error.clear();
  REQUIRE(sum_dt == SAS_F32 || sum_dt == SAS_BF16, SAS_ERR_INVALID_ARG,
          "summary dtype must be SAS_F32 or SAS_BF16");
  sas_status s = check_common(dt, B, H, H, N, d, 0);
  if (s != SAS_OK) return s;
  REQUIRE(N % 64 == 0, SAS_ERR_INVALID_ARG, "N must be a multiple of 64 (got %d)", N);
  if (block_table) REQUIRE(npages >= 1, SAS_ERR_INVALID_ARG, "npages must be >= 1 (got %d)", npages);
  if (B == 0 || N < 128) return SAS_OK;
  REQUIRE_PTR(k);
  REQUIRE_PTR(ksum);
  REQUIRE_PTR(lens);
  return cuda_status(sas::launch_summary_last(k, dt == SAS_BF16, B, H, N, d, lens, ksum,
                                              sum_dt == SAS_BF16, block_table, N / 64, npages,
                                              (cudaStream_t)stream),
                     "sas_block_summary_last launch");
}

size_t sas_select_workspace_size(int B, int Hq, int Hkv, int N, int d, int topk, sas_mode mode) {
  if (B <= 0 || Hkv <= 0 || N <= 0 || d <= 0 || topk < 0) return 0;
  if (mode == SAS_PREFILL) return a16(sas::select_prefill_ws_bytes(B, Hkv, N, d));
  const sas::SelectPlan p = sas::plan_decode_select(B, Hkv, N, topk);
  return a16(sizeof(int) * (size_t)B * Hkv) + a16(sas::decode_select_ws_bytes(p));
}

sas_status sas_select(const void* q, sas_dtype dt, const float* ksum, int B, int Hq, int Hkv,
                      int N, int d, int topk, sas_mode mode, const int32_t* lens, float scale,
                      int32_t* idx, int32_t* cnt, float* logg, float* scores_out, void* ws,
                      size_t ws_bytes, sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_common(dt, B, Hq, Hkv, N, d, topk);
  if (s != SAS_OK) return s;
  REQUIRE(mode == SAS_PREFILL || mode == SAS_DECODE, SAS_ERR_INVALID_ARG, "bad mode");
  if (B == 0 || N == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(cnt);
  if (topk > 0) {
    REQUIRE_PTR(idx);
    REQUIRE_PTR(logg);
  }
  if (N / 64 > 0) REQUIRE_PTR(ksum);
  if (scores_out)
    REQUIRE(aligned16(scores_out), SAS_ERR_INVALID_ARG, "scores_out must be 16-byte aligned");
  const size_t need = sas_select_workspace_size(B, Hq, Hkv, N, d, topk, mode);
  REQUIRE(ws_bytes >= need, SAS_ERR_INVALID_ARG, "workspace too small: %zu < %zu", ws_bytes, need);
  REQUIRE_PTR(ws);
  const float sc = resolve_scale(scale, d);
  cudaStream_t st = (cudaStream_t)stream;
  if (mode == SAS_PREFILL) {
    REQUIRE(lens == nullptr, SAS_ERR_INVALID_ARG, "lens must be NULL in prefill mode");
    REQUIRE((N + 63) / 64 - 1 <= 256 * 64, SAS_ERR_UNSUPPORTED, "prefill N too long for selection");
    return cuda_status(sas::launch_select_prefill(q, dt == SAS_BF16, ksum, B, Hq, Hkv, N, d, topk,
                                                  sc, idx, cnt, logg, scores_out, ws, st),
                       "sas_select launch");
  }
  REQUIRE_PTR(lens);
  REQUIRE(N % 64 == 0 && N >= 64, SAS_ERR_INVALID_ARG, "decode needs Lmax a positive multiple of 64");
  REQUIRE(topk > 0 || idx == nullptr || aligned16(idx), SAS_ERR_INVALID_ARG, "idx alignment");
  const sas::SelectPlan p = sas::plan_decode_select(B, Hkv, N, topk);
  int* counters = static_cast<int*>(ws);
  void* rest = static_cast<char*>(ws) + a16(sizeof(int) * (size_t)B * Hkv);
  cudaError_t e = cudaMemsetAsync(counters, 0, sizeof(int) * (size_t)B * Hkv, st);
  if (e != cudaSuccess) return cuda_status(e, "sas_select memset");
  return cuda_status(sas::launch_select_decode(q, dt == SAS_BF16, ksum, B, Hq, Hkv, N, d, topk,
                                               lens, sc, idx, cnt, logg, scores_out, p, counters,
                                               rest, st),
                     "sas_select launch");
}

size_t sas_select_prefill_noalloc_capacity(void) {
  return sas::select_prefill_static_capacity() * sizeof(float);
}

sas_status sas_select_prefill_noalloc(const void* q, sas_dtype dt, const float* ksum, int B,
                                      int Hq, int Hkv, int N, int d, int topk, float scale,
                                      int32_t* idx, int32_t* cnt, float* logg,
                                      sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_common(dt, B, Hq, Hkv, N, d, topk);
  if (s != SAS_OK) return s;
  if (B == 0 || N == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(cnt);
  if (topk > 0) {
    REQUIRE_PTR(idx);
    REQUIRE_PTR(logg);
  }
  if (N / 64 > 0) REQUIRE_PTR(ksum);
  REQUIRE((N + 63) / 64 - 1 <= 256 * 64, SAS_ERR_UNSUPPORTED, "prefill N too long for selection");
  const size_t need = sas::select_prefill_ws_bytes(B, Hkv, N, d);
  const size_t cap = sas_select_prefill_noalloc_capacity();
  REQUIRE(need <= cap, SAS_ERR_UNSUPPORTED,
          "sas_select_prefill_noalloc: B*Hkv*ceil(N/64)*d*4 = %zu bytes of query summaries exceed "
          "the fixed %zu-byte device array; use sas_select with a workspace",
          need, cap);
  return cuda_status(sas::launch_select_prefill_static(q, dt == SAS_BF16, ksum, B, Hq, Hkv, N, d,
                                                       topk, resolve_scale(scale, d), idx, cnt,
                                                       logg, (cudaStream_t)stream),
                     "sas_select_prefill_noalloc launch");
}

size_t sas_attn_fwd_workspace_size(int B, int Hq, int Hkv, int N, int d, int topk, sas_dtype dt) {
  (void)B; (void)Hq; (void)Hkv; (void)N; (void)d; (void)topk; (void)dt;
  return 0;
}

static sas_status check_attn_ptrs(const void* q, const void* k, const void* v, const int32_t* idx,
                                  const int32_t* cnt, const float* logg, int topk) {
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(cnt);
  if (topk > 0) {
    REQUIRE_PTR(idx);
    REQUIRE_PTR(logg);
  }
  return SAS_OK;
}

sas_status sas_attn_fwd(const void* q, const void* k, const void* v, sas_dtype dt, int B, int Hq,
                        int Hkv, int N, int d, const int32_t* idx, const int32_t* cnt,
                        const float* logg, int topk, float scale, void* o, float* lse, void* ws,
                        size_t ws_bytes, sas_stream_t stream) {
  g_last_error.clear();
  (void)ws; (void)ws_bytes;
  sas_status s = check_common(dt, B, Hq, Hkv, N, d, topk);
  if (s != SAS_OK) return s;
  if (B == 0 || N == 0) return SAS_OK;
  s = check_attn_ptrs(q, k, v, idx, cnt, logg, topk);
  if (s != SAS_OK) return s;
  REQUIRE_PTR(o);
  REQUIRE_PTR(lse);
  if (sas::attn_fwd_tc_supported(dt == SAS_BF16, d, Hq, Hkv) && topk > 0)
    return cuda_status(sas::launch_attn_fwd_tc(q, k, v, B, Hq, Hkv, N, idx, cnt, logg, topk,
                                               resolve_scale(scale, d), o, lse,
                                               (cudaStream_t)stream),
                       "sas_attn_fwd launch");
  return cuda_status(sas::launch_attn_fwd_simt(q, k, v, dt == SAS_BF16, B, Hq, Hkv, N, d, idx, cnt,
                                               logg, topk, resolve_scale(scale, d), o, lse,
                                               (cudaStream_t)stream),
                     "sas_attn_fwd launch");
}

size_t sas_attn_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d, int topk, sas_dtype dt) {
  (void)Hq; (void)topk; (void)dt;
  if (B <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return 0;
  return a16(sas::attn_bwd_simt_ws_bytes(B, Hkv, N, d));
}

sas_status sas_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, sas_dtype dt, int B, int Hq, int Hkv, int N, int d,
                        const float* lse, const int32_t* idx, const int32_t* cnt,
                        const float* logg, int topk, float scale, void* dq, void* dk, void* dv,
                        float* dlogg, void* ws, size_t ws_bytes, sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_common(dt, B, Hq, Hkv, N, d, topk);
  if (s != SAS_OK) return s;
  if (B == 0 || N == 0) return SAS_OK;
  s = check_attn_ptrs(q, k, v, idx, cnt, logg, topk);
  if (s != SAS_OK) return s;
  REQUIRE_PTR(o);
  REQUIRE_PTR(dout);
  REQUIRE_PTR(lse);
  REQUIRE_PTR(dq);
  REQUIRE_PTR(dk);
  REQUIRE_PTR(dv);
  if (topk > 0) REQUIRE_PTR(dlogg);
  const size_t need = sas_attn_bwd_workspace_size(B, Hq, Hkv, N, d, topk, dt);
  REQUIRE(ws_bytes >= need, SAS_ERR_INVALID_ARG, "workspace too small: %zu < %zu", ws_bytes, need);
  REQUIRE_PTR(ws);
  if (sas::attn_fwd_tc_supported(dt == SAS_BF16, d, Hq, Hkv) && topk > 0)
    return cuda_status(sas::launch_attn_bwd_tc(q, k, v, o, dout, B, Hq, Hkv, N, lse, idx, cnt,
                                               logg, topk, resolve_scale(scale, d), dq, dk, dv,
                                               dlogg, ws, (cudaStream_t)stream),
                       "sas_attn_bwd launch");
  return cuda_status(sas::launch_attn_bwd_simt(q, k, v, o, dout, dt == SAS_BF16, B, Hq, Hkv, N, d,
                                               lse, idx, cnt, logg, topk, resolve_scale(scale, d),
                                               dq, dk, dv, dlogg, ws, (cudaStream_t)stream),
                     "sas_attn_bwd launch");
}

static sas_status check_decode(sas_dtype dt, int B, int Hq, int Hkv, int Lmax, int d, int topk,
                               int gated) {
  sas_status s = check_common(dt, B, Hq, Hkv, Lmax, d, topk);
  if (s != SAS_OK) return s;
  const int G = Hq / Hkv;
  REQUIRE(G == 1 || G == 2 || G == 4 || G == 8, SAS_ERR_UNSUPPORTED,
          "decode supports 1, 2, 4 or 8 query heads per kv head (got %d)", G);
  REQUIRE(Lmax % 64 == 0 && Lmax >= 64, SAS_ERR_INVALID_ARG, "Lmax must be a positive multiple of 64");
  REQUIRE(gated == 0 || gated == 1, SAS_ERR_INVALID_ARG, "gated must be 0 or 1");
  return SAS_OK;
}

size_t sas_decode_attend_workspace_size(int B, int Hq, int Hkv, int Lmax, int d, int topk) {
  if (B <= 0 || Hkv <= 0 || Lmax <= 0 || d <= 0 || topk < 0) return 0;
  return a16(sizeof(int) * (size_t)B * Hkv) + a16(sas::decode_attend_ws_bytes(B, Hq, Hkv, topk, d));
}

sas_status sas_decode_attend(const void* q, const void* kc, const void* vc, sas_dtype dt, int B,
                             int Hq, int Hkv, int Lmax, int d, const int32_t* lens,
                             const int32_t* idx, const int32_t* cnt, const float* logg, int topk,
                             int gated, float scale, void* o, void* ws, size_t ws_bytes,
                             sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_decode(dt, B, Hq, Hkv, Lmax, d, topk, gated);
  if (s != SAS_OK) return s;
  if (B == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(kc);
  REQUIRE_PTR(vc);
  REQUIRE_PTR(lens);
  REQUIRE_PTR(cnt);
  REQUIRE_PTR(o);
  if (topk > 0) {
    REQUIRE_PTR(idx);
    REQUIRE_PTR(logg);
  }
  const size_t need = sas_decode_attend_workspace_size(B, Hq, Hkv, Lmax, d, topk);
  REQUIRE(ws_bytes >= need, SAS_ERR_INVALID_ARG, "workspace too small: %zu < %zu", ws_bytes, need);
  REQUIRE_PTR(ws);
  cudaStream_t st = (cudaStream_t)stream;
  int* counters = static_cast<int*>(ws);
  cudaError_t e = cudaMemsetAsync(counters, 0, sizeof(int) * (size_t)B * Hkv, st);
  if (e != cudaSuccess) return cuda_status(e, "sas_decode_attend memset");
  e = sas::launch_decode_attend(q, kc, vc, dt == SAS_BF16, B, Hq, Hkv, Lmax, d, lens, idx, cnt,
                                logg, topk, gated, resolve_scale(scale, d), o, counters,
                                static_cast<char*>(ws) + a16(sizeof(int) * (size_t)B * Hkv), st,
                                false);
  return cuda_status(e, "sas_decode_attend launch");
}

size_t sas_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int d, int topk) {
  (void)B; (void)Hq; (void)Hkv; (void)Lmax; (void)d; (void)topk;
  return 0;  // the one-launch cluster kernel keeps everything in shared memory
}

sas_status sas_decode(const void* q, const void* kc, const void* vc, sas_dtype dt, int B, int Hq,
                      int Hkv, int Lmax, int d, const int32_t* lens, const float* ksum, int topk,
                      int gated, float scale, void* o, int32_t* idx_out, void* ws,
                      size_t ws_bytes, sas_stream_t stream) {
  g_last_error.clear();
  (void)ws; (void)ws_bytes;
  sas_status s = check_decode(dt, B, Hq, Hkv, Lmax, d, topk, gated);
  if (s != SAS_OK) return s;
  if (B == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(kc);
  REQUIRE_PTR(vc);
  REQUIRE_PTR(lens);
  REQUIRE_PTR(ksum);
  REQUIRE_PTR(o);
  if (idx_out) REQUIRE(aligned16(idx_out), SAS_ERR_INVALID_ARG, "idx_out must be 16-byte aligned");
  return cuda_status(sas::launch_decode_fused(q, kc, vc, dt == SAS_BF16, B, Hq, Hkv, Lmax, d, lens,
                                              ksum, topk, gated, resolve_scale(scale, d), o,
                                              idx_out, (cudaStream_t)stream),
                     "sas_decode launch");
}

sas_status sas_decode_ex(const void* q, const void* kc, const void* vc, sas_dtype dt, int B,
                         int Hq, int Hkv, int Lmax, int d, const int32_t* lens, const void* ksum,
                         sas_dtype sum_dt, int topk, int gated, float scale, void* o,
                         int32_t* idx_out, sas_stream_t stream) {
  g_last_error.clear();
  REQUIRE(sum_dt == SAS_F32 || sum_dt == SAS_BF16, SAS_ERR_INVALID_ARG,
          "summary dtype must be SAS_F32 or SAS_BF16");
  sas_status s = check_decode(dt, B, Hq, Hkv, Lmax, d, topk, gated);
  if (s != SAS_OK) return s;
  if (B == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(kc);
  REQUIRE_PTR(vc);
  REQUIRE_PTR(lens);
  REQUIRE_PTR(ksum);
  REQUIRE_PTR(o);
  if (idx_out) REQUIRE(aligned16(idx_out), SAS_ERR_INVALID_ARG, "idx_out must be 16-byte aligned");
  return cuda_status(sas::launch_decode_fused_ex(q, kc, vc, dt == SAS_BF16, B, Hq, Hkv, Lmax, d,
                                                 lens, ksum, sum_dt == SAS_BF16, topk, gated,
                                                 resolve_scale(scale, d), o, idx_out,
                                                 (cudaStream_t)stream),
                     "sas_decode_ex launch");
}

// ---------------------------------------------------------------- decode from host buffers
sas_status sas_decode_host(const void* q_host, void* q_dev, const void* kc, const void* vc,
                           sas_dtype dt, int B, int Hq, int Hkv, int Lmax, int d,
                           const int32_t* lens, const float* ksum, int topk, int gated,
                           float scale, void* o_dev, void* o_host, int32_t* idx_out,
                           sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_decode(dt, B, Hq, Hkv, Lmax, d, topk, gated);
  if (s != SAS_OK) return s;
  if (B == 0) return SAS_OK;
  REQUIRE(q_host != nullptr && o_host != nullptr, SAS_ERR_INVALID_ARG,
          "q_host and o_host must not be NULL");
  REQUIRE_PTR(q_dev);
  REQUIRE_PTR(kc);
  REQUIRE_PTR(vc);
  REQUIRE_PTR(lens);
  REQUIRE_PTR(ksum);
  REQUIRE_PTR(o_dev);
  if (idx_out) REQUIRE(aligned16(idx_out), SAS_ERR_INVALID_ARG, "idx_out must be 16-byte aligned");
  const size_t bytes = (size_t)B * Hq * d * (dt == SAS_BF16 ? 2 : 4);
  cudaStream_t st = (cudaStream_t)stream;
  // Page-locked host buffers are addressable from the device (unified
  // addressing): the step then reads q and writes o straight over the bus,
  // with no separate copy; otherwise q is copied into q_dev first and o_dev
  // is copied back. A failed query only means "not page-locked".
  auto mapped = [](const void* p) -> const void* {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      cudaGetLastError();  // clears that query's own error
      return nullptr;
    }
    if (at.type == cudaMemoryTypeHost && at.devicePointer != nullptr && aligned16(at.devicePointer))
      return at.devicePointer;
    return nullptr;
  };
  const void* q_in = mapped(q_host);
  void* o_out = const_cast<void*>(mapped(o_host));
  cudaError_t e = cudaSuccess;
  if (!q_in) {
    e = cudaMemcpyAsync(q_dev, q_host, bytes, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_status(e, "sas_decode_host copy in");
    q_in = q_dev;
  }
  e = sas::launch_decode_fused(q_in, kc, vc, dt == SAS_BF16, B, Hq, Hkv, Lmax, d, lens, ksum,
                               topk, gated, resolve_scale(scale, d), o_out ? o_out : o_dev,
                               idx_out, st);
  if (e != cudaSuccess) return cuda_status(e, "sas_decode_host launch");
  if (o_out) return SAS_OK;
  return cuda_status(cudaMemcpyAsync(o_host, o_dev, bytes, cudaMemcpyDeviceToHost, st),
                     "sas_decode_host copy out");
}

// ---------------------------------------------------------------- paged decode
static sas_status decode_paged_impl(const char* fn, const void* q, const void* kpool,
                                    const void* vpool, const void* kspool, sas_dtype sum_dt,
                                    sas_dtype dt, int B, int Hq, int Hkv, int npages, int d,
                                    const int32_t* block_table, int max_blocks,
                                    const int32_t* lens, int topk, int gated, float scale,
                                    void* o, int32_t* idx_out, sas_stream_t stream) {
  REQUIRE(max_blocks >= 1 && max_blocks <= (1 << 24), SAS_ERR_INVALID_ARG,
          "max_blocks must be in [1, 2^24] (got %d)", max_blocks);
  REQUIRE(sum_dt == SAS_F32 || sum_dt == SAS_BF16, SAS_ERR_INVALID_ARG,
          "summary dtype must be SAS_F32 or SAS_BF16 (got %d)", (int)sum_dt);
  sas_status s = check_decode(dt, B, Hq, Hkv, max_blocks * 64, d, topk, gated);
  if (s != SAS_OK) return s;
  REQUIRE(npages >= 1, SAS_ERR_INVALID_ARG, "npages must be >= 1 (got %d)", npages);
  if (B == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(kpool);
  REQUIRE_PTR(vpool);
  REQUIRE_PTR(kspool);
  REQUIRE_PTR(block_table);
  REQUIRE_PTR(lens);
  REQUIRE_PTR(o);
  if (idx_out) REQUIRE(aligned16(idx_out), SAS_ERR_INVALID_ARG, "idx_out must be 16-byte aligned");
  return cuda_status(sas::launch_decode_paged(q, kpool, vpool, dt == SAS_BF16, B, Hq, Hkv, npages,
                                              d, block_table, max_blocks, lens, kspool,
                                              sum_dt == SAS_BF16, topk, gated,
                                              resolve_scale(scale, d), o, idx_out,
                                              (cudaStream_t)stream),
                     fn);
}

sas_status sas_decode_paged(const void* q, const void* kpool, const void* vpool,
                            const float* kspool, sas_dtype dt, int B, int Hq, int Hkv, int npages,
                            int d, const int32_t* block_table, int max_blocks,
                            const int32_t* lens, int topk, int gated, float scale, void* o,
                            int32_t* idx_out, sas_stream_t stream) {
  g_last_error.clear();
  return decode_paged_impl("sas_decode_paged launch", q, kpool, vpool, kspool, SAS_F32, dt, B,
                           Hq, Hkv, npages, d, block_table, max_blocks, lens, topk, gated, scale,
                           o, idx_out, stream);
}

sas_status sas_decode_paged_ex(const void* q, const void* kpool, const void* vpool,
                               const void* kspool, sas_dtype sum_dt, sas_dtype dt, int B, int Hq,
                               int Hkv, int npages, int d, const int32_t* block_table,
                               int max_blocks, const int32_t* lens, int topk, int gated,
                               float scale, void* o, int32_t* idx_out, sas_stream_t stream) {
  g_last_error.clear();
  return decode_paged_impl("sas_decode_paged_ex launch", q, kpool, vpool, kspool, sum_dt, dt, B,
                           Hq, Hkv, npages, d, block_table, max_blocks, lens, topk, gated, scale,
                           o, idx_out, stream);
}

// ---------------------------------------------------------------- selector backward
size_t sas_select_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d) {
  (void)Hq;
  if (B <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return 0;
  return a16(sas::select_bwd_ws_bytes(B, Hkv, N, d));
}

sas_status sas_select_bwd(const void* q, sas_dtype dt, const float* ksum, int B, int Hq, int Hkv,
                          int N, int d, int topk, float scale, const int32_t* idx,
                          const int32_t* cnt, const float* dlogg, void* dq, void* dk, void* ws,
                          size_t ws_bytes, sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_common(dt, B, Hq, Hkv, N, d, topk);
  if (s != SAS_OK) return s;
  if (B == 0 || N == 0 || topk == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(ksum);
  REQUIRE_PTR(idx);
  REQUIRE_PTR(cnt);
  REQUIRE_PTR(dlogg);
  REQUIRE_PTR(dq);
  REQUIRE_PTR(dk);
  const size_t need = sas_select_bwd_workspace_size(B, Hq, Hkv, N, d);
  REQUIRE(ws_bytes >= need, SAS_ERR_INVALID_ARG, "workspace too small: %zu < %zu", ws_bytes, need);
  REQUIRE_PTR(ws);
  return cuda_status(sas::launch_select_bwd(q, dt == SAS_BF16, ksum, B, Hq, Hkv, N, d, topk,
                                            resolve_scale(scale, d), idx, cnt, dlogg, dq, dk, ws,
                                            (cudaStream_t)stream),
                     "sas_select_bwd launch");
}

// ---------------------------------------------------------------- per-token selection
sas_status sas_select_tokens(const void* q, sas_dtype dt, const float* ksum, int B, int Hq,
                             int Hkv, int N, int d, int topk, float scale, int32_t* idx,
                             int32_t* cnt, float* logg, sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_common(dt, B, Hq, Hkv, N, d, topk);
  if (s != SAS_OK) return s;
  REQUIRE(N <= sas::tokens_max_n(), SAS_ERR_UNSUPPORTED,
          "per-token selection supports N <= %d (got %d)", sas::tokens_max_n(), N);
  if (B == 0 || N == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(cnt);
  if (topk > 0) {
    REQUIRE_PTR(idx);
    REQUIRE_PTR(logg);
  }
  if (N > 64) REQUIRE_PTR(ksum);
  return cuda_status(sas::launch_select_tokens(q, dt == SAS_BF16, ksum, B, Hq, Hkv, N, d, topk,
                                               resolve_scale(scale, d), idx, cnt, logg,
                                               (cudaStream_t)stream),
                     "sas_select_tokens launch");
}

sas_status sas_attn_fwd_tokens(const void* q, const void* k, const void* v, sas_dtype dt, int B,
                               int Hq, int Hkv, int N, int d, const int32_t* idx,
                               const int32_t* cnt, const float* logg, int topk, float scale,
                               void* o, float* lse, sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_common(dt, B, Hq, Hkv, N, d, topk);
  if (s != SAS_OK) return s;
  REQUIRE(N <= sas::tokens_max_n(), SAS_ERR_UNSUPPORTED,
          "per-token attention supports N <= %d (got %d)", sas::tokens_max_n(), N);
  if (B == 0 || N == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(cnt);
  REQUIRE_PTR(o);
  REQUIRE_PTR(lse);
  if (topk > 0) {
    REQUIRE_PTR(idx);
    REQUIRE_PTR(logg);
  }
  if (sas::attn_fwd_tc_supported(dt == SAS_BF16, d, Hq, Hkv) && topk > 0)
    return cuda_status(sas::launch_attn_fwd_tc_tokens(q, k, v, B, Hq, Hkv, N, idx, cnt, logg,
                                                      topk, resolve_scale(scale, d), o, lse,
                                                      (cudaStream_t)stream),
                       "sas_attn_fwd_tokens launch");
  return cuda_status(sas::launch_attn_fwd_tokens(q, k, v, dt == SAS_BF16, B, Hq, Hkv, N, d, idx,
                                                 cnt, logg, topk, resolve_scale(scale, d), o,
                                                 lse, (cudaStream_t)stream),
                     "sas_attn_fwd_tokens launch");
}

size_t sas_attn_bwd_tokens_workspace_size(int B, int Hq, int Hkv, int N, int d) {
  (void)Hq;
  if (B <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return 0;
  return a16(sas::attn_bwd_tokens_ws_bytes(B, Hkv, N, d));
}

sas_status sas_attn_bwd_tokens(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, sas_dtype dt, int B, int Hq, int Hkv, int N,
                               int d, const float* lse, const int32_t* idx, const int32_t* cnt,
                               const float* logg, int topk, float scale, void* dq, void* dk,
                               void* dv, float* dlogg, void* ws, size_t ws_bytes,
                               sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_common(dt, B, Hq, Hkv, N, d, topk);
  if (s != SAS_OK) return s;
  REQUIRE(N <= sas::tokens_max_n(), SAS_ERR_UNSUPPORTED,
          "per-token attention supports N <= %d (got %d)", sas::tokens_max_n(), N);
  if (B == 0 || N == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(k);
  REQUIRE_PTR(v);
  REQUIRE_PTR(o);
  REQUIRE_PTR(dout);
  REQUIRE_PTR(lse);
  REQUIRE_PTR(cnt);
  REQUIRE_PTR(dq);
  REQUIRE_PTR(dk);
  REQUIRE_PTR(dv);
  REQUIRE_PTR(ws);
  if (topk > 0) {
    REQUIRE_PTR(idx);
    REQUIRE_PTR(logg);
    REQUIRE_PTR(dlogg);
  }
  const size_t need = sas_attn_bwd_tokens_workspace_size(B, Hq, Hkv, N, d);
  REQUIRE(ws_bytes >= need, SAS_ERR_INVALID_ARG, "workspace too small (%zu < %zu bytes)",
          ws_bytes, need);
  if (sas::attn_fwd_tc_supported(dt == SAS_BF16, d, Hq, Hkv) && topk > 0)
    return cuda_status(sas::launch_attn_bwd_tc_tokens(q, k, v, o, dout, B, Hq, Hkv, N, lse, idx,
                                                      cnt, logg, topk, resolve_scale(scale, d),
                                                      dq, dk, dv, dlogg, ws,
                                                      (cudaStream_t)stream),
                       "sas_attn_bwd_tokens launch");
  return cuda_status(sas::launch_attn_bwd_tokens(q, k, v, o, dout, dt == SAS_BF16, B, Hq, Hkv, N,
                                                 d, lse, idx, cnt, logg, topk,
                                                 resolve_scale(scale, d), dq, dk, dv, dlogg, ws,
                                                 (cudaStream_t)stream),
                     "sas_attn_bwd_tokens launch");
}

size_t sas_select_bwd_tokens_workspace_size(int B, int Hq, int Hkv, int N, int d) {
  (void)Hq;
  if (B <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return 0;
  return a16(sas::select_bwd_tokens_ws_bytes(B, Hkv, N, d));
}

sas_status sas_select_bwd_tokens(const void* q, sas_dtype dt, const float* ksum, int B, int Hq,
                                 int Hkv, int N, int d, int topk, float scale, const int32_t* idx,
                                 const int32_t* cnt, const float* dlogg, void* dq, void* dk,
                                 void* ws, size_t ws_bytes, sas_stream_t stream) {
  g_last_error.clear();
  sas_status s = check_common(dt, B, Hq, Hkv, N, d, topk);
  if (s != SAS_OK) return s;
  REQUIRE(N <= sas::tokens_max_n(), SAS_ERR_UNSUPPORTED,
          "per-token selector backward supports N <= %d (got %d)", sas::tokens_max_n(), N);
  if (B == 0 || N < 128 || topk == 0) return SAS_OK;
  REQUIRE_PTR(q);
  REQUIRE_PTR(ksum);
  REQUIRE_PTR(idx);
  REQUIRE_PTR(cnt);
  REQUIRE_PTR(dlogg);
  REQUIRE_PTR(dq);
  REQUIRE_PTR(dk);
  const size_t need = sas_select_bwd_tokens_workspace_size(B, Hq, Hkv, N, d);
  REQUIRE(ws_bytes >= need, SAS_ERR_INVALID_ARG, "workspace too small: %zu < %zu", ws_bytes, need);
  REQUIRE_PTR(ws);
  return cuda_status(sas::launch_select_bwd_tokens(q, dt == SAS_BF16, ksum, B, Hq, Hkv, N, d,
                                                   topk, resolve_scale(scale, d), idx, cnt,
                                                   dlogg, dq, dk, ws, (cudaStream_t)stream),
                     "sas_select_bwd_tokens launch");
}

// ---------------------------------------------------------------- device status
sas_status sas_device_status(int clear, sas_stream_t stream) {
  g_last_error.clear();
  struct Word {
    const char* kernel;
    uint32_t* (*addr)();
  };
  static const Word words[] = {
      {"k_decode_fused", sas::decode_fused_error_word},
      {"k_decode_attend", sas::decode_error_word},
      {"k_attn_fwd_tc", sas::attn_fwd_tc_error_word},
      {"k_attn_bwd_tc", sas::attn_bwd_tc_error_word},
      {"k_attn_simt", sas::attn_simt_error_word},
      {"k_wait_selftest", sas::selftest_error_word},
      {"k_summary_last", sas::summary_error_word},
      {"k_attn_*_tokens", sas::tokens_error_word},
  };
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "sas_device_status synchronize");
  std::string msg;
  uint32_t all = 0;
  for (const Word& w : words) {
    uint32_t* p = w.addr();
    if (p == nullptr) return fail(SAS_ERR_CUDA, "sas_device_status: no address for %s", w.kernel);
    uint32_t v = 0;
    e = cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e, "sas_device_status read");
    if (v) {
      if (!msg.empty()) msg += "; ";
      msg += w.kernel;
      if (v & sas::kErrWaitTimeout) msg += ": a bounded wait gave up";
      if (v & sas::kErrBadIndex) msg += (v & sas::kErrWaitTimeout) ? ", " : ": ";
      if (v & sas::kErrBadIndex) msg += "a selection index out of range was replaced";
    }
    all |= v;
    if (clear && v) {
      e = cudaMemset(p, 0, sizeof(uint32_t));
      if (e != cudaSuccess) return cuda_status(e, "sas_device_status clear");
    }
  }
  if (clear) {
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e, "sas_device_status clear");
  }
  if (all & sas::kErrWaitTimeout) return fail(SAS_ERR_TIMEOUT, "%s", msg.c_str());
  if (all) return fail(SAS_ERR_INTERNAL, "%s", msg.c_str());
  return SAS_OK;
}

sas_status sas_debug_wait_timeout(sas_stream_t stream) {
  g_last_error.clear();
  return cuda_status(sas::launch_wait_selftest((cudaStream_t)stream), "sas_debug_wait_timeout");
}

}  // extern "C"
