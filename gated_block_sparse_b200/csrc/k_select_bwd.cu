// Selector backward: the gradient that reaches q and k through the selector.
//
// Method: SAS close reading (liuzhao09.github.io), section 2.3, eq. 8
// (sparse scope): with g = softmax(s) over the C = t visible history blocks
// of query block t and I its kept set,
//   ds_m = dlogg[slot of m] [m in I] - g_m sum_{l in I} dlogg[slot of l],
// i.e. the kept blocks' log-gate gradients pass through the shared
// normalisation log g = s - LSE(s) to every visible block. The selector is
// parameter-free, s_m = scale qbar_t . kbar_m (qbar_t the mean of the group's
// G heads over block t's n_t rows, kbar_m the mean of block m's 64 keys), so
//   dqbar_t = scale sum_m ds_m kbar_m   -> each of those rows and heads gets dqbar_t / (G n_t)
//   dkbar_m = scale sum_t ds_tm qbar_t  -> each of block m's keys gets dkbar_m / 64.
// Both are added into the caller's dq and dk (the attention backward's
// outputs), so the pair of calls gives the full gradient.
//
// Two passes (this work is small next to attention; plain fp32 SIMT):
//   k_select_bwd_rows: one CTA per (t, r, b): scores, gate, ds (kept in
//     workspace as a [T][T] row per (b, r)), dqbar, the add into dq;
//   k_select_bwd_cols: one CTA per (complete key block m, r, b): dkbar_m from
//     the ds column and the query means of blocks t > m, the add into dk.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace sas {

namespace {
constexpr int SB_THREADS = 256;
constexpr int SB_WARPS = SB_THREADS / 32;
}  // namespace

template <typename T, int D>
__global__ void __launch_bounds__(SB_THREADS) k_select_bwd_rows(
    const float* __restrict__ qbar, const float* __restrict__ ksum, int nblk,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
    const float* __restrict__ dlogg, int topk, float scale, int Hq, int Hkv, int N,
    T* __restrict__ dq, float* __restrict__ dsmat) {
  extern __shared__ float sds[];  // scores, then ds, of the row's C blocks
  __shared__ float qb[D], dqb[D], red[SB_WARPS];
  __shared__ float total_s;
  const int t = blockIdx.x, r = blockIdx.y, b = blockIdx.z, T_ = gridDim.x;
  const int C = min(t, nblk);
  if (C == 0) return;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const size_t row = ((size_t)b * Hkv + r) * T_ + t;
  const float* ks = ksum + ((size_t)b * Hkv + r) * nblk * D;
  for (int i = tid; i < D; i += SB_THREADS) qb[i] = qbar[row * D + i];
  __syncthreads();
  // scores s_m = scale qbar . kbar_m, one warp per block
  for (int m = wid; m < C; m += SB_WARPS) {
    float a = 0.f;
    for (int i = lane; i < D; i += 32) a += qb[i] * ks[(size_t)m * D + i];
    a = warp_sum(a);
    if (lane == 0) sds[m] = a * scale;
  }
  __syncthreads();
  // gate: max and sum of exp over the C blocks
  float mx = -FLT_MAX;
  for (int m = tid; m < C; m += SB_THREADS) mx = fmaxf(mx, sds[m]);
  mx = warp_max(mx);
  if (lane == 0) red[wid] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < SB_WARPS; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float se = 0.f;
  for (int m = tid; m < C; m += SB_THREADS) se += __expf(sds[m] - mx);
  se = warp_sum(se);
  if (lane == 0) red[wid] = se;
  const int kk = min(max(cnt[row], 0), topk);
  if (wid == 0) {  // sum of the kept slots' gradients
    float a = 0.f;
    for (int j = lane; j < kk; j += 32) a += dlogg[row * topk + j];
    a = warp_sum(a);
    if (lane == 0) total_s = a;
  }
  __syncthreads();
  float S = 0.f;
  for (int w = 0; w < SB_WARPS; ++w) S += red[w];
  const float total = total_s;
  for (int m = tid; m < C; m += SB_THREADS) sds[m] = -(__expf(sds[m] - mx) / S) * total;
  __syncthreads();
  for (int j = tid; j < kk; j += SB_THREADS) {  // the kept blocks' own term
    const int m = idx[row * topk + j];
    if (m >= 0 && m < C) atomicAdd(&sds[m], dlogg[row * topk + j]);
  }
  __syncthreads();
  for (int m = tid; m < C; m += SB_THREADS) dsmat[row * T_ + m] = sds[m];
  // dqbar = scale sum_m ds_m kbar_m (one column per thread, coalesced summaries)
  for (int col = tid; col < D; col += SB_THREADS) {
    float a0 = 0.f, a1 = 0.f;
    int m = 0;
    for (; m + 1 < C; m += 2) {
      a0 += sds[m] * ks[(size_t)m * D + col];
      a1 += sds[m + 1] * ks[(size_t)(m + 1) * D + col];
    }
    if (m < C) a0 += sds[m] * ks[(size_t)m * D + col];
    dqb[col] = (a0 + a1) * scale;
  }
  __syncthreads();
  // spread over the block's rows and the group's heads: dq += dqbar / (G n_t)
  constexpr int VEC = Vec16<T>::N;
  const int G = Hq / Hkv, r0 = t * SAS_BLOCK, nt = min(SAS_BLOCK, N - r0);
  const float w = 1.0f / (float)(G * nt);
  const int per_row = D / VEC, nchunk = G * nt * per_row;
  for (int e = tid; e < nchunk; e += SB_THREADS) {
    const int h = e / (nt * per_row), rem = e - h * nt * per_row;
    const int i = rem / per_row, c = (rem - i * per_row) * VEC;
    T* p = dq + (((size_t)b * Hq + r * G + h) * N + r0 + i) * D + c;
    float x[VEC];
    Vec16<T>::load(p, x);
#pragma unroll
    for (int u = 0; u < VEC; ++u) x[u] += dqb[c + u] * w;
    Vec16<T>::store(p, x);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(D) k_select_bwd_cols(const float* __restrict__ qbar,
                                                        const float* __restrict__ dsmat, int T_,
                                                        float scale, int Hkv, int N,
                                                        T* __restrict__ dk) {
  const int m = blockIdx.x, r = blockIdx.y, b = blockIdx.z, col = threadIdx.x;
  const size_t base = ((size_t)b * Hkv + r) * T_;
  float a0 = 0.f, a1 = 0.f;
  int t = m + 1;
  for (; t + 1 < T_; t += 2) {
    a0 += dsmat[(base + t) * T_ + m] * qbar[(base + t) * D + col];
    a1 += dsmat[(base + t + 1) * T_ + m] * qbar[(base + t + 1) * D + col];
  }
  if (t < T_) a0 += dsmat[(base + t) * T_ + m] * qbar[(base + t) * D + col];
  const float add = (a0 + a1) * scale / (float)SAS_BLOCK;
  T* p = dk + (((size_t)b * Hkv + r) * N + (size_t)m * SAS_BLOCK) * D + col;
  for (int j = 0; j < SAS_BLOCK; ++j) p[(size_t)j * D] = from_f<T>(to_f(p[(size_t)j * D]) + add);
}

size_t select_bwd_ws_bytes(int B, int Hkv, int N, int d) {
  const size_t T_ = (size_t)(N + SAS_BLOCK - 1) / SAS_BLOCK;
  return (size_t)B * Hkv * T_ * d * 4 + (size_t)B * Hkv * T_ * T_ * 4;
}

template <typename T, int D>
static cudaError_t select_bwd_t(const float* qbar, const float* ksum, int B, int Hq, int Hkv,
                                int N, int topk, float scale, const int32_t* idx,
                                const int32_t* cnt, const float* dlogg, void* dq, void* dk,
                                float* dsmat, cudaStream_t st) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK, nblk = N / SAS_BLOCK;
  const size_t smem = (size_t)T_ * 4;
  cudaError_t e = ensure_smem(k_select_bwd_rows<T, D>, smem);
  if (e != cudaSuccess) return e;
  k_select_bwd_rows<T, D><<<dim3(T_, Hkv, B), SB_THREADS, smem, st>>>(
      qbar, ksum, nblk, idx, cnt, dlogg, topk, scale, Hq, Hkv, N, static_cast<T*>(dq), dsmat);
  e = cudaGetLastError();
  if (e != cudaSuccess || nblk == 0) return e;
  k_select_bwd_cols<T, D><<<dim3(nblk, Hkv, B), D, 0, st>>>(qbar, dsmat, T_, scale, Hkv, N,
                                                           static_cast<T*>(dk));
  return cudaGetLastError();
}

cudaError_t launch_select_bwd(const void* q, int bf16, const float* ksum, int B, int Hq, int Hkv,
                              int N, int d, int topk, float scale, const int32_t* idx,
                              const int32_t* cnt, const float* dlogg, void* dq, void* dk,
                              void* ws, cudaStream_t st) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK;
  if (B == 0 || T_ < 2 || topk == 0) return cudaSuccess;  // no history block anywhere
  float* qbar = static_cast<float*>(ws);
  float* dsmat = qbar + (size_t)B * Hkv * T_ * d;
  cudaError_t e = launch_qbar_prefill(q, bf16, B, Hq, Hkv, N, d, qbar, st);
  if (e != cudaSuccess) return e;
  if (bf16)
    return d == 128 ? select_bwd_t<__nv_bfloat16, 128>(qbar, ksum, B, Hq, Hkv, N, topk, scale,
                                                       idx, cnt, dlogg, dq, dk, dsmat, st)
                    : select_bwd_t<__nv_bfloat16, 64>(qbar, ksum, B, Hq, Hkv, N, topk, scale,
                                                      idx, cnt, dlogg, dq, dk, dsmat, st);
  return d == 128 ? select_bwd_t<float, 128>(qbar, ksum, B, Hq, Hkv, N, topk, scale, idx, cnt,
                                             dlogg, dq, dk, dsmat, st)
                  : select_bwd_t<float, 64>(qbar, ksum, B, Hq, Hkv, N, topk, scale, idx, cnt,
                                            dlogg, dq, dk, dsmat, st);
}

}  // namespace sas
