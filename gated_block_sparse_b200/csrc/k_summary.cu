// Block summaries: the mean of each complete 64-key block (SAS close reading,
// liuzhao09.github.io, section 2.1: a block summary compresses the block's
// adjacent keys and is what the selector reads).
//
// One CTA per (block m, head h, sequence b); 256 threads. Each thread loads
// 16-byte vectors of one key row and accumulates fp32 column sums; the row
// groups are reduced through shared memory. HBM-bound: every key is read
// once, 4 bytes per column are written per block (2 with bf16 summaries,
// the fp32 mean rounded to nearest even).
#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace sas {

template <typename T, int D, typename S>
__global__ void __launch_bounds__(256) k_block_summary(const T* __restrict__ k, int N, int nblk,
                                                       const int32_t* __restrict__ lens,
                                                       S* __restrict__ ksum) {
  constexpr int VEC = Vec16<T>::N;
  constexpr int TPR = D / VEC;   // threads per key row
  constexpr int RP = 256 / TPR;  // key rows per pass
  __shared__ float red[RP][D];
  const int m = blockIdx.x, h = blockIdx.y, b = blockIdx.z, H = gridDim.y;
  const int tid = threadIdx.x, c = tid % TPR, rg = tid / TPR;
  int nvalid = nblk;
  if (lens) nvalid = min(nblk, lens[b] / SAS_BLOCK);
  const T* base = k + (((size_t)b * H + h) * N + (size_t)m * SAS_BLOCK) * D + c * VEC;
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
  if (m < nvalid) {
#pragma unroll
    for (int r = rg; r < SAS_BLOCK; r += RP) {
      float x[VEC];
      Vec16<T>::load_nc(base + (size_t)r * D, x);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc[i] += x[i];
    }
  }
#pragma unroll
  for (int i = 0; i < VEC; ++i) red[rg][c * VEC + i] = acc[i];
  __syncthreads();
  S* out = ksum + (((size_t)b * H + h) * nblk + m) * D;
  for (int col = tid; col < D; col += 256) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < RP; ++r) s += red[r][col];
    out[col] = from_f<S>((m < nvalid) ? s * (1.0f / SAS_BLOCK) : 0.f);
  }
}

template <typename S>
static cudaError_t block_summary_s(const void* k, int bf16, int B, int H, int N, int d,
                                   const int32_t* lens, S* ksum, cudaStream_t st) {
  const int nblk = N / SAS_BLOCK;
  if (nblk == 0 || B == 0 || H == 0) return cudaSuccess;
  dim3 grid(nblk, H, B);
#define SAS_SUM(T, D) \
  k_block_summary<T, D, S><<<grid, 256, 0, st>>>(static_cast<const T*>(k), N, nblk, lens, ksum)
  if (bf16) {
    if (d == 128) SAS_SUM(__nv_bfloat16, 128); else SAS_SUM(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_SUM(float, 128); else SAS_SUM(float, 64);
  }
#undef SAS_SUM
  return cudaGetLastError();
}

cudaError_t launch_block_summary(const void* k, int bf16, int B, int H, int N, int d,
                                 const int32_t* lens, float* ksum, cudaStream_t st) {
  return block_summary_s<float>(k, bf16, B, H, N, d, lens, ksum, st);
}

cudaError_t launch_block_summary_bf16(const void* k, int bf16, int B, int H, int N, int d,
                                      const int32_t* lens, void* ksum, cudaStream_t st) {
  return block_summary_s<__nv_bfloat16>(k, bf16, B, H, N, d, lens,
                                        static_cast<__nv_bfloat16*>(ksum), st);
}

// Summary upkeep during decode: the summary of block C - 1 of every
// (sequence, head), the last complete block before the current one
// (C = (lens[b] - 1) / 64), the block that completed when the current one
// began. One CTA per (head, sequence); nothing is written when C = 0.
// PAGED: k is a pool [npages][H][64][D] and ksum [npages][H][D], the block's
// page read from bt [B][max_blocks] (an entry outside [0, npages) skips the
// row and sets kErrBadIndex in the error word).
template <typename T, int D, typename S, bool PAGED>
__global__ void __launch_bounds__(256) k_summary_last(const T* __restrict__ k, int N,
                                                      const int32_t* __restrict__ lens,
                                                      S* __restrict__ ksum,
                                                      const int32_t* __restrict__ bt,
                                                      int max_blocks, int npages,
                                                      uint32_t* err) {
  constexpr int VEC = Vec16<T>::N;
  constexpr int TPR = D / VEC;
  constexpr int RP = 256 / TPR;
  __shared__ float red[RP][D];
  const int h = blockIdx.x, b = blockIdx.y, H = gridDim.x;
  const int tid = threadIdx.x, c = tid % TPR, rg = tid / TPR;
  const int n = min(max(lens[b], 1), N);
  const int m = (n - 1) / SAS_BLOCK - 1;
  if (m < 0) return;
  const T* base;
  S* out;
  if constexpr (PAGED) {
    const int p = bt[(size_t)b * max_blocks + m];
    if (p < 0 || p >= npages) {
      if (tid == 0) atomicOr(err, kErrBadIndex);
      return;
    }
    base = k + ((size_t)p * H + h) * SAS_BLOCK * D + c * VEC;
    out = ksum + ((size_t)p * H + h) * D;
  } else {
    base = k + (((size_t)b * H + h) * N + (size_t)m * SAS_BLOCK) * D + c * VEC;
    out = ksum + (((size_t)b * H + h) * (N / SAS_BLOCK) + m) * D;
  }
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
#pragma unroll
  for (int r = rg; r < SAS_BLOCK; r += RP) {
    float x[VEC];
    Vec16<T>::load_nc(base + (size_t)r * D, x);
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] += x[i];
  }
#pragma unroll
  for (int i = 0; i < VEC; ++i) red[rg][c * VEC + i] = acc[i];
  __syncthreads();
  for (int col = tid; col < D; col += 256) {
    float s2 = 0.f;
#pragma unroll
    for (int r = 0; r < RP; ++r) s2 += red[r][col];
    out[col] = from_f<S>(s2 * (1.0f / SAS_BLOCK));
  }
}

__device__ uint32_t g_summary_err = 0;

template <typename S, bool PAGED>
static cudaError_t summary_last_s(const void* k, int bf16, int B, int H, int N, int d,
                                  const int32_t* lens, S* ksum, const int32_t* bt,
                                  int max_blocks, int npages, cudaStream_t st) {
  if (B == 0 || H == 0 || N < 2 * SAS_BLOCK) return cudaSuccess;
  uint32_t* err = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_summary_err);
  if (e != cudaSuccess) return e;
  dim3 grid(H, B);
#define SAS_LAST(T, D)                                                                     \
  k_summary_last<T, D, S, PAGED><<<grid, 256, 0, st>>>(static_cast<const T*>(k), N, lens, \
                                                       ksum, bt, max_blocks, npages, err)
  if (bf16) {
    if (d == 128) SAS_LAST(__nv_bfloat16, 128); else SAS_LAST(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_LAST(float, 128); else SAS_LAST(float, 64);
  }
#undef SAS_LAST
  return cudaGetLastError();
}

cudaError_t launch_summary_last(const void* k, int bf16, int B, int H, int N, int d,
                                const int32_t* lens, void* ksum, int sum_bf16,
                                const int32_t* bt, int max_blocks, int npages,
                                cudaStream_t st) {
  if (bt) {
    if (sum_bf16)
      return summary_last_s<__nv_bfloat16, true>(k, bf16, B, H, N, d, lens,
                                                 static_cast<__nv_bfloat16*>(ksum), bt,
                                                 max_blocks, npages, st);
    return summary_last_s<float, true>(k, bf16, B, H, N, d, lens, static_cast<float*>(ksum), bt,
                                       max_blocks, npages, st);
  }
  if (sum_bf16)
    return summary_last_s<__nv_bfloat16, false>(k, bf16, B, H, N, d, lens,
                                                static_cast<__nv_bfloat16*>(ksum), nullptr, 0, 0,
                                                st);
  return summary_last_s<float, false>(k, bf16, B, H, N, d, lens, static_cast<float*>(ksum),
                                      nullptr, 0, 0, st);
}

uint32_t* summary_error_word() {
  void* p = nullptr;
  cudaGetSymbolAddress(&p, g_summary_err);
  return static_cast<uint32_t*>(p);
}

}  // namespace sas
