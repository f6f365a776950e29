// Gated sparse attention, prefill forward and backward on the CUDA cores
// (fp32 FMA). Used for fp32 inputs, where tensor cores would miss a 1e-4
// tolerance, and as a reference-shaped path for bf16.
//
// Definitions (SAS close reading, liuzhao09.github.io, sections 2.1, 2.2 and
// 2.4; SAS reproduction note, daiwk.github.io, core formula):
//   z_ij = scale * q_i . k_j + log g of j's block (0 in the current block),
//   keys: the kept history blocks of query block t, then the current block
//   with j <= i; o = softmax(z) V; lse = log sum exp z.
//   Backward: D_i = dO_i . o_i, dz = p (dO V^T - D), dq = scale dz K,
//   dk = scale dz^T Q, dv = p^T dO, dlogg[t][slot] = sum of dz over the slot's
//   64 keys, the block's rows and the group's heads.
//
// One CTA per (query block t, head h, sequence b), 256 threads. Thread
// (tr, tc) = (tid / 16, tid % 16) holds rows tr + 16*ii and keys tc + 16*jj
// (ii, jj < 4) of each 64 x 64 score tile, and rows tr + 16*ii x columns
// 4*tc + 64*g of the 64 x d output tile. Tiles live in shared memory as fp32
// with a row stride of d + 4 floats, so that the 16-byte row reads of a
// quarter warp fall in distinct banks. Unselected blocks are never visited.
#include <float.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "simt_tile.cuh"

namespace sas {

__device__ uint32_t g_attn_simt_err = 0;

// Unit u of query block t's key list: the kept history blocks, then the
// current block. Returns the block index, its bias, or -1 for an invalid
// entry (skipped and reported).
__device__ __forceinline__ int unit_block(int u, int kk, int t, const int32_t* idx_row,
                                          const float* logg_row, float* bias) {
  if (u == kk) {
    *bias = 0.f;
    return t;
  }
  const int m = idx_row[u];
  if (m < 0 || m >= t) {
    atomicOr(&g_attn_simt_err, kErrBadIndex);
    return -1;
  }
  *bias = logg_row[u];
  return m;
}

template <typename T, int D>
__global__ void __launch_bounds__(AT_THREADS) k_attn_fwd_simt(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, int Hq, int Hkv,
    int N, const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
    const float* __restrict__ logg, int topk, float scale, T* __restrict__ o,
    float* __restrict__ lse) {
  using S = AtShape<D>;
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;
  float* Ks = Qs + S::TILE;
  float* Vs = Ks + S::TILE;
  float* Ps = Vs + S::TILE;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z, T_ = gridDim.x;
  const int G = Hq / Hkv, r = h / G;
  const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15;
  const int row0 = t * SAS_BLOCK, nr = min(SAS_BLOCK, N - row0);
  const size_t srow = ((size_t)b * Hkv + r) * T_ + t;
  const int kk = min(max(cnt[srow], 0), topk);
  const int32_t* idx_row = idx + srow * topk;
  const float* logg_row = logg + srow * topk;
  const T* kbase = k + ((size_t)b * Hkv + r) * N * D;
  const T* vbase = v + ((size_t)b * Hkv + r) * N * D;

  load_tile<T, D>(Qs, q + (((size_t)b * Hq + h) * N + row0) * D, nr);
  float acc[4][S::NG][4];
  float m_i[4], l_i[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m_i[i] = -INFINITY;
    l_i[i] = 0.f;
#pragma unroll
    for (int g = 0; g < S::NG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][g][e] = 0.f;
  }
  for (int u = 0; u <= kk; ++u) {
    float bias;
    const int blk = unit_block(u, kk, t, idx_row, logg_row, &bias);
    if (blk < 0) continue;
    const bool cur = (u == kk);
    const int nvalid = cur ? nr : SAS_BLOCK;
    __syncthreads();  // previous unit done with Ks/Vs/Ps
    load_tile<T, D>(Ks, kbase + (size_t)blk * SAS_BLOCK * D, nvalid);
    load_tile<T, D>(Vs, vbase + (size_t)blk * SAS_BLOCK * D, nvalid);
    __syncthreads();
    float s[4][4];
    tile_dot<D>(Qs, Ks, tr, tc, s);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ri = tr + 16 * i;
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kj = tc + 16 * j;
        float z = s[i][j] * scale + bias;
        if (cur && kj > ri) z = -INFINITY;
        s[i][j] = z;
        mx = fmaxf(mx, z);
      }
      mx = half_max(mx);
      const float mn = fmaxf(m_i[i], mx);
      const float alpha = __expf(m_i[i] - mn);
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float p = __expf(s[i][j] - mn);
        rs += p;
        Ps[ri * S::PLD + tc + 16 * j] = p;
      }
      rs = half_sum(rs);
      l_i[i] = l_i[i] * alpha + rs;
      m_i[i] = mn;
#pragma unroll
      for (int g = 0; g < S::NG; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[i][g][e] *= alpha;
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < SAS_BLOCK; ++j) {
      float pj[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) pj[i] = Ps[(tr + 16 * i) * S::PLD + j];
#pragma unroll
      for (int g = 0; g < S::NG; ++g) {
        const float4 vv = *reinterpret_cast<const float4*>(Vs + j * S::LD + 4 * tc + 64 * g);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i][g][0] += pj[i] * vv.x;
          acc[i][g][1] += pj[i] * vv.y;
          acc[i][g][2] += pj[i] * vv.z;
          acc[i][g][3] += pj[i] * vv.w;
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ri = tr + 16 * i;
    if (ri >= nr) continue;
    const float inv = 1.f / l_i[i];
    T* orow = o + (((size_t)b * Hq + h) * N + row0 + ri) * D;
#pragma unroll
    for (int g = 0; g < S::NG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) orow[4 * tc + 64 * g + e] = from_f<T>(acc[i][g][e] * inv);
    if (tc == 0) lse[((size_t)b * Hq + h) * N + row0 + ri] = m_i[i] + __logf(l_i[i]);
  }
}

// ------------------------------------------------------------------ backward
template <typename T, int D>
__global__ void __launch_bounds__(AT_THREADS) k_attn_bwd_simt(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const T* __restrict__ o, const T* __restrict__ dout, int Hq, int Hkv, int N,
    const float* __restrict__ lse, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ cnt, const float* __restrict__ logg, int topk, float scale,
    T* __restrict__ dq, float* __restrict__ dk_acc, float* __restrict__ dv_acc,
    float* __restrict__ dlogg) {
  using S = AtShape<D>;
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;
  float* dOs = Qs + S::TILE;
  float* Ks = dOs + S::TILE;
  float* Vs = Ks + S::TILE;
  float* Ps = Vs + S::TILE;
  float* dSs = Ps + SAS_BLOCK * S::PLD;
  __shared__ float Drow[SAS_BLOCK], Lrow[SAS_BLOCK];
  __shared__ float red[AT_THREADS / 32];
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z, T_ = gridDim.x;
  const int G = Hq / Hkv, r = h / G;
  const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15;
  const int lane = tid & 31, wid = tid >> 5;
  const int row0 = t * SAS_BLOCK, nr = min(SAS_BLOCK, N - row0);
  const size_t srow = ((size_t)b * Hkv + r) * T_ + t;
  const int kk = min(max(cnt[srow], 0), topk);
  const int32_t* idx_row = idx + srow * topk;
  const float* logg_row = logg + srow * topk;
  const size_t kvoff = ((size_t)b * Hkv + r) * N * D;
  const size_t qoff = (((size_t)b * Hq + h) * N + row0) * D;

  load_tile<T, D>(Qs, q + qoff, nr);
  load_tile<T, D>(dOs, dout + qoff, nr);
  // D_i = dO_i . o_i (8 lanes per row) and the forward's lse.
  for (int rr = tid >> 3; rr < SAS_BLOCK; rr += AT_THREADS / 8) {
    float a = 0.f;
    if (rr < nr) {
      const T* orow = o + qoff + (size_t)rr * D;
      for (int c = (tid & 7); c < D; c += 8) a += to_f(orow[c]) * to_f(dout[qoff + (size_t)rr * D + c]);
    }
    a += __shfl_xor_sync(0xffffffffu, a, 1);
    a += __shfl_xor_sync(0xffffffffu, a, 2);
    a += __shfl_xor_sync(0xffffffffu, a, 4);
    if ((tid & 7) == 0) {
      Drow[rr] = a;
      Lrow[rr] = rr < nr ? lse[((size_t)b * Hq + h) * N + row0 + rr] : 0.f;
    }
  }
  float dqa[4][S::NG][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int g = 0; g < S::NG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) dqa[i][g][e] = 0.f;

  for (int u = 0; u <= kk; ++u) {
    float bias;
    const int blk = unit_block(u, kk, t, idx_row, logg_row, &bias);
    if (blk < 0) continue;
    const bool cur = (u == kk);
    const int nvalid = cur ? nr : SAS_BLOCK;
    __syncthreads();
    load_tile<T, D>(Ks, k + kvoff + (size_t)blk * SAS_BLOCK * D, nvalid);
    load_tile<T, D>(Vs, v + kvoff + (size_t)blk * SAS_BLOCK * D, nvalid);
    __syncthreads();
    float s[4][4], dp[4][4];
    tile_dot<D>(Qs, Ks, tr, tc, s);
    tile_dot<D>(dOs, Vs, tr, tc, dp);
    float dsum = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ri = tr + 16 * i;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kj = tc + 16 * j;
        float p = __expf(s[i][j] * scale + bias - Lrow[ri]);
        if ((cur && kj > ri) || ri >= nr) p = 0.f;
        const float ds = p * (dp[i][j] - Drow[ri]);
        Ps[ri * S::PLD + kj] = p;
        dSs[ri * S::PLD + kj] = ds;
        dsum += ds;
      }
    }
    if (!cur) {  // d(log g) of this slot: the tile's sum of logit gradients
      dsum = warp_sum(dsum);
      if (lane == 0) red[wid] = dsum;
    }
    __syncthreads();
    if (!cur && tid == 0) {
      float a = 0.f;
      for (int i = 0; i < AT_THREADS / 32; ++i) a += red[i];
      atomicAdd(dlogg + srow * topk + u, a);
    }
    // dQ += dS K
#pragma unroll 4
    for (int j = 0; j < SAS_BLOCK; ++j) {
      float dsj[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) dsj[i] = dSs[(tr + 16 * i) * S::PLD + j];
#pragma unroll
      for (int g = 0; g < S::NG; ++g) {
        const float4 kv = *reinterpret_cast<const float4*>(Ks + j * S::LD + 4 * tc + 64 * g);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          dqa[i][g][0] += dsj[i] * kv.x;
          dqa[i][g][1] += dsj[i] * kv.y;
          dqa[i][g][2] += dsj[i] * kv.z;
          dqa[i][g][3] += dsj[i] * kv.w;
        }
      }
    }
    // dK[j] += scale sum_i dS[i][j] Q[i];  dV[j] += sum_i P[i][j] dO[i]
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const float* W = pass == 0 ? dSs : Ps;
      const float* X = pass == 0 ? Qs : dOs;
      float* dst = pass == 0 ? dk_acc : dv_acc;
      const float f = pass == 0 ? scale : 1.f;
      float a[4][S::NG][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int g = 0; g < S::NG; ++g)
#pragma unroll
          for (int e = 0; e < 4; ++e) a[i][g][e] = 0.f;
#pragma unroll 4
      for (int i2 = 0; i2 < SAS_BLOCK; ++i2) {
        float wj[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) wj[jj] = W[i2 * S::PLD + tr + 16 * jj];
#pragma unroll
        for (int g = 0; g < S::NG; ++g) {
          const float4 xv = *reinterpret_cast<const float4*>(X + i2 * S::LD + 4 * tc + 64 * g);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            a[jj][g][0] += wj[jj] * xv.x;
            a[jj][g][1] += wj[jj] * xv.y;
            a[jj][g][2] += wj[jj] * xv.z;
            a[jj][g][3] += wj[jj] * xv.w;
          }
        }
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int kj = tr + 16 * jj;
        if (kj >= nvalid) continue;
        float* drow = dst + kvoff + ((size_t)blk * SAS_BLOCK + kj) * D;
#pragma unroll
        for (int g = 0; g < S::NG; ++g)
          atomicAdd(reinterpret_cast<float4*>(drow + 4 * tc + 64 * g),
                    make_float4(a[jj][g][0] * f, a[jj][g][1] * f, a[jj][g][2] * f, a[jj][g][3] * f));
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ri = tr + 16 * i;
    if (ri >= nr) continue;
    T* drow = dq + qoff + (size_t)ri * D;
#pragma unroll
    for (int g = 0; g < S::NG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) drow[4 * tc + 64 * g + e] = from_f<T>(dqa[i][g][e] * scale);
  }
}

template <typename T>
__global__ void k_convert(const float* __restrict__ src, T* __restrict__ dst, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = from_f<T>(src[i]);
}

template <int D> static size_t fwd_smem() { return sizeof(float) * (3 * AtShape<D>::TILE + SAS_BLOCK * AtShape<D>::PLD); }
template <int D> static size_t bwd_smem() { return sizeof(float) * (4 * AtShape<D>::TILE + 2 * SAS_BLOCK * AtShape<D>::PLD); }

cudaError_t launch_attn_fwd_simt(const void* q, const void* k, const void* v, int bf16, int B,
                                 int Hq, int Hkv, int N, int d, const int32_t* idx,
                                 const int32_t* cnt, const float* logg, int topk, float scale,
                                 void* o, float* lse, cudaStream_t st) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK;
  if (B == 0 || T_ == 0 || Hq == 0) return cudaSuccess;
  dim3 grid(T_, Hq, B);
#define SAS_FWD(TT, DD)                                                                        \
  do {                                                                                         \
    auto kern = k_attn_fwd_simt<TT, DD>;                                                       \
    const size_t sm = fwd_smem<DD>();                                                          \
    ensure_smem(kern, sm);                                                                     \
    kern<<<grid, AT_THREADS, sm, st>>>(static_cast<const TT*>(q), static_cast<const TT*>(k),   \
                                       static_cast<const TT*>(v), Hq, Hkv, N, idx, cnt, logg,  \
                                       topk, scale, static_cast<TT*>(o), lse);                 \
  } while (0)
  if (bf16) {
    if (d == 128) SAS_FWD(__nv_bfloat16, 128); else SAS_FWD(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_FWD(float, 128); else SAS_FWD(float, 64);
  }
#undef SAS_FWD
  return cudaGetLastError();
}

size_t attn_bwd_simt_ws_bytes(int B, int Hkv, int N, int d) {
  return 2 * (size_t)B * Hkv * N * d * sizeof(float);
}

cudaError_t launch_attn_bwd_simt(const void* q, const void* k, const void* v, const void* o,
                                 const void* dout, int bf16, int B, int Hq, int Hkv, int N, int d,
                                 const float* lse, const int32_t* idx, const int32_t* cnt,
                                 const float* logg, int topk, float scale, void* dq, void* dk,
                                 void* dv, float* dlogg, void* ws, cudaStream_t st) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK;
  if (B == 0 || T_ == 0 || Hq == 0) return cudaSuccess;
  const size_t nkv = (size_t)B * Hkv * N * d;
  float* dk_acc = static_cast<float*>(ws);
  float* dv_acc = dk_acc + nkv;
  cudaError_t e = cudaMemsetAsync(ws, 0, 2 * nkv * sizeof(float), st);
  if (e != cudaSuccess) return e;
  if (topk > 0) {
    e = cudaMemsetAsync(dlogg, 0, (size_t)B * Hkv * T_ * topk * sizeof(float), st);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(T_, Hq, B);
  const int cgrid = (int)((nkv + 255) / 256 < 4096 ? (nkv + 255) / 256 : 4096);
#define SAS_BWD(TT, DD)                                                                       \
  do {                                                                                        \
    auto kern = k_attn_bwd_simt<TT, DD>;                                                      \
    const size_t sm = bwd_smem<DD>();                                                         \
    ensure_smem(kern, sm);                                                                    \
    kern<<<grid, AT_THREADS, sm, st>>>(                                                       \
        static_cast<const TT*>(q), static_cast<const TT*>(k), static_cast<const TT*>(v),      \
        static_cast<const TT*>(o), static_cast<const TT*>(dout), Hq, Hkv, N, lse, idx, cnt,   \
        logg, topk, scale, static_cast<TT*>(dq), dk_acc, dv_acc, dlogg);                      \
    k_convert<TT><<<cgrid, 256, 0, st>>>(dk_acc, static_cast<TT*>(dk), nkv);                  \
    k_convert<TT><<<cgrid, 256, 0, st>>>(dv_acc, static_cast<TT*>(dv), nkv);                  \
  } while (0)
  if (bf16) {
    if (d == 128) SAS_BWD(__nv_bfloat16, 128); else SAS_BWD(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_BWD(float, 128); else SAS_BWD(float, 64);
  }
#undef SAS_BWD
  return cudaGetLastError();
}

uint32_t* attn_simt_error_word() {
  void* p = nullptr;
  cudaGetSymbolAddress(&p, g_attn_simt_err);
  return static_cast<uint32_t*>(p);
}

}  // namespace sas
