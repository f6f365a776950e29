// Per-token selection prefill on the CUDA cores (fp32). SAS close reading,
// liuzhao09.github.io, section 2.4: the fused kernel masks, per query, the
// blocks below that query's gate threshold, and skips a key tile no query of
// the tile selected. Each query token i of kv group r selects its own blocks:
// qbar_i = mean of the group's G heads at token i, scores
// s_m = scale * qbar_i . kbar_m over its C = i / 64 history blocks, the gate
// log g = s - LSE(s) and Top-K with ties to the lower block index (sections
// 2.1 and 2.2). Every head of the group attends over its token's own set.
//
// Selection: one CTA per (query block t, kv group r, sequence b) scores its
// 64 token means against the C = t summaries (64 x 64 tiles, fp32), then one
// warp per row takes the row's gate and its Top-K by a bitwise search for the
// k-th largest score.
// Attention: one CTA per (query block, head, sequence) walks the union of the
// blocks its rows selected (built from the rows' lists in shared memory),
// then the current block. Each row finds its bias for a unit by walking its
// own ascending list: log g where it selected the unit's block, -inf
// elsewhere. The backward sums each row's logit gradients over a selected
// unit into that row's slot.
#include <float.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "simt_tile.cuh"

namespace sas {

__device__ uint32_t g_tokens_err = 0;

constexpr int TOK_CMAX = 512;  // history blocks of a query block at most

// ------------------------------------------------------------------ selection
// Order-preserving unsigned key of a score: a larger score has a larger key,
// and -0 was mapped to +0 before, so equal scores have equal keys.
__device__ __forceinline__ uint32_t score_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}

// One warp: the gate and the Top-K of one row's C scores si[0 .. C) (C <= 32
// KPL). kk = min(topk, C) blocks are kept, ordered by (score desc, block
// asc): tau, the kk-th largest key, is found bit by bit (the largest value
// with at least kk keys at or above it); the keys above tau are kept, and of
// the keys equal to tau the lowest-numbered ones until kk are reached. The
// kept blocks and their log g = s - LSE(s) are written in ascending block
// order, the rest of the row padded with -1 / 0.
template <int KPL>
__device__ __forceinline__ void select_row(const float* si, int C, int kk, int topk,
                                           int32_t* __restrict__ idx_row,
                                           float* __restrict__ logg_row,
                                           int32_t* __restrict__ cnt_row) {
  const int lane = threadIdx.x & 31;
  float sv[KPL];
  uint32_t kv[KPL];
  float mx = -FLT_MAX;
#pragma unroll
  for (int j = 0; j < KPL; ++j) {
    const int m = j * 32 + lane;
    sv[j] = m < C ? si[m] : -FLT_MAX;
    kv[j] = m < C ? score_key(sv[j]) : 0u;
    mx = fmaxf(mx, sv[j]);
  }
  mx = warp_max(mx);
  float z = 0.f;
#pragma unroll
  for (int j = 0; j < KPL; ++j)
    if (j * 32 + lane < C) z += __expf(sv[j] - mx);
  z = warp_sum(z);
  const float lse_i = mx + __logf(z);
  uint32_t tau = 0u;  // keys of m >= C are 0 and every real key is above 0
  if (kk > 0 && kk < C) {
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      int n = 0;
#pragma unroll
      for (int j = 0; j < KPL; ++j) n += kv[j] >= cand;
      if ((int)__reduce_add_sync(0xffffffffu, (unsigned)n) >= kk) tau = cand;
    }
  }
  int above = 0;
#pragma unroll
  for (int j = 0; j < KPL; ++j) above += (j * 32 + lane < C) && kv[j] > tau;
  above = (int)__reduce_add_sync(0xffffffffu, (unsigned)above);
  const int need = kk > 0 ? kk - above : 0;  // keys equal to tau still to keep
  int ties = 0, pos = 0;
#pragma unroll
  for (int j = 0; j < KPL; ++j) {
    const int m = j * 32 + lane;
    const bool in = m < C && kk > 0;
    const bool eq = in && kv[j] == tau;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const int tr = ties + __popc(eqb & ((1u << lane) - 1u));
    ties += __popc(eqb);
    const bool sel = in && (kv[j] > tau || (eq && tr < need));
    const unsigned bal = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int p = pos + __popc(bal & ((1u << lane) - 1u));
      if (p < topk) {
        idx_row[p] = m;
        logg_row[p] = sv[j] - lse_i;
      }
    }
    pos += __popc(bal);
  }
  pos = min(pos, topk);
  for (int p = pos + lane; p < topk; p += 32) {
    idx_row[p] = -1;
    logg_row[p] = 0.f;
  }
  if (lane == 0) *cnt_row = pos;
}

template <typename T, int D>
__global__ void __launch_bounds__(AT_THREADS) k_select_tokens(
    const T* __restrict__ q, const float* __restrict__ ksum, int Hq, int Hkv, int N, int topk,
    float scale, int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
    float* __restrict__ logg) {
  using S = AtShape<D>;
  extern __shared__ __align__(16) float sm[];
  float* Qb = sm;            // [64][LD] the rows' query means
  float* Kb = Qb + S::TILE;  // [64][LD] 64 summaries
  float* sc = Kb + S::TILE;  // [64][C + 1] scores
  const int t = blockIdx.x, r = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv, nblk = N / SAS_BLOCK;
  const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15, wid = tid >> 5;
  const int row0 = t * SAS_BLOCK, nr = min(SAS_BLOCK, N - row0);
  const int C = t, CP = t + 1;
  for (int e = tid; e < SAS_BLOCK * D; e += AT_THREADS) {
    const int i = e / D, c = e % D;
    float a = 0.f;
    if (i < nr)
      for (int g = 0; g < G; ++g)
        a += to_f(q[(((size_t)b * Hq + r * G + g) * N + row0 + i) * D + c]);
    Qb[i * S::LD + c] = a / (float)G;
  }
  const float* krow = ksum + ((size_t)b * Hkv + r) * (size_t)nblk * D;
  for (int m0 = 0; m0 < C; m0 += SAS_BLOCK) {
    __syncthreads();  // Qb written; the previous chunk's Kb consumed
    for (int e = tid; e < SAS_BLOCK * D; e += AT_THREADS) {
      const int jj = e / D, c = e % D;
      Kb[jj * S::LD + c] = (m0 + jj < C) ? krow[(size_t)(m0 + jj) * D + c] : 0.f;
    }
    __syncthreads();
    float s[4][4];
    tile_dot<D>(Qb, Kb, tr, tc, s);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int m = m0 + tc + 16 * j;
        if (m < C) sc[(tr + 16 * i) * CP + m] = s[i][j] * scale + 0.0f;  // -0 -> +0
      }
  }
  __syncthreads();
  const int kk = min(topk, C);
  for (int i = wid; i < nr; i += AT_THREADS / 32) {
    const size_t orow = ((size_t)b * Hkv + r) * N + row0 + i;
    if (C <= 256) select_row<8>(sc + i * CP, C, kk, topk, idx + orow * topk, logg + orow * topk,
                                cnt + orow);
    else select_row<TOK_CMAX / 32>(sc + i * CP, C, kk, topk, idx + orow * topk,
                                   logg + orow * topk, cnt + orow);
  }
}

// ------------------------------------------------------------------ attention
// Union of the blocks the nr rows of this query block selected (rows' lists
// at idx + (rbase + i) * topk, cnt[rbase + i] entries), ascending, into
// ulist; returns its length. Entries outside [0, C) are skipped and
// reported. All threads call it; it ends with a barrier.
__device__ inline int build_union(const int32_t* __restrict__ idx,
                                  const int32_t* __restrict__ cnt, size_t rbase, int nr,
                                  int topk, int C, uint32_t* umask, int16_t* ulist,
                                  int* ucnt) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int words = (C + 31) / 32;
  for (int w = tid; w < words; w += blockDim.x) umask[w] = 0u;
  __syncthreads();
  for (int e = tid; e < nr * topk; e += blockDim.x) {
    const int i = e / topk, p = e - i * topk;
    if (p < min(max(cnt[rbase + i], 0), topk)) {
      const int m = idx[(rbase + i) * topk + p];
      if (m >= 0 && m < C) atomicOr(&umask[m >> 5], 1u << (m & 31));
      else atomicOr(&g_tokens_err, kErrBadIndex);
    }
  }
  __syncthreads();
  if (tid < 32) {
    int base = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      uint32_t word = w < words ? umask[w] : 0u;
      const int c = __popc(word);
      int off = c;  // inclusive scan over the lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, off, o);
        if (lane >= o) off += y;
      }
      int at = base + off - c;
      while (word) {
        const int bit = __ffs(word) - 1;
        ulist[at++] = (int16_t)(w * 32 + bit);
        word &= word - 1u;
      }
      base += __shfl_sync(0xffffffffu, off, 31);
    }
    if (lane == 0) *ucnt = base;
  }
  __syncthreads();
  return *ucnt;
}

// Bias of unit block blk for one row: log g of the row's slot holding blk,
// -inf when the row did not select it. The row's list is ascending and the
// units come in ascending order, so *ptr only moves forward.
__device__ __forceinline__ float row_bias(const int32_t* __restrict__ ri_idx,
                                          const float* __restrict__ ri_logg, int n, int blk,
                                          int* ptr) {
  int p = *ptr;
  while (p < n && ri_idx[p] < blk) ++p;
  *ptr = p;
  return (p < n && ri_idx[p] == blk) ? ri_logg[p] : -INFINITY;
}

template <typename T, int D>
__global__ void __launch_bounds__(AT_THREADS) k_attn_fwd_tokens(
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
  __shared__ uint32_t umask[TOK_CMAX / 32];
  __shared__ int16_t ulist[TOK_CMAX];
  __shared__ int ucnt;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv, r = h / G;
  const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15;
  const int row0 = t * SAS_BLOCK, nr = min(SAS_BLOCK, N - row0);
  const size_t rbase = ((size_t)b * Hkv + r) * N + row0;
  const T* kbase = k + ((size_t)b * Hkv + r) * N * D;
  const T* vbase = v + ((size_t)b * Hkv + r) * N * D;
  const int U = build_union(idx, cnt, rbase, nr, topk, t, umask, ulist, &ucnt);

  load_tile<T, D>(Qs, q + (((size_t)b * Hq + h) * N + row0) * D, nr);
  float acc[4][S::NG][4];
  float m_i[4], l_i[4];
  int ptr[4], nsel[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ri = tr + 16 * i;
    m_i[i] = -INFINITY;
    l_i[i] = 0.f;
    ptr[i] = 0;
    nsel[i] = ri < nr ? min(max(cnt[rbase + ri], 0), topk) : 0;
#pragma unroll
    for (int g = 0; g < S::NG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][g][e] = 0.f;
  }
  for (int u = 0; u <= U; ++u) {
    const bool cur = (u == U);
    const int blk = cur ? t : ulist[u];
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
      const float bias = cur ? 0.f
                             : row_bias(idx + (rbase + ri) * topk, logg + (rbase + ri) * topk,
                                        nsel[i], blk, &ptr[i]);
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
      const bool none = (mn == -INFINITY);  // nothing visible to this row yet
      const float alpha = none ? 1.f : __expf(m_i[i] - mn);
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float p = none ? 0.f : __expf(s[i][j] - mn);
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

template <typename T, int D>
__global__ void __launch_bounds__(AT_THREADS) k_attn_bwd_tokens(
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
  __shared__ uint32_t umask[TOK_CMAX / 32];
  __shared__ int16_t ulist[TOK_CMAX];
  __shared__ int ucnt;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = Hq / Hkv, r = h / G;
  const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15;
  const int row0 = t * SAS_BLOCK, nr = min(SAS_BLOCK, N - row0);
  const size_t rbase = ((size_t)b * Hkv + r) * N + row0;
  const size_t kvoff = ((size_t)b * Hkv + r) * N * D;
  const size_t qoff = (((size_t)b * Hq + h) * N + row0) * D;
  const int U = build_union(idx, cnt, rbase, nr, topk, t, umask, ulist, &ucnt);

  load_tile<T, D>(Qs, q + qoff, nr);
  load_tile<T, D>(dOs, dout + qoff, nr);
  // D_i = dO_i . o_i (8 lanes per row) and the forward's lse
  for (int rr = tid >> 3; rr < SAS_BLOCK; rr += AT_THREADS / 8) {
    float a = 0.f;
    if (rr < nr) {
      const T* orow = o + qoff + (size_t)rr * D;
      for (int c = (tid & 7); c < D; c += 8)
        a += to_f(orow[c]) * to_f(dout[qoff + (size_t)rr * D + c]);
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
  int ptr[4], nsel[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ri = tr + 16 * i;
    ptr[i] = 0;
    nsel[i] = ri < nr ? min(max(cnt[rbase + ri], 0), topk) : 0;
#pragma unroll
    for (int g = 0; g < S::NG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) dqa[i][g][e] = 0.f;
  }

  for (int u = 0; u <= U; ++u) {
    const bool cur = (u == U);
    const int blk = cur ? t : ulist[u];
    const int nvalid = cur ? nr : SAS_BLOCK;
    __syncthreads();
    load_tile<T, D>(Ks, k + kvoff + (size_t)blk * SAS_BLOCK * D, nvalid);
    load_tile<T, D>(Vs, v + kvoff + (size_t)blk * SAS_BLOCK * D, nvalid);
    __syncthreads();
    float s[4][4], dp[4][4];
    tile_dot<D>(Qs, Ks, tr, tc, s);
    tile_dot<D>(dOs, Vs, tr, tc, dp);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ri = tr + 16 * i;
      const float bias = cur ? 0.f
                             : row_bias(idx + (rbase + ri) * topk, logg + (rbase + ri) * topk,
                                        nsel[i], blk, &ptr[i]);
      float dsum = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kj = tc + 16 * j;
        float p = __expf(s[i][j] * scale + bias - Lrow[ri]);
        if ((cur && kj > ri) || ri >= nr || bias == -INFINITY) p = 0.f;
        const float ds = p * (dp[i][j] - Drow[ri]);
        Ps[ri * S::PLD + kj] = p;
        dSs[ri * S::PLD + kj] = ds;
        dsum += ds;
      }
      // d(log g) of this row's slot for the unit: its logit gradients summed
      // over the unit's keys (the group's heads add into the same slot)
      dsum = half_sum(dsum);
      if (!cur && tc == 0 && ri < nr && bias != -INFINITY)
        atomicAdd(dlogg + (rbase + ri) * topk + ptr[i], dsum);
    }
    __syncthreads();
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
                    make_float4(a[jj][g][0] * f, a[jj][g][1] * f, a[jj][g][2] * f,
                                a[jj][g][3] * f));
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
__global__ void k_convert_tokens(const float* __restrict__ src, T* __restrict__ dst, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = from_f<T>(src[i]);
}

// ------------------------------------------------------------------ host
int tokens_max_n() { return (TOK_CMAX + 1) * SAS_BLOCK; }

template <int D> static size_t tok_sel_smem(int C) {
  return sizeof(float) * (2 * AtShape<D>::TILE + (size_t)SAS_BLOCK * (C + 1));
}
template <int D> static size_t tok_fwd_smem() {
  return sizeof(float) * (3 * AtShape<D>::TILE + SAS_BLOCK * AtShape<D>::PLD);
}
template <int D> static size_t tok_bwd_smem() {
  return sizeof(float) * (4 * AtShape<D>::TILE + 2 * SAS_BLOCK * AtShape<D>::PLD);
}

cudaError_t launch_select_tokens(const void* q, int bf16, const float* ksum, int B, int Hq,
                                 int Hkv, int N, int d, int topk, float scale, int32_t* idx,
                                 int32_t* cnt, float* logg, cudaStream_t st) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK;
  if (B == 0 || T_ == 0) return cudaSuccess;
  dim3 grid(T_, Hkv, B);
#define SAS_TSEL(TT, DD)                                                                       \
  do {                                                                                         \
    auto kern = k_select_tokens<TT, DD>;                                                       \
    const size_t smb = tok_sel_smem<DD>(T_ - 1);                                               \
    cudaError_t e2 = ensure_smem(kern, smb);                                                   \
    if (e2 != cudaSuccess) return e2;                                                          \
    kern<<<grid, AT_THREADS, smb, st>>>(static_cast<const TT*>(q), ksum, Hq, Hkv, N, topk,     \
                                        scale, idx, cnt, logg);                                \
  } while (0)
  if (bf16) {
    if (d == 128) SAS_TSEL(__nv_bfloat16, 128); else SAS_TSEL(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_TSEL(float, 128); else SAS_TSEL(float, 64);
  }
#undef SAS_TSEL
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_tokens(const void* q, const void* k, const void* v, int bf16, int B,
                                   int Hq, int Hkv, int N, int d, const int32_t* idx,
                                   const int32_t* cnt, const float* logg, int topk, float scale,
                                   void* o, float* lse, cudaStream_t st) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK;
  if (B == 0 || T_ == 0) return cudaSuccess;
  dim3 grid(T_, Hq, B);
#define SAS_TFWD(TT, DD)                                                                       \
  do {                                                                                         \
    auto kern = k_attn_fwd_tokens<TT, DD>;                                                     \
    const size_t smb = tok_fwd_smem<DD>();                                                     \
    cudaError_t e2 = ensure_smem(kern, smb);                                                   \
    if (e2 != cudaSuccess) return e2;                                                          \
    kern<<<grid, AT_THREADS, smb, st>>>(static_cast<const TT*>(q), static_cast<const TT*>(k),  \
                                        static_cast<const TT*>(v), Hq, Hkv, N, idx, cnt, logg, \
                                        topk, scale, static_cast<TT*>(o), lse);                \
  } while (0)
  if (bf16) {
    if (d == 128) SAS_TFWD(__nv_bfloat16, 128); else SAS_TFWD(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_TFWD(float, 128); else SAS_TFWD(float, 64);
  }
#undef SAS_TFWD
  return cudaGetLastError();
}

size_t attn_bwd_tokens_ws_bytes(int B, int Hkv, int N, int d) {
  return 2 * (size_t)B * Hkv * N * d * sizeof(float);
}

cudaError_t launch_attn_bwd_tokens(const void* q, const void* k, const void* v, const void* o,
                                   const void* dout, int bf16, int B, int Hq, int Hkv, int N,
                                   int d, const float* lse, const int32_t* idx,
                                   const int32_t* cnt, const float* logg, int topk, float scale,
                                   void* dq, void* dk, void* dv, float* dlogg, void* ws,
                                   cudaStream_t st) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK;
  if (B == 0 || T_ == 0) return cudaSuccess;
  const size_t nkv = (size_t)B * Hkv * N * d;
  float* dk_acc = static_cast<float*>(ws);
  float* dv_acc = dk_acc + nkv;
  cudaError_t e = cudaMemsetAsync(ws, 0, 2 * nkv * sizeof(float), st);
  if (e != cudaSuccess) return e;
  if (topk > 0) {
    e = cudaMemsetAsync(dlogg, 0, (size_t)B * Hkv * N * topk * sizeof(float), st);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(T_, Hq, B);
  const int cgrid = (int)((nkv + 255) / 256 < 4096 ? (nkv + 255) / 256 : 4096);
#define SAS_TBWD(TT, DD)                                                                      \
  do {                                                                                        \
    auto kern = k_attn_bwd_tokens<TT, DD>;                                                    \
    const size_t smb = tok_bwd_smem<DD>();                                                    \
    cudaError_t e2 = ensure_smem(kern, smb);                                                  \
    if (e2 != cudaSuccess) return e2;                                                         \
    kern<<<grid, AT_THREADS, smb, st>>>(                                                      \
        static_cast<const TT*>(q), static_cast<const TT*>(k), static_cast<const TT*>(v),      \
        static_cast<const TT*>(o), static_cast<const TT*>(dout), Hq, Hkv, N, lse, idx, cnt,   \
        logg, topk, scale, static_cast<TT*>(dq), dk_acc, dv_acc, dlogg);                      \
    k_convert_tokens<TT><<<cgrid, 256, 0, st>>>(dk_acc, static_cast<TT*>(dk), nkv);           \
    k_convert_tokens<TT><<<cgrid, 256, 0, st>>>(dv_acc, static_cast<TT*>(dv), nkv);           \
  } while (0)
  if (bf16) {
    if (d == 128) SAS_TBWD(__nv_bfloat16, 128); else SAS_TBWD(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_TBWD(float, 128); else SAS_TBWD(float, 64);
  }
#undef SAS_TBWD
  return cudaGetLastError();
}

// ------------------------------------------------------------------ selector backward
// fp32 -> tf32 (round to nearest) and one m16n8k8 tf32 warp MMA (c += a b,
// fp32 accumulation). Fragments: a0 = A[g][t], a1 = A[g + 8][t], a2 =
// A[g][t + 4], a3 = A[g + 8][t + 4]; b0 = B[t][g], b1 = B[t + 4][g]; c0, c1 =
// C[g][2t], C[g][2t + 1], c2, c3 = C[g + 8][2t], C[g + 8][2t + 1], with
// g = lane / 4, t = lane % 4.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void mma_tf32(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Eq. 8 (section 2.3, sparse scope) for per-token rows: for token i of kv
// group r with C = i / 64, kept set I_i and g = softmax(s_i),
//   ds_m = dlogg[slot of m] [m in I_i] - g_m sum_{l in I_i} dlogg[slot of l];
// through s_m = scale qbar_i . kbar_m, every head of the group gets
// scale sum_m ds_m kbar_m / G at token i (added into dq) and block m's
// summary gets scale sum_i ds_im qbar_i (accumulated in dkbar; a second
// kernel adds dkbar_m / 64 into each of block m's 64 keys of dk).
// One CTA per (query block t, kv group r, sequence b): the rows' query means
// and scores as in k_select_tokens, the gate and ds per row (one warp per
// row), then dqbar = ds kbar over 64-block chunks and each chunk's
// ds^T qbar added into dkbar. The three tile products run on the CUDA cores
// in fp32 for fp32 inputs, and as tf32 warp MMAs (fp32 accumulation) for bf16
// inputs, whose outputs are stored in bf16: each warp takes a 16-row slice
// (warp % 4) and half of the columns (warp / 4) of every 64 x 64 or 64 x d
// product.
template <typename T, int D>
__global__ void __launch_bounds__(AT_THREADS) k_select_bwd_tokens(
    const T* __restrict__ q, const float* __restrict__ ksum, int Hq, int Hkv, int N, int topk,
    float scale, const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
    const float* __restrict__ dlogg, T* __restrict__ dq, float* __restrict__ dkbar) {
  using S = AtShape<D>;
  extern __shared__ __align__(16) float sm[];
  float* Qb = sm;            // [64][LD] the rows' query means
  float* Kb = Qb + S::TILE;  // [64][LD] 64 summaries
  float* sc = Kb + S::TILE;  // [64][C + 1] scores, then ds
  constexpr bool TC = std::is_same<T, __nv_bfloat16>::value;
  constexpr int NT2 = D / 16;  // 8-column tiles of half of d (tensor-core path)
  const int t = blockIdx.x, r = blockIdx.y, b = blockIdx.z;
  const int C = t, CP = t + 1;
  if (C == 0) return;  // no history: the selector has no gradient here
  const int G = Hq / Hkv, nblk = N / SAS_BLOCK;
  const int tid = threadIdx.x, tr = tid >> 4, tc = tid & 15, lane = tid & 31, wid = tid >> 5;
  const int row0 = t * SAS_BLOCK, nr = min(SAS_BLOCK, N - row0);
  const int g8 = lane >> 2, t4 = lane & 3, mi = wid & 3, hw = wid >> 2;  // tensor-core path
  for (int e = tid; e < SAS_BLOCK * D; e += AT_THREADS) {
    const int i = e / D, c = e % D;
    float a = 0.f;
    if (i < nr)
      for (int g = 0; g < G; ++g)
        a += to_f(q[(((size_t)b * Hq + r * G + g) * N + row0 + i) * D + c]);
    Qb[i * S::LD + c] = a / (float)G;
  }
  const float* krow = ksum + ((size_t)b * Hkv + r) * (size_t)nblk * D;
  for (int m0 = 0; m0 < C; m0 += SAS_BLOCK) {
    __syncthreads();  // Qb written; the previous chunk's Kb consumed
    for (int e = tid; e < SAS_BLOCK * D; e += AT_THREADS) {
      const int jj = e / D, c = e % D;
      Kb[jj * S::LD + c] = (m0 + jj < C) ? krow[(size_t)(m0 + jj) * D + c] : 0.f;
    }
    __syncthreads();
    if constexpr (TC) {
      // rows 16 mi + g8 (+8) x summaries m0 + 32 hw + 8 nt + 2 t4 (+1)
      float c4[4][4] = {};
#pragma unroll 4
      for (int k0 = 0; k0 < D; k0 += 8) {
        const float* qa = Qb + (16 * mi + g8) * S::LD + k0 + t4;
        const uint32_t a0 = to_tf32(qa[0]), a1 = to_tf32(qa[8 * S::LD]), a2 = to_tf32(qa[4]),
                       a3 = to_tf32(qa[8 * S::LD + 4]);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          const float* kb = Kb + (32 * hw + 8 * nt + g8) * S::LD + k0 + t4;
          mma_tf32(c4[nt], a0, a1, a2, a3, to_tf32(kb[0]), to_tf32(kb[4]));
        }
      }
      const int row = 16 * mi + g8;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int m = m0 + 32 * hw + 8 * nt + 2 * t4;
        if (m < C) {
          sc[row * CP + m] = c4[nt][0] * scale;
          sc[(row + 8) * CP + m] = c4[nt][2] * scale;
        }
        if (m + 1 < C) {
          sc[row * CP + m + 1] = c4[nt][1] * scale;
          sc[(row + 8) * CP + m + 1] = c4[nt][3] * scale;
        }
      }
    } else {
      float s[4][4];
      tile_dot<D>(Qb, Kb, tr, tc, s);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int m = m0 + tc + 16 * j;
          if (m < C) sc[(tr + 16 * i) * CP + m] = s[i][j] * scale;
        }
    }
  }
  __syncthreads();
  // ds per row (one warp per row); rows past the sequence end get ds = 0
  for (int i = wid; i < SAS_BLOCK; i += AT_THREADS / 32) {
    float* si = sc + i * CP;
    if (i >= nr) {
      for (int m = lane; m < C; m += 32) si[m] = 0.f;
      continue;
    }
    const size_t orow = ((size_t)b * Hkv + r) * N + row0 + i;
    const int kk = min(max(cnt[orow], 0), topk);
    float mx = -FLT_MAX;
    for (int m = lane; m < C; m += 32) mx = fmaxf(mx, si[m]);
    mx = warp_max(mx);
    float z = 0.f;
    for (int m = lane; m < C; m += 32) z += __expf(si[m] - mx);
    z = warp_sum(z);
    float tot = 0.f;
    for (int j = lane; j < kk; j += 32) tot += dlogg[orow * topk + j];
    tot = warp_sum(tot);
    const float f = tot / z;
    for (int m = lane; m < C; m += 32) si[m] = -__expf(si[m] - mx) * f;
    __syncwarp();
    for (int j = lane; j < kk; j += 32) {  // kept blocks are distinct: no two lanes share m
      const int m = idx[orow * topk + j];
      if (m >= 0 && m < C) si[m] += dlogg[orow * topk + j];
      else atomicOr(&g_tokens_err, kErrBadIndex);
    }
  }
  float dqa[4][S::NG][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int g = 0; g < S::NG; ++g)
#pragma unroll
      for (int e = 0; e < 4; ++e) dqa[i][g][e] = 0.f;
  // tensor-core path: rows 16 mi + g8 (+8) x columns (d / 2) hw + 8 nt + 2 t4 (+1)
  float dqc[NT2][4] = {};
  float* dkb = dkbar + ((size_t)b * Hkv + r) * (size_t)nblk * D;
  for (int m0 = 0; m0 < C; m0 += SAS_BLOCK) {
    __syncthreads();  // ds written; the previous chunk's Kb consumed
    const int nm = min(SAS_BLOCK, C - m0);
    for (int e = tid; e < SAS_BLOCK * D; e += AT_THREADS) {
      const int jj = e / D, c = e % D;
      Kb[jj * S::LD + c] = (jj < nm) ? krow[(size_t)(m0 + jj) * D + c] : 0.f;
    }
    __syncthreads();
    if constexpr (TC) {
      // dqbar[rows] += ds[rows][m0 + m] kbar[m], m over the chunk
#pragma unroll 2
      for (int k0 = 0; k0 < SAS_BLOCK; k0 += 8) {
        const int ka = m0 + k0 + t4;
        const float* da = sc + (16 * mi + g8) * CP;
        const uint32_t a0 = to_tf32(ka < C ? da[ka] : 0.f);
        const uint32_t a1 = to_tf32(ka < C ? da[8 * CP + ka] : 0.f);
        const uint32_t a2 = to_tf32(ka + 4 < C ? da[ka + 4] : 0.f);
        const uint32_t a3 = to_tf32(ka + 4 < C ? da[8 * CP + ka + 4] : 0.f);
#pragma unroll
        for (int nt = 0; nt < NT2; ++nt) {
          const float* kb = Kb + (k0 + t4) * S::LD + (D / 2) * hw + 8 * nt + g8;
          mma_tf32(dqc[nt], a0, a1, a2, a3, to_tf32(kb[0]), to_tf32(kb[4 * S::LD]));
        }
      }
      // dkbar[m0 + m] += scale sum_rows ds[row][m0 + m] qbar[row]
      float dkc[NT2][4] = {};
      const int mm = m0 + 16 * mi + g8;
#pragma unroll 2
      for (int k0 = 0; k0 < SAS_BLOCK; k0 += 8) {
        const float* da = sc + (k0 + t4) * CP;
        const uint32_t a0 = to_tf32(mm < C ? da[mm] : 0.f);
        const uint32_t a1 = to_tf32(mm + 8 < C ? da[mm + 8] : 0.f);
        const uint32_t a2 = to_tf32(mm < C ? da[4 * CP + mm] : 0.f);
        const uint32_t a3 = to_tf32(mm + 8 < C ? da[4 * CP + mm + 8] : 0.f);
#pragma unroll
        for (int nt = 0; nt < NT2; ++nt) {
          const float* qb = Qb + (k0 + t4) * S::LD + (D / 2) * hw + 8 * nt + g8;
          mma_tf32(dkc[nt], a0, a1, a2, a3, to_tf32(qb[0]), to_tf32(qb[4 * S::LD]));
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT2; ++nt) {
        const int col = (D / 2) * hw + 8 * nt + 2 * t4;
        if (mm < C)
          atomicAdd(reinterpret_cast<float2*>(dkb + (size_t)mm * D + col),
                    make_float2(dkc[nt][0] * scale, dkc[nt][1] * scale));
        if (mm + 8 < C)
          atomicAdd(reinterpret_cast<float2*>(dkb + (size_t)(mm + 8) * D + col),
                    make_float2(dkc[nt][2] * scale, dkc[nt][3] * scale));
      }
    } else {
      // dqbar[i] += sum_m ds[i][m] kbar_m
#pragma unroll 4
      for (int j = 0; j < nm; ++j) {
        float dsj[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) dsj[i] = sc[(tr + 16 * i) * CP + m0 + j];
#pragma unroll
        for (int g = 0; g < S::NG; ++g) {
          const float4 kv = *reinterpret_cast<const float4*>(Kb + j * S::LD + 4 * tc + 64 * g);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dqa[i][g][0] += dsj[i] * kv.x;
            dqa[i][g][1] += dsj[i] * kv.y;
            dqa[i][g][2] += dsj[i] * kv.z;
            dqa[i][g][3] += dsj[i] * kv.w;
          }
        }
      }
      // dkbar[m] += scale sum_i ds[i][m] qbar_i (rows m = tr + 16 jj of the chunk)
      float a[4][S::NG][4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
#pragma unroll
        for (int g = 0; g < S::NG; ++g)
#pragma unroll
          for (int e = 0; e < 4; ++e) a[jj][g][e] = 0.f;
#pragma unroll 4
      for (int i2 = 0; i2 < nr; ++i2) {
        float wj[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int m = tr + 16 * jj;
          wj[jj] = m < nm ? sc[i2 * CP + m0 + m] : 0.f;
        }
#pragma unroll
        for (int g = 0; g < S::NG; ++g) {
          const float4 xv = *reinterpret_cast<const float4*>(Qb + i2 * S::LD + 4 * tc + 64 * g);
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
        const int m = tr + 16 * jj;
        if (m >= nm) continue;
        float* drow = dkb + (size_t)(m0 + m) * D;
#pragma unroll
        for (int g = 0; g < S::NG; ++g)
          atomicAdd(reinterpret_cast<float4*>(drow + 4 * tc + 64 * g),
                    make_float4(a[jj][g][0] * scale, a[jj][g][1] * scale, a[jj][g][2] * scale,
                                a[jj][g][3] * scale));
      }
    }
  }
  const float fq = scale / (float)G;
  if constexpr (TC) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int ri = 16 * mi + g8 + 8 * hf;
      if (ri >= nr) continue;
      for (int g = 0; g < G; ++g) {
        T* drow = dq + (((size_t)b * Hq + r * G + g) * N + row0 + ri) * D;
#pragma unroll
        for (int nt = 0; nt < NT2; ++nt) {
          __nv_bfloat162* p2 =
              reinterpret_cast<__nv_bfloat162*>(drow + (D / 2) * hw + 8 * nt + 2 * t4);
          float2 v = __bfloat1622float2(*p2);
          v.x += dqc[nt][2 * hf] * fq;
          v.y += dqc[nt][2 * hf + 1] * fq;
          *p2 = __float22bfloat162_rn(v);
        }
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ri = tr + 16 * i;
      if (ri >= nr) continue;
      for (int g = 0; g < G; ++g) {
        T* drow = dq + (((size_t)b * Hq + r * G + g) * N + row0 + ri) * D;
#pragma unroll
        for (int gg = 0; gg < S::NG; ++gg)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * tc + 64 * gg + e;
            drow[c] = from_f<T>(to_f(drow[c]) + dqa[i][gg][e] * fq);
          }
      }
    }
  }
}

// dk[b, r, 64 m + j] += dkbar[b, r, m] / 64 for every complete block m.
template <typename T, int D>
__global__ void __launch_bounds__(256) k_spread_dkbar(const float* __restrict__ dkbar, int Hkv,
                                                      int N, T* __restrict__ dk) {
  const int m = blockIdx.x, r = blockIdx.y, b = blockIdx.z;
  const int nblk = N / SAS_BLOCK;
  const float* src = dkbar + (((size_t)b * Hkv + r) * nblk + m) * D;
  T* dst = dk + (((size_t)b * Hkv + r) * N + (size_t)m * SAS_BLOCK) * D;
  for (int e = threadIdx.x; e < SAS_BLOCK * D; e += blockDim.x) {
    const int c = e % D;
    dst[e] = from_f<T>(to_f(dst[e]) + src[c] * (1.0f / SAS_BLOCK));
  }
}

size_t select_bwd_tokens_ws_bytes(int B, int Hkv, int N, int d) {
  return (size_t)B * Hkv * (N / SAS_BLOCK) * d * sizeof(float);
}

cudaError_t launch_select_bwd_tokens(const void* q, int bf16, const float* ksum, int B, int Hq,
                                     int Hkv, int N, int d, int topk, float scale,
                                     const int32_t* idx, const int32_t* cnt, const float* dlogg,
                                     void* dq, void* dk, void* ws, cudaStream_t st) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK;
  const int nblk = N / SAS_BLOCK;
  if (B == 0 || nblk == 0 || topk == 0) return cudaSuccess;
  float* dkbar = static_cast<float*>(ws);
  cudaError_t e = cudaMemsetAsync(dkbar, 0, select_bwd_tokens_ws_bytes(B, Hkv, N, d), st);
  if (e != cudaSuccess) return e;
  dim3 grid(T_, Hkv, B), sgrid(nblk, Hkv, B);
#define SAS_TSBW(TT, DD)                                                                       \
  do {                                                                                         \
    auto kern = k_select_bwd_tokens<TT, DD>;                                                   \
    const size_t smb = tok_sel_smem<DD>(T_ - 1);                                               \
    cudaError_t e2 = ensure_smem(kern, smb);                                                   \
    if (e2 != cudaSuccess) return e2;                                                          \
    kern<<<grid, AT_THREADS, smb, st>>>(static_cast<const TT*>(q), ksum, Hq, Hkv, N, topk,     \
                                        scale, idx, cnt, dlogg, static_cast<TT*>(dq), dkbar);  \
    k_spread_dkbar<TT, DD><<<sgrid, 256, 0, st>>>(dkbar, Hkv, N, static_cast<TT*>(dk));       \
  } while (0)
  if (bf16) {
    if (d == 128) SAS_TSBW(__nv_bfloat16, 128); else SAS_TSBW(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_TSBW(float, 128); else SAS_TSBW(float, 64);
  }
#undef SAS_TSBW
  return cudaGetLastError();
}

uint32_t* tokens_error_word() {
  void* p = nullptr;
  cudaGetSymbolAddress(&p, g_tokens_err);
  return static_cast<uint32_t*>(p);
}

}  // namespace sas
