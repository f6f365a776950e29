// One decode step in one launch: selection (scores, softmax gate, Top-K) and
// split-K attention with the exact combine, one thread-block cluster per
// (sequence, kv group).
//
// Method: SAS close reading (liuzhao09.github.io), section 2.1 (block
// summaries, I = TopK(s, k), the current block always kept), section 2.2
// (g = softmax(s) over the C visible history blocks, log g = s - LSE,
// o = softmax(q K_S^T + log g_S) V_S), section 2.4 (serving: GQA groups share
// one block set); the 1/sqrt(d) logit scale from the reproduction note.
//
// Cluster of CS CTAs (16, or 8 when the batch has many rows). CTA c of the
// cluster:
//   1. bulk-copies its contiguous range of the row's block summaries through
//      a two-slot shared-memory ring and scores them against qbar (mean of
//      the group's query heads); the current block's K/V, known before any
//      selection, is prefetched at the same time by the CTA that owns it;
//   2. reduces its range to a best-first list of min(k, n) candidates (rank
//      counting per warp, then a pairwise tree merge of the 8 warp lists) and
//      the range's (max, sum exp), and stores list and sums into the stage
//      slot of every CTA of the cluster (remote shared-memory stores);
//   3. after a cluster barrier every CTA merges the CS staged lists the same
//      way and holds the row's kept blocks (ascending) and the gate's LSE;
//   4. bulk-copies the K/V blocks of its share of the units (the current
//      block first, then kept blocks) through a two-slot ring that reuses
//      the summary ring, keeping an online softmax state (m, l, acc) for
//      every head of the group, and stores head h's state into CTA h;
//   5. after a second cluster barrier CTA h < G combines head h from the CS
//      states (exact LSE rescaling) in its own shared memory and writes o.
// Data moves between CTAs only by stores made before a barrier, so every
// read after it is local. No global scratch, atomics or memsets; every wait
// is bounded.
#include <cooperative_groups.h>
#include <float.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace sas {

__device__ uint32_t g_decode_fused_err = 0;

constexpr int FD_THREADS = 256;
constexpr int FD_WARPS = FD_THREADS / 32;

// Two adjacent elements as fp32.
__device__ __forceinline__ void load2(const float* p, float2& v) {
  v = *reinterpret_cast<const float2*>(p);
}
__device__ __forceinline__ void load2(const __nv_bfloat16* p, float2& v) {
  v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

struct FdSmem {  // byte offsets into dynamic shared memory
  size_t kv0, u1, q, qbar, sc, zs, wa, wb, wlen_a, wlen_b, sa, sb, slen_a, slen_b, smx, sse, kidx,
      klogg, cm, cl, cacc, bars, total;
};

__host__ __device__ inline size_t fd_al(size_t x) { return (x + 127) & ~(size_t)127; }

// kv0: K/V slot 0 (the current block is prefetched into it). u1: the summary
// ring (2 x subc summaries) during the scan, K/V slot 1 afterwards.
__host__ __device__ inline FdSmem fd_layout(int D, int G, int es, int subc, int per, int k, int CS) {
  FdSmem L;
  const size_t kvslot = (size_t)2 * SAS_BLOCK * D * es;
  const size_t ring = (size_t)2 * subc * D * 4;
  const size_t kq = (size_t)1 << ceil_log2(k > 0 ? k : 1);  // list stride (power of two)
  size_t o = 0;
  L.kv0 = o; o += fd_al(kvslot);
  L.u1 = o; o += fd_al(kvslot > ring ? kvslot : ring);
  L.q = o; o += fd_al((size_t)G * D * 4);
  L.qbar = o; o += fd_al((size_t)D * 4);
  L.sc = o; o += fd_al((size_t)(per > 0 ? per : 1) * 4);
  L.zs = o; o += fd_al((size_t)G * SAS_BLOCK * 4);
  L.wa = o; o += fd_al(FD_WARPS * kq * 8);
  L.wb = o; o += fd_al(FD_WARPS * kq * 8);
  L.wlen_a = o; o += fd_al(FD_WARPS * 4);
  L.wlen_b = o; o += fd_al(FD_WARPS * 4);
  L.sa = o; o += fd_al((size_t)CS * kq * 8);
  L.sb = o; o += fd_al((size_t)CS * kq * 8);
  L.slen_a = o; o += fd_al((size_t)CS * 4);
  L.slen_b = o; o += fd_al((size_t)CS * 4);
  L.smx = o; o += fd_al((size_t)CS * 4);
  L.sse = o; o += fd_al((size_t)CS * 4);
  L.kidx = o; o += fd_al(128 * 4);
  L.klogg = o; o += fd_al(128 * 4);
  L.cm = o; o += fd_al((size_t)CS * 4);
  L.cl = o; o += fd_al((size_t)CS * 4);
  L.cacc = o; o += fd_al((size_t)CS * D * 4);
  L.bars = o; o += fd_al(4 * 8);
  L.total = o;
  return L;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(FD_THREADS, 2) k_decode_fused(
    const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
    const float* __restrict__ ksum, int Hkv, int Lmax, const int32_t* __restrict__ lens, int topk,
    int gated, float scale, int subc, int per_max, T* __restrict__ o,
    int32_t* __restrict__ idx_out) {
  constexpr int TILE = SAS_BLOCK * D;
  constexpr int PER = D / 32;
  constexpr int VEC = Vec16<T>::N;
  constexpr int NCH = D / (8 * VEC);
  extern __shared__ __align__(128) unsigned char sm[];
  cg::cluster_group cluster = cg::this_cluster();
  // Every CTA of the cluster must be running before anyone stores into its
  // shared memory: arrive now, wait just before the first remote store.
  cluster_arrive_relaxed();
  const int CS = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const FdSmem L = fd_layout(D, G, (int)sizeof(T), subc, per_max, topk, CS);
  const int lg = ceil_log2(topk > 0 ? topk : 1);
  const int kq = 1 << lg;  // list stride
  T* kv0 = reinterpret_cast<T*>(sm + L.kv0);
  T* kv1 = reinterpret_cast<T*>(sm + L.u1);
  float* sumbuf = reinterpret_cast<float*>(sm + L.u1);
  float* q_s = reinterpret_cast<float*>(sm + L.q);
  float* qbar = reinterpret_cast<float*>(sm + L.qbar);
  float* sc = reinterpret_cast<float*>(sm + L.sc);
  float* zs = reinterpret_cast<float*>(sm + L.zs);
  unsigned long long* wa = reinterpret_cast<unsigned long long*>(sm + L.wa);
  unsigned long long* wb = reinterpret_cast<unsigned long long*>(sm + L.wb);
  int* wlen_a = reinterpret_cast<int*>(sm + L.wlen_a);
  int* wlen_b = reinterpret_cast<int*>(sm + L.wlen_b);
  unsigned long long* sa = reinterpret_cast<unsigned long long*>(sm + L.sa);
  unsigned long long* sb = reinterpret_cast<unsigned long long*>(sm + L.sb);
  int* slen_a = reinterpret_cast<int*>(sm + L.slen_a);
  int* slen_b = reinterpret_cast<int*>(sm + L.slen_b);
  float* smx = reinterpret_cast<float*>(sm + L.smx);
  float* sse = reinterpret_cast<float*>(sm + L.sse);
  int* kidx = reinterpret_cast<int*>(sm + L.kidx);
  float* klogg = reinterpret_cast<float*>(sm + L.klogg);
  float* cm = reinterpret_cast<float*>(sm + L.cm);
  float* cl = reinterpret_cast<float*>(sm + L.cl);
  float* cacc = reinterpret_cast<float*>(sm + L.cacc);
  uint64_t* sum_bar = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* kv_bar = sum_bar + 2;
  __shared__ float red[FD_WARPS];
  __shared__ float alpha_s[G], m_run[G], l_run[G];
  __shared__ float loc_mx, loc_se;
  __shared__ int ok_s;

  const int r = blockIdx.y, b = blockIdx.z;
  const int Hq = Hkv * G;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const size_t row = (size_t)b * Hkv + r;
  const int nblk = Lmax / SAS_BLOCK;
  const int n = min(max(lens[b], 1), Lmax);
  const int t = (n - 1) / SAS_BLOCK;  // current block; C = t history blocks
  const int C = t;
  const int ncur = n - t * SAS_BLOCK;
  const int kk = min(topk, C);
  const int units = kk + 1;
  const int per = (C + CS - 1) / CS;  // history blocks scored by each CTA
  const int m0 = min(C, crank * per), m1 = min(C, m0 + per), nmine = m1 - m0;
  const int upc = (units + CS - 1) / CS;  // units attended by each CTA
  const int u0 = min(units, crank * upc), u1 = min(units, u0 + upc), nu = u1 - u0;
  const bool own_cur = (kk >= u0 && kk < u1);
  const int nsub = (nmine + subc - 1) / subc;
  const size_t kvrow = row * (size_t)Lmax * D;
  const float* ks_row = ksum + row * (size_t)nblk * D;
  uint32_t* err = &g_decode_fused_err;

  if (tid == 0) {
    mbar_init(&sum_bar[0], 1);
    mbar_init(&sum_bar[1], 1);
    mbar_init(&kv_bar[0], 1);
    mbar_init(&kv_bar[1], 1);
    fence_mbar_init();
    ok_s = 1;
  }
  __syncthreads();
  if (tid == 0) {
    for (int i = 0; i < min(2, nsub); ++i) {
      const int cnt_i = min(subc, nmine - i * subc);
      mbar_arrive_expect_tx(&sum_bar[i], (uint32_t)(cnt_i * D * 4));
      bulk_g2s(sumbuf + (size_t)i * subc * D, ks_row + (size_t)(m0 + i * subc) * D,
               (uint32_t)(cnt_i * D * 4), &sum_bar[i]);
    }
    if (own_cur) {  // the current block is unit 0 of this CTA's order, slot 0
      mbar_arrive_expect_tx(&kv_bar[0], (uint32_t)(2 * TILE * sizeof(T)));
      bulk_g2s(kv0, kc + kvrow + (size_t)t * TILE, TILE * sizeof(T), &kv_bar[0]);
      bulk_g2s(kv0 + TILE, vc + kvrow + (size_t)t * TILE, TILE * sizeof(T), &kv_bar[0]);
    }
  }
  for (int i = tid; i < G * D; i += FD_THREADS) q_s[i] = to_f(q[((size_t)b * Hq + r * G) * D + i]);
  __syncthreads();
  for (int i = tid; i < D; i += FD_THREADS) {
    float a = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) a += q_s[g * D + i];
    qbar[i] = a / (float)G;
  }
  __syncthreads();

  // ---- 1. score this CTA's range of history blocks (4 blocks per warp in flight)
  {
    float qv[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) qv[i] = qbar[lane * PER + i];
    for (int i = 0; i < nsub; ++i) {
      const int slot = i & 1;
      const int cnt_i = min(subc, nmine - i * subc);
      if (!mbar_wait(&sum_bar[slot], (uint32_t)((i >> 1) & 1), err)) ok_s = 0;
      const float* sb = sumbuf + (size_t)slot * subc * D;
      for (int j0 = wid; j0 < cnt_i; j0 += 4 * FD_WARPS) {
        float part[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + u * FD_WARPS;
          float a = 0.f;
          if (j < cnt_i) {
            const float* p = sb + (size_t)j * D + lane * PER;
#pragma unroll
            for (int e = 0; e < PER; ++e) a += p[e] * qv[e];
          }
          part[u] = a;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) part[u] = warp_sum(part[u]);
        if (lane == 0) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = j0 + u * FD_WARPS;
            if (j < cnt_i) sc[i * subc + j] = part[u] * scale + 0.0f;
          }
        }
      }
      __syncthreads();  // slot consumed
      if (tid == 0 && i + 2 < nsub) {
        const int cnt_n = min(subc, nmine - (i + 2) * subc);
        mbar_arrive_expect_tx(&sum_bar[slot], (uint32_t)(cnt_n * D * 4));
        bulk_g2s(sumbuf + (size_t)slot * subc * D, ks_row + (size_t)(m0 + (i + 2) * subc) * D,
                 (uint32_t)(cnt_n * D * 4), &sum_bar[slot]);
      }
    }
  }
  // ---- 2. this range's (max, sum exp) and best-first list
  {
    float mx = -FLT_MAX;
    for (int j = tid; j < nmine; j += FD_THREADS) mx = fmaxf(mx, sc[j]);
    mx = warp_max(mx);
    if (lane == 0) red[wid] = mx;
    __syncthreads();
    mx = -FLT_MAX;
    for (int i = 0; i < FD_WARPS; ++i) mx = fmaxf(mx, red[i]);
    __syncthreads();
    float se = 0.f;
    for (int j = tid; j < nmine; j += FD_THREADS) se += __expf(sc[j] - mx);
    se = warp_sum(se);
    if (lane == 0) red[wid] = se;
    __syncthreads();
    if (tid == 0) {
      float a = 0.f;
      for (int i = 0; i < FD_WARPS; ++i) a += red[i];
      loc_mx = mx;
      loc_se = a;
    }
  }
  int wsel = 0;  // which warp-list buffer holds this CTA's merged list (list 0)
  if (topk > 0 && nmine <= FD_THREADS) {
    // small range: one rank-counting pass over the whole range, one item per
    // thread (broadcast shared-memory reads), straight into list 0 of A
    if (tid < nmine) {
      const float sj = sc[tid];
      int rk = 0;
      for (int x = 0; x < nmine; ++x) {
        const float sx = sc[x];
        rk += (sx > sj) || (sx == sj && x < tid);
      }
      if (rk < topk) wa[rk] = cand_key(sj, m0 + tid);
    }
    if (tid == 0) wlen_a[0] = min(topk, nmine);
  } else if (topk > 0) {
    // each warp ranks its contiguous share of the range
    const int pw = (nmine + FD_WARPS - 1) / FD_WARPS;
    const int a0 = min(nmine, wid * pw), a1 = min(nmine, a0 + pw);
    for (int j = a0 + lane; j < a1; j += 32) {
      const float sj = sc[j];
      int rk = 0;
      for (int x = a0; x < a1; ++x) {
        const float sx = sc[x];
        rk += (sx > sj) || (sx == sj && x < j);
      }
      if (rk < topk) wa[wid * kq + rk] = cand_key(sj, m0 + j);
    }
    if (lane == 0) wlen_a[wid] = min(topk, a1 - a0);
    __syncthreads();
    wsel = tree_merge(wa, wlen_a, wb, wlen_b, FD_WARPS, lg, topk);
  }
  __syncthreads();
  // ---- push this CTA's list and partial sums into every CTA's stage slot
  cluster_wait_acquire();  // every CTA of the cluster is running
  {
    const unsigned long long* mine = wsel ? wb : wa;
    const int my_len = topk > 0 ? (wsel ? wlen_b[0] : wlen_a[0]) : 0;
    for (int e = tid; e < CS * (my_len + 1); e += FD_THREADS) {
      const int c = e / (my_len + 1), p = e - c * (my_len + 1);
      if (p < my_len) {
        *cluster.map_shared_rank(sa + crank * kq + p, c) = mine[p];
      } else {
        *cluster.map_shared_rank(slen_a + crank, c) = my_len;
        *cluster.map_shared_rank(smx + crank, c) = loc_mx;
        *cluster.map_shared_rank(sse + crank, c) = loc_se;
      }
    }
  }
  cluster_arrive_release();
  cluster_wait_acquire();  // all lists are in this CTA's shared memory

  // ---- 3. merge the CS lists (every CTA, identically) and the LSE
  float lse;
  {
    float M = -FLT_MAX;
    for (int c = 0; c < CS; ++c) M = fmaxf(M, smx[c]);
    float S = 0.f;
    for (int c = 0; c < CS; ++c)
      if (sse[c] > 0.f) S += sse[c] * __expf(smx[c] - M);
    lse = (C > 0) ? M + __logf(S) : 0.f;
  }
  if (topk > 0) {
    const int ssel = tree_merge(sa, slen_a, sb, slen_b, CS, lg, topk);
    const unsigned long long* fk = ssel ? sb : sa;
    for (int i = tid; i < kk; i += FD_THREADS) {  // ascending block order
      const int mi = key_block(fk[i]);
      int pos = 0;
      for (int j = 0; j < kk; ++j) pos += key_block(fk[j]) < mi;
      kidx[pos] = mi;
      klogg[pos] = key_score(fk[i]) - lse;
    }
    __syncthreads();
    if (crank == 0 && idx_out != nullptr)
      for (int i = tid; i < topk; i += FD_THREADS) idx_out[row * topk + i] = i < kk ? kidx[i] : -1;
  }

  // ---- 4. attention over this CTA's units: the current block first when
  // owned (already in flight in slot 0), then its kept blocks ascending.
  auto unit_of = [&](int i) -> int {
    if (own_cur) return i == 0 ? kk : u0 + i - 1;
    return u0 + i;
  };
  auto issue_unit = [&](int i) {
    const int u = unit_of(i);
    int blk = (u == kk) ? t : kidx[u];
    if (blk < 0 || blk >= nblk) {
      atomicOr(err, kErrBadIndex);
      blk = t;
    }
    const int slot = i & 1;
    T* kdst = slot ? kv1 : kv0;
    mbar_arrive_expect_tx(&kv_bar[slot], (uint32_t)(2 * TILE * sizeof(T)));
    bulk_g2s(kdst, kc + kvrow + (size_t)blk * TILE, TILE * sizeof(T), &kv_bar[slot]);
    bulk_g2s(kdst + TILE, vc + kvrow + (size_t)blk * TILE, TILE * sizeof(T), &kv_bar[slot]);
  };
  if (tid == 0)
    for (int i = own_cur ? 1 : 0; i < min(2, nu); ++i) issue_unit(i);
  if (tid < G) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.f;
  }
  constexpr int NITEM = (G * D / 2 + FD_THREADS - 1) / FD_THREADS;
  float acc[NITEM][2];
#pragma unroll
  for (int it = 0; it < NITEM; ++it) acc[it][0] = acc[it][1] = 0.f;
  const int jq = lane >> 3, pp = lane & 7;
  for (int i = 0; i < nu; ++i) {
    const int slot = i & 1;
    const int u = unit_of(i);
    const bool cur = (u == kk);
    const float bias = (!cur && gated) ? klogg[u] : 0.f;
    if (!mbar_wait(&kv_bar[slot], (uint32_t)((i >> 1) & 1), err)) ok_s = 0;
    const T* kt = slot ? kv1 : kv0;
    const T* vt = kt + TILE;
    for (int j0 = wid * 4; j0 < SAS_BLOCK; j0 += 4 * FD_WARPS) {
      const int j = j0 + jq;
      float kv[NCH * VEC];
#pragma unroll
      for (int c = 0; c < NCH; ++c)
        Vec16<T>::load(kt + (size_t)j * D + c * 8 * VEC + pp * VEC, kv + c * VEC);
      float dot[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          const float* qp = q_s + h * D + c * 8 * VEC + pp * VEC;
#pragma unroll
          for (int e = 0; e < VEC; ++e) a += kv[c * VEC + e] * qp[e];
        }
        dot[h] = a;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        dot[h] += __shfl_xor_sync(0xffffffffu, dot[h], 1);
        dot[h] += __shfl_xor_sync(0xffffffffu, dot[h], 2);
        dot[h] += __shfl_xor_sync(0xffffffffu, dot[h], 4);
      }
      if (pp == 0) {
        const bool masked = cur && j >= ncur;
#pragma unroll
        for (int h = 0; h < G; ++h) zs[h * SAS_BLOCK + j] = masked ? -INFINITY : dot[h] * scale + bias;
      }
    }
    __syncthreads();
    for (int h = wid; h < G; h += FD_WARPS) {  // online softmax state per head
      float* z = zs + h * SAS_BLOCK;
      const float mx = warp_max(fmaxf(z[lane], z[lane + 32]));
      const float mold = m_run[h];
      const float mnew = fmaxf(mold, mx);
      const float e0 = __expf(z[lane] - mnew), e1 = __expf(z[lane + 32] - mnew);
      z[lane] = e0;
      z[lane + 32] = e1;
      const float sum = warp_sum(e0 + e1);
      if (lane == 0) {
        const float al = __expf(mold - mnew);
        alpha_s[h] = al;
        l_run[h] = l_run[h] * al + sum;
        m_run[h] = mnew;
      }
    }
    __syncthreads();
#pragma unroll
    for (int it = 0; it < NITEM; ++it) {
      const int pi = tid + it * FD_THREADS;
      if (pi < G * D / 2) {
        const int h = pi / (D / 2), c = (pi % (D / 2)) * 2;
        const float* z = zs + h * SAS_BLOCK;
        const float al = alpha_s[h];
        float a0 = acc[it][0] * al, a1 = acc[it][1] * al;
        float b0 = 0.f, b1 = 0.f;  // two independent chains per column
#pragma unroll 8
        for (int j = 0; j < SAS_BLOCK; j += 2) {
          float2 v0, v1;
          load2(vt + (size_t)j * D + c, v0);
          load2(vt + (size_t)(j + 1) * D + c, v1);
          a0 += z[j] * v0.x;
          a1 += z[j] * v0.y;
          b0 += z[j + 1] * v1.x;
          b1 += z[j + 1] * v1.y;
        }
        acc[it][0] = a0 + b0;
        acc[it][1] = a1 + b1;
      }
    }
    __syncthreads();  // slot and zs consumed
    if (tid == 0 && i + 2 < nu) issue_unit(i + 2);
  }
  // ---- push this CTA's partial state of head h into CTA h's combine slot
#pragma unroll
  for (int it = 0; it < NITEM; ++it) {
    const int pi = tid + it * FD_THREADS;
    if (pi < G * D / 2) {
      const int h = pi / (D / 2), c = (pi % (D / 2)) * 2;
      float* dst = cluster.map_shared_rank(cacc + crank * D + c, h);
      dst[0] = acc[it][0];
      dst[1] = acc[it][1];
    }
  }
  if (tid < G) {
    *cluster.map_shared_rank(cm + crank, tid) = m_run[tid];
    *cluster.map_shared_rank(cl + crank, tid) = l_run[tid];
  }
  if (tid == 0 && ok_s == 0) atomicOr(err, kErrWaitTimeout);
  cluster_arrive_release();
  cluster_wait_acquire();  // every partial state has arrived; no remote access follows

  // ---- 5. CTA h < G combines head h (exact LSE rescaling)
  if (crank < G) {
    const int h = crank;
    float M = -FLT_MAX;
    for (int c = 0; c < CS; ++c) M = fmaxf(M, cm[c]);
    float Lsum = 0.f;
    for (int c = 0; c < CS; ++c)
      if (cl[c] > 0.f) Lsum += cl[c] * __expf(cm[c] - M);
    const float inv = 1.f / Lsum;
    for (int col = tid; col < D; col += FD_THREADS) {
      float a = 0.f;
      for (int c = 0; c < CS; ++c)
        if (cl[c] > 0.f) a += cacc[c * D + col] * __expf(cm[c] - M);
      o[((size_t)b * Hq + r * G + h) * D + col] = from_f<T>(a * inv);
    }
  }
}

// ------------------------------------------------------------------ host
struct FdPlan {
  int CS, subc, per_max;
  size_t smem;
};

static FdPlan fd_plan(int B, int Hkv, int Lmax, int d, int G, int es, int topk, int CS) {
  FdPlan p;
  p.CS = CS;
  p.subc = 32;  // 2 x 32 summaries in flight per CTA; aliased with K/V slot 1
  const int nblk = Lmax / SAS_BLOCK;
  p.per_max = (nblk + CS - 1) / CS;
  p.smem = fd_layout(d, G, es, p.subc, p.per_max, topk, CS).total;
  (void)B; (void)Hkv;
  return p;
}

template <typename T, int D, int G>
static cudaError_t launch_fused_t(const void* q, const void* kc, const void* vc, const float* ksum,
                                  int B, int Hkv, int Lmax, const int32_t* lens, int topk,
                                  int gated, float scale, void* o, int32_t* idx_out,
                                  cudaStream_t st) {
  auto kern = k_decode_fused<T, D, G>;
  const int rows = B * Hkv;
  // 16-CTA clusters while the rows fill the GPU with them; 8 otherwise.
  int CS = rows <= 9 ? 16 : 8;
  for (;;) {
    FdPlan p = fd_plan(B, Hkv, Lmax, D, G, (int)sizeof(T), topk, CS);
    if (p.smem > 227 * 1024) return cudaErrorInvalidConfiguration;
    cudaError_t e = ensure_smem(kern, p.smem);
    if (e != cudaSuccess) return e;
    if (CS > 8) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) { cudaGetLastError(); CS = 8; continue; }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CS, Hkv, B);
    cfg.blockDim = dim3(FD_THREADS);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
    if (e != cudaSuccess || nclusters < 1) {
      cudaGetLastError();
      if (CS > 8) { CS = 8; continue; }
      return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
    }
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(q), static_cast<const T*>(kc),
                              static_cast<const T*>(vc), ksum, Hkv, Lmax, lens, topk, gated,
                              scale, p.subc, p.per_max, static_cast<T*>(o), idx_out);
  }
}

template <typename T, int D>
static cudaError_t launch_fused_g(int G, const void* q, const void* kc, const void* vc,
                                  const float* ksum, int B, int Hkv, int Lmax, const int32_t* lens,
                                  int topk, int gated, float scale, void* o, int32_t* idx_out,
                                  cudaStream_t st) {
#define SAS_FD(GG)                                                                              \
  return launch_fused_t<T, D, GG>(q, kc, vc, ksum, B, Hkv, Lmax, lens, topk, gated, scale, o, \
                                  idx_out, st)
  switch (G) {
    case 1: SAS_FD(1);
    case 2: SAS_FD(2);
    case 4: SAS_FD(4);
    case 8: SAS_FD(8);
    default: return cudaErrorInvalidValue;
  }
#undef SAS_FD
}

cudaError_t launch_decode_fused(const void* q, const void* kc, const void* vc, int bf16, int B,
                                int Hq, int Hkv, int Lmax, int d, const int32_t* lens,
                                const float* ksum, int topk, int gated, float scale, void* o,
                                int32_t* idx_out, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  const int G = Hq / Hkv;
  if (bf16) {
    if (d == 128)
      return launch_fused_g<__nv_bfloat16, 128>(G, q, kc, vc, ksum, B, Hkv, Lmax, lens, topk,
                                                gated, scale, o, idx_out, st);
    return launch_fused_g<__nv_bfloat16, 64>(G, q, kc, vc, ksum, B, Hkv, Lmax, lens, topk, gated,
                                             scale, o, idx_out, st);
  }
  if (d == 128)
    return launch_fused_g<float, 128>(G, q, kc, vc, ksum, B, Hkv, Lmax, lens, topk, gated, scale,
                                      o, idx_out, st);
  return launch_fused_g<float, 64>(G, q, kc, vc, ksum, B, Hkv, Lmax, lens, topk, gated, scale, o,
                                   idx_out, st);
}

uint32_t* decode_fused_error_word() {
  void* p = nullptr;
  cudaGetSymbolAddress(&p, g_decode_fused_err);
  return static_cast<uint32_t*>(p);
}

}  // namespace sas
