// Decode attention over the selected blocks (SAS close reading,
// liuzhao09.github.io, section 2.4 serving path: one query token per
// sequence, GQA groups share one block set; section 2.1: the current block is
// always kept; section 2.2: o = softmax(q K_S^T + log g_S) V_S).
//
// Split-K over the row's units (the kept history blocks, then the current
// block). One CTA per (split, kv group, sequence) bulk-copies whole 64-token
// K and V blocks of its kv head into shared memory (each block of one head is
// a contiguous 64 x d slab of the cache), scores every head of the group with
// lane-split dot products and 3-step shuffle reductions, and writes a partial
// (m, l, acc[d]) per head. The last CTA of a row (atomic counter, no waiting)
// combines the partials with the exact LSE rescaling (the same two-phase
// pattern as the MSA notes' Obuf/LSEbuf combine, papercache, forward kernel
// section) and writes o.
//
// The kernel may be launched as a programmatic dependent of the selection
// kernel: it loads q before griddepcontrol.wait and everything that depends
// on the selection after it.
#include <float.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace sas {

constexpr int DEC_THREADS = 256;

__device__ uint32_t g_decode_err = 0;

struct DecodeAttendWs {
  int* counter;  // [B*Hkv], zero on entry (caller-cleared)
  float* pm;     // [B][Hq][nsplit]
  float* pl;     // [B][Hq][nsplit]
  float* pacc;   // [B][Hq][nsplit][d]
  int nsplit;
  int units;     // units per split
};

static size_t a16(size_t x) { return (x + 15) & ~(size_t)15; }

static void decode_split(int topk, int rows, int* nsplit, int* units) {
  // One 64-token block per CTA unless that gives far more CTAs than SMs.
  int u = 1;
  while (u < 2 && (long long)rows * ((topk + 1 + u - 1) / u) > 8LL * 148) ++u;
  *units = u;
  *nsplit = (topk + 1 + u - 1) / u;
}

size_t decode_attend_ws_bytes(int B, int Hq, int Hkv, int topk, int d) {
  int ns, u;
  decode_split(topk, B * Hkv, &ns, &u);
  const size_t e = (size_t)B * Hq * ns;
  return 2 * a16(sizeof(float) * e) + a16(sizeof(float) * e * d);
}

static DecodeAttendWs carve_attend(int* counters, void* ws, int B, int Hq, int Hkv, int topk,
                                   int d) {
  DecodeAttendWs w;
  decode_split(topk, B * Hkv, &w.nsplit, &w.units);
  const size_t e = (size_t)B * Hq * w.nsplit;
  char* c = static_cast<char*>(ws);
  w.counter = counters;
  w.pm = reinterpret_cast<float*>(c); c += a16(sizeof(float) * e);
  w.pl = reinterpret_cast<float*>(c); c += a16(sizeof(float) * e);
  w.pacc = reinterpret_cast<float*>(c);
  return w;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(DEC_THREADS) k_decode_attend(
    const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc, int Hkv,
    int Lmax, const int32_t* __restrict__ lens, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ cnt, const float* __restrict__ logg, int topk, int gated,
    float scale, DecodeAttendWs w, T* __restrict__ o) {
  constexpr int VEC = Vec16<T>::N;         // elements per 16-byte piece
  constexpr int NCH = D / (8 * VEC);       // 16-byte pieces per lane and key
  constexpr int TILE = SAS_BLOCK * D;      // elements per K or V block
  extern __shared__ __align__(128) unsigned char smem[];
  const int U = w.units;
  T* ks = reinterpret_cast<T*>(smem);
  T* vs = ks + (size_t)U * TILE;
  float* zs = reinterpret_cast<float*>(vs + (size_t)U * TILE);  // [G][U*64]
  float* q_s = zs + G * U * SAS_BLOCK;                           // [G][D]
  __shared__ uint64_t bar;
  __shared__ int is_last;
  __shared__ float m_s[G], l_s[G];

  const int s = blockIdx.x, r = blockIdx.y, b = blockIdx.z;
  const int Hq = Hkv * G, nsplit = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int row = b * Hkv + r;

  for (int i = tid; i < G * D; i += DEC_THREADS)
    q_s[i] = to_f(q[((size_t)b * Hq + r * G) * D + i]);
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  grid_dep_wait();  // the selection below comes from the preceding kernel

  const int nblk = Lmax / SAS_BLOCK;
  const int n = min(max(lens[b], 1), Lmax);  // 1 <= n <= Lmax
  const int t = (n - 1) / SAS_BLOCK;
  const int ncur = n - t * SAS_BLOCK;
  const int kk = min(max(cnt[row], 0), topk);
  const int u0 = s * U;
  const int nu = max(0, min(U, kk + 1 - u0));

  if (tid == 0 && nu > 0) {
    mbar_arrive_expect_tx(&bar, (uint32_t)(nu * 2 * TILE * sizeof(T)));
    for (int i = 0; i < nu; ++i) {
      const int unit = u0 + i;
      int blk = unit < kk ? idx[(size_t)row * topk + unit] : t;
      if (blk < 0 || blk >= nblk) {
        atomicOr(&g_decode_err, kErrBadIndex);
        blk = t;
      }
      const size_t off = ((size_t)row * Lmax + (size_t)blk * SAS_BLOCK) * D;
      bulk_g2s(ks + (size_t)i * TILE, kc + off, TILE * sizeof(T), &bar);
      bulk_g2s(vs + (size_t)i * TILE, vc + off, TILE * sizeof(T), &bar);
    }
  }
  bool ok = true;
  if (nu > 0) ok = mbar_wait_data(&bar, 0, &g_decode_err);
  ok = __syncthreads_and(ok) != 0;  // block-uniform before the barriers below

  if (nu > 0 && ok) {
    // ---- scores: a warp covers 4 keys at a time, 8 lanes per key.
    const int jq = lane >> 3, p = lane & 7;
    for (int i = 0; i < nu; ++i) {
      const int unit = u0 + i;
      const bool cur = (unit == kk);
      const float bias = (!cur && gated) ? logg[(size_t)row * topk + unit] : 0.f;
      const T* kt = ks + (size_t)i * TILE;
      for (int j0 = wid * 4; j0 < SAS_BLOCK; j0 += 32) {
        const int j = j0 + jq;
        float kv[NCH * VEC];
#pragma unroll
        for (int c = 0; c < NCH; ++c)
          Vec16<T>::load(kt + (size_t)j * D + c * 8 * VEC + p * VEC, kv + c * VEC);
        float dot[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float a = 0.f;
#pragma unroll
          for (int c = 0; c < NCH; ++c) {
            const float* qp = q_s + h * D + c * 8 * VEC + p * VEC;
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
        if (p == 0) {
          const bool masked = cur && j >= ncur;
#pragma unroll
          for (int h = 0; h < G; ++h)
            zs[h * U * SAS_BLOCK + i * SAS_BLOCK + j] = masked ? -INFINITY : dot[h] * scale + bias;
        }
      }
    }
    __syncthreads();
    // ---- per-head partial softmax over this split's keys.
    const int nk = nu * SAS_BLOCK;
    for (int h = wid; h < G; h += DEC_THREADS / 32) {
      float* z = zs + h * U * SAS_BLOCK;
      float mx = -INFINITY;
      for (int j = lane; j < nk; j += 32) mx = fmaxf(mx, z[j]);
      mx = warp_max(mx);
      float sum = 0.f;
      for (int j = lane; j < nk; j += 32) {
        const float e = __expf(z[j] - mx);
        z[j] = e;
        sum += e;
      }
      sum = warp_sum(sum);
      if (lane == 0) {
        m_s[h] = mx;
        l_s[h] = sum;
      }
    }
    __syncthreads();
    // ---- acc[h][c] = sum_j p[h][j] v_j[c], two columns per thread.
    for (int pi = tid; pi < G * D / 2; pi += DEC_THREADS) {
      const int h = pi / (D / 2), c = (pi % (D / 2)) * 2;
      const float* z = zs + h * U * SAS_BLOCK;
      float a0 = 0.f, a1 = 0.f;
      for (int i = 0; i < nu; ++i) {
        const T* vt = vs + (size_t)i * TILE + c;
        const float* zi = z + i * SAS_BLOCK;
#pragma unroll 8
        for (int j = 0; j < SAS_BLOCK; ++j) {
          const float pj = zi[j];
          a0 += pj * to_f(vt[(size_t)j * D]);
          a1 += pj * to_f(vt[(size_t)j * D + 1]);
        }
      }
      const size_t e = ((size_t)b * Hq + r * G + h) * nsplit + s;
      w.pacc[e * D + c] = a0;
      w.pacc[e * D + c + 1] = a1;
    }
    if (tid < G) {
      const size_t e = ((size_t)b * Hq + r * G + tid) * nsplit + s;
      w.pm[e] = m_s[tid];
      w.pl[e] = l_s[tid];
    }
  } else if (tid < G) {  // empty split (or a failed wait): contributes nothing
    const size_t e = ((size_t)b * Hq + r * G + tid) * nsplit + s;
    w.pm[e] = -FLT_MAX;
    w.pl[e] = 0.f;
  }

  // ---- the last split of the row combines.
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(w.counter + row, 1) == nsplit - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // Combine. The split statistics are staged in shared memory (the K tile
  // region is free now) with one parallel pass of L2 loads; each head's
  // weights f_s = exp(m_s - M) / L are formed once; then every output column
  // sums its splits with independent, unrolled loads.
  float* pm_s = reinterpret_cast<float*>(ks);  // [G][nsplit]
  float* f_s = pm_s + G * nsplit;              // [G][nsplit]
  const size_t e_row = ((size_t)b * Hq + r * G) * nsplit;
  for (int i = tid; i < G * nsplit; i += DEC_THREADS) {
    pm_s[i] = __ldcg(w.pm + e_row + i);
    f_s[i] = __ldcg(w.pl + e_row + i);
  }
  __syncthreads();
  for (int h = wid; h < G; h += DEC_THREADS / 32) {
    float M = -FLT_MAX;
    for (int i = lane; i < nsplit; i += 32) M = fmaxf(M, pm_s[h * nsplit + i]);
    M = warp_max(M);
    float L = 0.f;
    for (int i = lane; i < nsplit; i += 32) {
      const float l = f_s[h * nsplit + i];
      if (l > 0.f) L += l * __expf(pm_s[h * nsplit + i] - M);
    }
    L = warp_sum(L);
    __syncwarp();
    for (int i = lane; i < nsplit; i += 32) {
      const float l = f_s[h * nsplit + i];
      f_s[h * nsplit + i] = (l > 0.f) ? __expf(pm_s[h * nsplit + i] - M) / L : 0.f;
    }
  }
  __syncthreads();
  for (int oi = tid; oi < G * D; oi += DEC_THREADS) {
    const int h = oi / D, c = oi % D;
    const float* fh = f_s + h * nsplit;
    const float* src = w.pacc + (e_row + (size_t)h * nsplit) * D + c;
    float A = 0.f;
#pragma unroll 8
    for (int i = 0; i < nsplit; ++i) {
      const float f = fh[i];
      const float x = __ldcg(src + (size_t)i * D);  // unwritten for empty splits: masked
      A += (f != 0.f) ? x * f : 0.f;
    }
    o[((size_t)b * Hq + r * G + h) * D + c] = from_f<T>(A);
  }
  if (tid == 0) w.counter[row] = 0;
}

template <typename T, int D, int G>
static cudaError_t launch_attend_t(const void* q, const void* kc, const void* vc, int B, int Hkv,
                                   int Lmax, const int32_t* lens, const int32_t* idx,
                                   const int32_t* cnt, const float* logg, int topk, int gated,
                                   float scale, void* o, DecodeAttendWs w, cudaStream_t st,
                                   bool pdl) {
  const size_t smem = (size_t)w.units * 2 * SAS_BLOCK * D * sizeof(T) +
                      sizeof(float) * ((size_t)G * w.units * SAS_BLOCK + (size_t)G * D);
  auto kern = k_decode_attend<T, D, G>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(w.nsplit, Hkv, B);
  cfg.blockDim = dim3(DEC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(q), static_cast<const T*>(kc),
                            static_cast<const T*>(vc), Hkv, Lmax, lens, idx, cnt, logg, topk,
                            gated, scale, w, static_cast<T*>(o));
}

template <typename T, int D>
static cudaError_t launch_attend_g(int G, const void* q, const void* kc, const void* vc, int B,
                                   int Hkv, int Lmax, const int32_t* lens, const int32_t* idx,
                                   const int32_t* cnt, const float* logg, int topk, int gated,
                                   float scale, void* o, DecodeAttendWs w, cudaStream_t st,
                                   bool pdl) {
#define SAS_ATT(GG)                                                                        \
  return launch_attend_t<T, D, GG>(q, kc, vc, B, Hkv, Lmax, lens, idx, cnt, logg, topk, \
                                   gated, scale, o, w, st, pdl)
  switch (G) {
    case 1: SAS_ATT(1);
    case 2: SAS_ATT(2);
    case 4: SAS_ATT(4);
    case 8: SAS_ATT(8);
    default: return cudaErrorInvalidValue;
  }
#undef SAS_ATT
}

cudaError_t launch_decode_attend(const void* q, const void* kc, const void* vc, int bf16, int B,
                                 int Hq, int Hkv, int Lmax, int d, const int32_t* lens,
                                 const int32_t* idx, const int32_t* cnt, const float* logg,
                                 int topk, int gated, float scale, void* o, int* counters,
                                 void* ws, cudaStream_t st, bool pdl) {
  if (B == 0) return cudaSuccess;
  DecodeAttendWs w = carve_attend(counters, ws, B, Hq, Hkv, topk, d);
  const int G = Hq / Hkv;
  if (bf16) {
    if (d == 128)
      return launch_attend_g<__nv_bfloat16, 128>(G, q, kc, vc, B, Hkv, Lmax, lens, idx, cnt, logg,
                                                 topk, gated, scale, o, w, st, pdl);
    return launch_attend_g<__nv_bfloat16, 64>(G, q, kc, vc, B, Hkv, Lmax, lens, idx, cnt, logg,
                                              topk, gated, scale, o, w, st, pdl);
  }
  if (d == 128)
    return launch_attend_g<float, 128>(G, q, kc, vc, B, Hkv, Lmax, lens, idx, cnt, logg, topk,
                                       gated, scale, o, w, st, pdl);
  return launch_attend_g<float, 64>(G, q, kc, vc, B, Hkv, Lmax, lens, idx, cnt, logg, topk, gated,
                                    scale, o, w, st, pdl);
}

uint32_t* decode_error_word() {
  void* p = nullptr;
  cudaGetSymbolAddress(&p, g_decode_err);
  return static_cast<uint32_t*>(p);
}

}  // namespace sas
