// Selector scores, softmax gate and Top-K over the history blocks (SAS close
// reading, liuzhao09.github.io, sections 2.1-2.2: s = R(q, {K_Bm}),
// I = TopK(s, k), g = softmax(s) over the C history blocks, log g = s - LSE).
// The selector is parameter-free: s_m = scale * qbar . kbar_m.
//
// Top-K is exact and deterministic for any tie pattern. A candidate's order
// key is (score descending, block index ascending), packed into one 64-bit
// integer. Each chunk of up to 256 history blocks is scored into shared
// memory and reduced to its own best-first list of min(k, n) candidates by
// rank counting. The lists are then merged pairwise in a tree (each entry
// ranked in its partner list by one binary search, the best k kept per
// level), and the kept blocks are written in ascending block order. (The MSA
// notes, papercache, Top-K kernel section, use per-lane heaps and a shuffle
// merge on H800; chunk lists plus a parallel tree merge suit wide CTAs.)
//
// Prefill: one CTA per (b, kv group, query block). Decode: one CTA per
// (b, kv group, chunk); the last CTA to finish a row (atomic counter, no
// waiting) merges, writes the row and resets the counter.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace sas {

constexpr int SEL_THREADS = 256;
constexpr int SEL_CHUNK_MAX = 256;      // prefill chunk
constexpr int DEC_CHUNK_MAX = 512;      // decode chunk upper bound
constexpr int DEC_NCHUNK_MAX = 128;     // decode chunks per row upper bound

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float r = -FLT_MAX;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) r = fmaxf(r, red[i]);
  return r;
}

__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) r += red[i];
  return r;
}

// s[j] = scale * qbar . ksum_row[m0 + j] for j < n. Warp-per-block with the
// d dimension split over the lanes (D/32 floats each), four blocks in flight
// per warp. A -0 score is stored as +0 so that exact ties compare equal.
// gs (nullable): the row's raw-score output, written at gs[m0 + j] as well.
template <int D>
__device__ void score_chunk(const float* __restrict__ ks_row, int m0, int n,
                            const float* qbar_s, float scale, float* sc, float* gs) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  float qv[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) qv[i] = qbar_s[lane * PER + i];
  for (int base = w; base < n; base += nw * 4) {
    float part[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = base + u * nw;
      float acc = 0.f;
      if (j < n) {
        const float* p = ks_row + (size_t)(m0 + j) * D + lane * PER;
        if constexpr (PER == 4) {
          const float4 x = __ldg(reinterpret_cast<const float4*>(p));
          acc = x.x * qv[0] + x.y * qv[1] + x.z * qv[2] + x.w * qv[3];
        } else {
          const float2 x = __ldg(reinterpret_cast<const float2*>(p));
          acc = x.x * qv[0] + x.y * qv[1];
        }
      }
      part[u] = acc;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) part[u] = warp_sum(part[u]);
    if (lane == 0) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = base + u * nw;
        if (j < n) {
          const float sj = part[u] * scale + 0.0f;
          sc[j] = sj;
          if (gs != nullptr) gs[m0 + j] = sj;
        }
      }
    }
  }
}

// Best-first list of the keys of the min(k, n) best entries of sc[0..n)
// (blocks m0 + j), by rank counting.
__device__ void chunk_topk(const float* sc, int m0, int n, int k, unsigned long long* out) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float si = sc[i];
    int r = 0;
    for (int j = 0; j < n; ++j) {
      const float sj = sc[j];
      r += (sj > si) || (sj == si && j < i);
    }
    if (r < k) out[r] = cand_key(si, m0 + i);
  }
}

// Writes the kk best entries of a best-first key list to out_idx/out_logg in
// ascending block order (log g = s - lse), padded to k with -1 / 0.
__device__ void write_selection(const unsigned long long* keys, int kk, int k, float lse,
                                int32_t* out_idx, float* out_logg) {
  for (int i = threadIdx.x; i < kk; i += blockDim.x) {
    const int mi = key_block(keys[i]);
    int pos = 0;
    for (int j = 0; j < kk; ++j) pos += key_block(keys[j]) < mi;
    out_idx[pos] = mi;
    out_logg[pos] = key_score(keys[i]) - lse;
  }
  for (int i = kk + threadIdx.x; i < k; i += blockDim.x) {
    out_idx[i] = -1;
    out_logg[i] = 0.f;
  }
}

// ------------------------------------------------------------------ prefill
// qbar[b, r, t] = mean of q over the group's G heads and query block t's rows.
template <typename T, int D>
__global__ void __launch_bounds__(256) k_qbar_prefill(const T* __restrict__ q, int Hq, int Hkv,
                                                      int N, float* __restrict__ qbar) {
  constexpr int VEC = Vec16<T>::N;
  constexpr int TPR = D / VEC;
  constexpr int RP = 256 / TPR;
  __shared__ float red[RP][D];
  const int t = blockIdx.x, r = blockIdx.y, b = blockIdx.z, T_ = gridDim.x;
  const int G = Hq / Hkv;
  const int tid = threadIdx.x, c = tid % TPR, rg = tid / TPR;
  const int row0 = t * SAS_BLOCK, nr = min(SAS_BLOCK, N - row0);
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
  for (int g = 0; g < G; ++g) {
    const T* base = q + (((size_t)b * Hq + r * G + g) * N + row0) * D + c * VEC;
    for (int i = rg; i < nr; i += RP) {
      float x[VEC];
      Vec16<T>::load_nc(base + (size_t)i * D, x);
#pragma unroll
      for (int u = 0; u < VEC; ++u) acc[u] += x[u];
    }
  }
#pragma unroll
  for (int i = 0; i < VEC; ++i) red[rg][c * VEC + i] = acc[i];
  __syncthreads();
  const float inv = 1.0f / (float)(G * nr);
  float* out = qbar + (((size_t)b * Hkv + r) * T_ + t) * D;
  for (int col = tid; col < D; col += 256) {
    float s = 0.f;
    for (int i = 0; i < RP; ++i) s += red[i][col];
    out[col] = s * inv;
  }
}

template <int D>
__global__ void __launch_bounds__(SEL_THREADS) k_select_prefill(
    const float* __restrict__ qbar, const float* __restrict__ ksum, int Hkv, int nblk, int topk,
    float scale, int32_t* __restrict__ idx, int32_t* __restrict__ cnt, float* __restrict__ logg,
    float* __restrict__ scores) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int t = blockIdx.x, r = blockIdx.y, b = blockIdx.z, T_ = gridDim.x;
  const int C = t;
  const int nchunk = (C + SEL_CHUNK_MAX - 1) / SEL_CHUNK_MAX;
  const int nck = (nchunk + 3) & ~3;
  float* q_s = reinterpret_cast<float*>(smem_raw);
  float* sc = q_s + D;
  float* red = sc + SEL_CHUNK_MAX;
  int* len = reinterpret_cast<int*>(red + 32);
  int* len_b = len + nck;
  const int lg = ceil_log2(topk);
  unsigned long long* la = reinterpret_cast<unsigned long long*>(len_b + nck);  // 8-byte aligned
  unsigned long long* lb = la + ((size_t)nchunk << lg);

  const size_t row = ((size_t)b * Hkv + r) * T_ + t;
  const float* qrow = qbar + row * D;
  for (int i = threadIdx.x; i < D; i += blockDim.x) q_s[i] = qrow[i];
  __syncthreads();
  const float* ks_row = ksum + ((size_t)b * Hkv + r) * nblk * D;
  float* gs = scores != nullptr ? scores + row * T_ : nullptr;  // [T] of this row
  if (gs != nullptr)
    for (int m = C + threadIdx.x; m < T_; m += blockDim.x) gs[m] = -INFINITY;
  float run_m = -FLT_MAX, run_s = 0.f;
  for (int c = 0; c < nchunk; ++c) {
    const int m0 = c * SEL_CHUNK_MAX, n = min(SEL_CHUNK_MAX, C - m0);
    score_chunk<D>(ks_row, m0, n, q_s, scale, sc, gs);
    __syncthreads();
    if (topk > 0) chunk_topk(sc, m0, n, topk, la + ((size_t)c << lg));
    float lm = -FLT_MAX;
    for (int i = threadIdx.x; i < n; i += blockDim.x) lm = fmaxf(lm, sc[i]);
    lm = block_reduce_max(lm, red);
    float le = 0.f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) le += __expf(sc[i] - lm);
    le = block_reduce_sum(le, red);
    const float nm = fmaxf(run_m, lm);
    run_s = run_s * __expf(run_m - nm) + le * __expf(lm - nm);
    run_m = nm;
    if (threadIdx.x == 0) len[c] = min(topk, n);
    __syncthreads();
  }
  const int kk = min(topk, C);
  const float lse = (C > 0) ? run_m + __logf(run_s) : 0.f;
  if (topk > 0) {
    const int wb = tree_merge(la, len, lb, len_b, nchunk, lg, topk);
    write_selection(wb ? lb : la, kk, topk, lse, idx + row * topk,
                    logg + row * topk);
  }
  if (threadIdx.x == 0) cnt[row] = kk;
}

size_t select_prefill_ws_bytes(int B, int Hkv, int N, int d) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK;
  return (size_t)B * Hkv * T_ * d * sizeof(float);
}

static size_t prefill_select_smem(int d, int nchunk, int topk) {
  size_t n = (size_t)d + SEL_CHUNK_MAX + 32;  // q, sc, red
  n += 2 * (size_t)((nchunk + 3) & ~3);       // len, len_b
  n += 4 * ((size_t)nchunk << ceil_log2(topk));  // two key buffers (8 bytes each)
  return n * 4 + 8;
}

cudaError_t launch_qbar_prefill(const void* q, int bf16, int B, int Hq, int Hkv, int N, int d,
                                float* qbar, cudaStream_t st) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK;
  if (B == 0 || T_ == 0) return cudaSuccess;
  dim3 grid(T_, Hkv, B);
#define SAS_QBAR(T, D) \
  k_qbar_prefill<T, D><<<grid, 256, 0, st>>>(static_cast<const T*>(q), Hq, Hkv, N, qbar)
  if (bf16) {
    if (d == 128) SAS_QBAR(__nv_bfloat16, 128); else SAS_QBAR(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_QBAR(float, 128); else SAS_QBAR(float, 64);
  }
#undef SAS_QBAR
  return cudaGetLastError();
}

cudaError_t launch_select_prefill(const void* q, int bf16, const float* ksum, int B, int Hq,
                                  int Hkv, int N, int d, int topk, float scale, int32_t* idx,
                                  int32_t* cnt, float* logg, float* scores, void* ws,
                                  cudaStream_t st) {
  const int T_ = (N + SAS_BLOCK - 1) / SAS_BLOCK;
  if (B == 0 || T_ == 0) return cudaSuccess;
  float* qbar = static_cast<float*>(ws);
  dim3 grid(T_, Hkv, B);
#define SAS_QBAR(T, D) \
  k_qbar_prefill<T, D><<<grid, 256, 0, st>>>(static_cast<const T*>(q), Hq, Hkv, N, qbar)
  if (bf16) {
    if (d == 128) SAS_QBAR(__nv_bfloat16, 128); else SAS_QBAR(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_QBAR(float, 128); else SAS_QBAR(float, 64);
  }
#undef SAS_QBAR
  const int nblk = N / SAS_BLOCK;
  const int nchunk_max = (T_ - 1 + SEL_CHUNK_MAX - 1) / SEL_CHUNK_MAX;
  const size_t smem = prefill_select_smem(d, nchunk_max > 0 ? nchunk_max : 1, topk);
  if (d == 128) {
    ensure_smem(k_select_prefill<128>, smem);
    k_select_prefill<128><<<grid, SEL_THREADS, smem, st>>>(qbar, ksum, Hkv, nblk, topk, scale,
                                                           idx, cnt, logg, scores);
  } else {
    ensure_smem(k_select_prefill<64>, smem);
    k_select_prefill<64><<<grid, SEL_THREADS, smem, st>>>(qbar, ksum, Hkv, nblk, topk, scale,
                                                          idx, cnt, logg, scores);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------ prefill, no allocation
// For callers that cannot allocate device memory at call time, the prefill
// selection can keep its query summaries in a fixed array that is part of
// the library image instead of a caller-provided workspace. The array is
// statically sized (kStaticQbarFloats fp32 values, 4 MiB); every GPU that
// loads the library holds it until the process exits. All calls share it:
// each call overwrites the part it uses before reading it (nothing needs
// to start at zero), and calls that overlap on the GPU race on it.
constexpr size_t kStaticQbarFloats = size_t(1) << 20;
static __device__ __align__(256) float g_qbar_static[kStaticQbarFloats];

size_t select_prefill_static_capacity() { return kStaticQbarFloats; }

// Device address of the array for the current device: looked up with
// cudaGetSymbolAddress on the first call per device (the host-side name is
// only a stand-in and must never be passed to a kernel), then cached.
static cudaError_t static_qbar_address(float** out) {
  static std::mutex mu;
  static std::map<int, float*> addr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = addr.find(dev);
  if (it == addr.end()) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_qbar_static);
    if (e != cudaSuccess) return e;
    it = addr.emplace(dev, static_cast<float*>(p)).first;
  }
  *out = it->second;
  return cudaSuccess;
}

cudaError_t launch_select_prefill_static(const void* q, int bf16, const float* ksum, int B,
                                         int Hq, int Hkv, int N, int d, int topk, float scale,
                                         int32_t* idx, int32_t* cnt, float* logg,
                                         cudaStream_t st) {
  float* qbar = nullptr;
  cudaError_t e = static_qbar_address(&qbar);
  if (e != cudaSuccess) return e;
  return launch_select_prefill(q, bf16, ksum, B, Hq, Hkv, N, d, topk, scale, idx, cnt, logg,
                               nullptr, qbar, st);
}

// ------------------------------------------------------------------ decode
// Scratch layout per plan (rows = B*Hkv, nchunk chunks per row):
//   counters [rows] int | len [rows][nchunk] int | cmax, csum [rows][nchunk]
//   float | keys [rows][nchunk][k] u64
struct DecodeSelectWs {
  int* counter;
  int* len;
  float* cmax;
  float* csum;
  unsigned long long* lk;
};

static size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

static DecodeSelectWs carve_decode_select(int* counters, void* ws, const SelectPlan& p) {
  DecodeSelectWs w;
  char* c = static_cast<char*>(ws);
  const size_t rc = (size_t)p.rows * p.nchunk;
  w.counter = counters;
  w.len = reinterpret_cast<int*>(c); c += align16(sizeof(int) * rc);
  w.cmax = reinterpret_cast<float*>(c); c += align16(sizeof(float) * rc);
  w.csum = reinterpret_cast<float*>(c); c += align16(sizeof(float) * rc);
  w.lk = reinterpret_cast<unsigned long long*>(c);
  return w;
}

size_t decode_select_ws_bytes(const SelectPlan& p) {
  const size_t rc = (size_t)p.rows * p.nchunk;
  return align16(sizeof(int) * rc) + 2 * align16(sizeof(float) * rc) +
         align16(sizeof(unsigned long long) * rc * p.topk);
}

SelectPlan plan_decode_select(int B, int Hkv, int Lmax, int topk) {
  SelectPlan p;
  p.rows = B * Hkv;
  p.topk = topk;
  const int nblk = Lmax / SAS_BLOCK;
  // Aim for about two CTAs per SM over all rows, chunks of 64..256 blocks.
  const long long target = 2LL * 148;
  int chunk = 64;
  while (chunk < DEC_CHUNK_MAX &&
         ((long long)p.rows * ((nblk + chunk - 1) / chunk) > target ||
          (nblk + chunk - 1) / chunk > DEC_NCHUNK_MAX))
    chunk *= 2;
  p.chunk = chunk;
  p.nchunk = nblk > 0 ? (nblk + chunk - 1) / chunk : 1;
  return p;
}

static size_t decode_merge_smem(int nchunk, int topk) {
  const size_t nck = (nchunk + 3) & ~3;
  return sizeof(float) * 4 * nck + 2 * 8 * ((size_t)nchunk << ceil_log2(topk));
}

template <typename T, int D>
__global__ void __launch_bounds__(SEL_THREADS) k_select_decode(
    const T* __restrict__ q, const float* __restrict__ ksum, int Hq, int Hkv, int nblk,
    const int32_t* __restrict__ lens, int topk, float scale, int chunk, DecodeSelectWs w,
    int32_t* __restrict__ idx, int32_t* __restrict__ cnt, float* __restrict__ logg,
    float* __restrict__ scores) {
  __shared__ __align__(16) float q_s[D];
  __shared__ float sc[DEC_CHUNK_MAX];
  __shared__ float red[32];
  __shared__ int is_last;
  // merge staging (last CTA of a row): the row's chunk partials and lists
  extern __shared__ __align__(16) unsigned char dsm[];
  const int c = blockIdx.x, r = blockIdx.y, b = blockIdx.z;
  const int nchunk = gridDim.x;
  const int G = Hq / Hkv;
  const int row = b * Hkv + r;
  // A programmatic dependent (the decode attention) may be scheduled now and
  // load what does not depend on this grid; it waits for this grid's
  // completion, with every write visible, before it reads the selection.
  grid_dep_launch();
  const int n_tok = min(max(lens[b], 1), nblk * SAS_BLOCK);  // 1 <= n <= Lmax
  const int C = (n_tok - 1) / SAS_BLOCK;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    float s = 0.f;
    for (int g = 0; g < G; ++g) s += to_f(q[((size_t)b * Hq + r * G + g) * D + i]);
    q_s[i] = s / (float)G;
  }
  __syncthreads();
  const int m0 = c * chunk, n = max(0, min(chunk, C - m0));
  const float* ks_row = ksum + (size_t)row * nblk * D;
  float* gs = scores != nullptr ? scores + (size_t)row * nblk : nullptr;  // [nblk] of this row
  if (gs != nullptr)
    for (int m = max(C, m0) + threadIdx.x; m < min(m0 + chunk, nblk); m += blockDim.x)
      gs[m] = -INFINITY;
  score_chunk<D>(ks_row, m0, n, q_s, scale, sc, gs);
  __syncthreads();
  const size_t rc = (size_t)row * nchunk + c;
  if (topk > 0) chunk_topk(sc, m0, n, topk, w.lk + rc * topk);
  float lm = -FLT_MAX;
  for (int i = threadIdx.x; i < n; i += blockDim.x) lm = fmaxf(lm, sc[i]);
  lm = block_reduce_max(lm, red);
  float le = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) le += __expf(sc[i] - lm);
  le = block_reduce_sum(le, red);
  if (threadIdx.x == 0) {
    w.len[rc] = min(topk, n);
    w.cmax[rc] = lm;
    w.csum[rc] = le;
  }
  // Publish this chunk, then count it; the last chunk of the row merges.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(w.counter + row, 1) == nchunk - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // Stage the row's partials in shared memory with one parallel pass of L2
  // loads, then merge there (a serial walk over L2 would be latency-bound).
  const int nck = (nchunk + 3) & ~3;
  float* cm_s = reinterpret_cast<float*>(dsm);
  float* cs_s = cm_s + nck;
  int* len_s = reinterpret_cast<int*>(cs_s + nck);
  int* len_b = len_s + nck;
  const int lg = ceil_log2(topk);
  unsigned long long* la = reinterpret_cast<unsigned long long*>(len_b + nck);
  unsigned long long* lb = la + ((size_t)nchunk << lg);
  const size_t r0 = (size_t)row * nchunk;
  for (int i = threadIdx.x; i < nchunk; i += blockDim.x) {
    cm_s[i] = __ldcg(w.cmax + r0 + i);  // empty chunks: -FLT_MAX and 0
    cs_s[i] = __ldcg(w.csum + r0 + i);
    len_s[i] = __ldcg(w.len + r0 + i);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < nchunk * topk; e += blockDim.x) {
    const int cc = e / topk, p = e - cc * topk;
    if (p < len_s[cc]) la[((size_t)cc << lg) + p] = __ldcg(w.lk + r0 * topk + e);
  }
  float mx = -FLT_MAX;
  for (int i = threadIdx.x; i < nchunk; i += blockDim.x) mx = fmaxf(mx, cm_s[i]);
  const float M = block_reduce_max(mx, red);
  float lsum = 0.f;
  for (int i = threadIdx.x; i < nchunk; i += blockDim.x)
    if (cs_s[i] > 0.f) lsum += cs_s[i] * __expf(cm_s[i] - M);
  const float S = block_reduce_sum(lsum, red);
  const float lse = (C > 0) ? M + __logf(S) : 0.f;
  const int kk = min(topk, C);
  if (topk > 0) {
    __syncthreads();
    const int wb = tree_merge(la, len_s, lb, len_b, nchunk, lg, topk);
    write_selection(wb ? lb : la, kk, topk, lse, idx + (size_t)row * topk,
                    logg + (size_t)row * topk);
  }
  if (threadIdx.x == 0) {
    cnt[row] = kk;
    w.counter[row] = 0;  // ready for the next call
  }
}

cudaError_t launch_select_decode(const void* q, int bf16, const float* ksum, int B, int Hq,
                                 int Hkv, int Lmax, int d, int topk, const int32_t* lens,
                                 float scale, int32_t* idx, int32_t* cnt, float* logg,
                                 float* scores, const SelectPlan& plan, int* counters, void* ws,
                                 cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  DecodeSelectWs w = carve_decode_select(counters, ws, plan);
  const int nblk = Lmax / SAS_BLOCK;
  dim3 grid(plan.nchunk, Hkv, B);
const size_t smem = decode_merge_smem(plan.nchunk, topk);
#define SAS_SELD(T, D)                                                                       \
  do {                                                                                       \
    ensure_smem(k_select_decode<T, D>, smem);                                                \
    k_select_decode<T, D><<<grid, SEL_THREADS, smem, st>>>(static_cast<const T*>(q), ksum,   \
                                                           Hq, Hkv, nblk, lens, topk, scale, \
                                                           plan.chunk, w, idx, cnt, logg,    \
                                                           scores);                          \
  } while (0)
  if (bf16) {
    if (d == 128) SAS_SELD(__nv_bfloat16, 128); else SAS_SELD(__nv_bfloat16, 64);
  } else {
    if (d == 128) SAS_SELD(float, 128); else SAS_SELD(float, 64);
  }
#undef SAS_SELD
  return cudaGetLastError();
}

}  // namespace sas
