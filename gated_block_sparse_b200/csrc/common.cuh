// Shared device helpers for the SAS kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <utility>

#define SAS_BLOCK 64

namespace sas {

// ---------------------------------------------------------------- numerics
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// 16-byte vector of T converted to fp32: 8 bf16 or 4 fp32 values.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float* out) {
    float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
  __device__ __forceinline__ static void load_nc(const float* p, float* out) {
    float4 v = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
  __device__ __forceinline__ static void store(float* p, const float* in) {
    *reinterpret_cast<float4*>(p) = make_float4(in[0], in[1], in[2], in[3]);
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void unpack(uint4 v, float* out) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* out) {
    unpack(*reinterpret_cast<const uint4*>(p), out);
  }
  __device__ __forceinline__ static void load_nc(const __nv_bfloat16* p, float* out) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), out);
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float* in) {
    uint4 v;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    v.x = w[0]; v.y = w[1]; v.z = w[2]; v.w = w[3];
    *reinterpret_cast<uint4*>(p) = v;
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Order key of a selection candidate: larger score first, then lower index.
// Returns true when (sa, ia) ranks ahead of (sb, ib).
__device__ __forceinline__ bool beats(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

// ---------------------------------------------------------------- Top-K lists
// Order key of a candidate block: larger score first, then lower block index,
// packed into one unsigned 64-bit integer (larger key = better candidate).
// A -0 score must be stored as +0 beforehand so that exact ties are equal.
__device__ __forceinline__ unsigned long long cand_key(float s, int m) {
  uint32_t u = __float_as_uint(s);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // order-preserving map
  return ((unsigned long long)u << 32) | (0xffffffffu - (uint32_t)m);
}

__device__ __forceinline__ float key_score(unsigned long long key) {
  const uint32_t u = (uint32_t)(key >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
__device__ __forceinline__ int key_block(unsigned long long key) {
  return (int)(0xffffffffu - (uint32_t)key);
}

// Pairwise tree merge of nl best-first candidate lists of keys in shared
// memory (list l: len[l] keys at A + (l << lg), i.e. a power-of-two stride
// 2^lg >= k) into one best-first list of the min(k, total) best keys, left
// in list 0 of the buffer it returns (0 = A, 1 = B). Each level merges lists
// 2i and 2i+1: a key at position p of one list has rank p plus the number of
// keys of the other list that are larger (one binary search); ranks below k
// are kept. Keys are unique, so ranks never collide. All threads of the
// block must call it.
__device__ inline int tree_merge(unsigned long long* A, int* Alen, unsigned long long* B, int* Blen,
                                 int nl, int lg, int k) {
  int which = 0;
  const int stride = 1 << lg;
  while (nl > 1) {
    const unsigned long long* src = which ? B : A;
    const int* sl = which ? Blen : Alen;
    unsigned long long* dst = which ? A : B;
    int* dl = which ? Alen : Blen;
    const int npairs = (nl + 1) >> 1;
    for (int e = threadIdx.x; e < (nl << lg); e += blockDim.x) {
      const int l = e >> lg, p = e & (stride - 1);
      if (p >= sl[l]) continue;
      const unsigned long long key = src[e];
      const int partner = l ^ 1;
      int rank = p;
      if (partner < nl) {
        const unsigned long long* ps = src + (partner << lg);
        int lo = 0, hi = sl[partner];
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (ps[mid] > key) lo = mid + 1; else hi = mid;
        }
        rank += lo;
      }
      if (rank < k) dst[((l >> 1) << lg) + rank] = key;
    }
    for (int o = threadIdx.x; o < npairs; o += blockDim.x) {
      const int a = sl[2 * o], b2 = (2 * o + 1 < nl) ? sl[2 * o + 1] : 0;
      dl[o] = min(k, a + b2);
    }
    __syncthreads();
    which ^= 1;
    nl = npairs;
  }
  return which;
}

// Top-k of nl <= 32 descending lists of unique 64-bit keys (list l at
// A[l << lg], len[l] <= 2^lg entries) into out[0 .. min(k, sum len) - 1],
// descending. The pruning threshold is the largest k-th key among the lists
// that hold k keys: a key below it has at least k keys above it. Keys at or
// above it are compacted into tmp; when at most 512 survive, each survivor
// counts the survivors above it, which is its global rank (every key above a
// survivor is a survivor). Otherwise the lists are merged pairwise
// (tree_merge over A and B, whose length arrays it overwrites). *cnt is 0 on
// entry; th_s is one shared word for the threshold. All threads of the
// block call it; it ends with a barrier.
__device__ inline void topk_of_lists(unsigned long long* A, int* len, int nl, int lg, int k,
                                     unsigned long long* out, unsigned long long* tmp,
                                     unsigned long long* B, int* Blen, int* cnt,
                                     unsigned long long* th_s) {
  const int kq = 1 << lg;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {  // one warp finds the threshold; the block reads it back
    unsigned long long th = 0;
    if (lane < nl && k > 0 && len[lane] >= k) th = A[(lane << lg) + k - 1];
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      const unsigned long long w = __shfl_xor_sync(0xffffffffu, th, off);
      th = w > th ? w : th;
    }
    // A tighter bound when k <= 32: the k-th largest of the 32 keys made of
    // each list's first 32/nl' entries (nl' = nl rounded up to a power of
    // two) is also at most the k-th largest of all keys. Each lane counts the
    // keys of that sample above its own.
    if (k <= 32) {
      int nlp = 1;
      while (nlp < nl) nlp <<= 1;
      const int m = 32 / nlp, l = lane / m, p = lane % m;
      const unsigned long long mine = (l < nl && p < len[l]) ? A[(l << lg) + p] : 0ull;
      int above = 0;
#pragma unroll 8
      for (int j = 0; j < 32; ++j) above += __shfl_sync(0xffffffffu, mine, j) > mine;
      const unsigned hit = __ballot_sync(0xffffffffu, mine != 0ull && above == k - 1);
      if (hit) {
        const unsigned long long kth = __shfl_sync(0xffffffffu, mine, __ffs(hit) - 1);
        th = kth > th ? kth : th;
      }
    }
    if (lane == 0) *th_s = th;
  }
  __syncthreads();
  const unsigned long long th = *th_s;
  const int total = nl << lg;
  for (int e0 = 0; e0 < total; e0 += blockDim.x) {
    const int e = e0 + (int)threadIdx.x;
    bool keep = false;
    unsigned long long key = 0;
    if (e < total && (e & (kq - 1)) < len[e >> lg]) {
      key = A[e];
      keep = key >= th;
    }
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    int base = 0;
    if (lane == 0 && m) base = atomicAdd(cnt, __popc(m));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (keep) tmp[base + __popc(m & ((1u << lane) - 1u))] = key;
  }
  __syncthreads();
  const int S = *cnt;
  if (S <= 512) {
    for (int i = threadIdx.x; i < S; i += blockDim.x) {
      const unsigned long long key = tmp[i];
      int rank = 0;
#pragma unroll 8
      for (int j = 0; j < S; ++j) rank += tmp[j] > key;
      if (rank < k) out[rank] = key;
    }
    __syncthreads();
    return;
  }
  const int which = tree_merge(A, len, B, Blen, nl, lg, k);
  const unsigned long long* res = which ? B : A;
  const int n0 = which ? Blen[0] : len[0];
  for (int i = threadIdx.x; i < n0; i += blockDim.x) out[i] = res[i];
  __syncthreads();
}

// log2 of the smallest power of two >= max(k, 1).
__host__ __device__ inline int ceil_log2(int k) {
  int lg = 0;
  while ((1 << lg) < k) ++lg;
  return lg;
}

// ---------------------------------------------------------------- PDL
// Programmatic dependent launch: a kernel launched with the programmatic
// stream serialization attribute may start before its predecessor ends.
// grid_dep_wait() blocks until every CTA of the predecessor has triggered
// (grid_dep_launch) or exited; only the predecessor's writes made before its
// trigger are guaranteed visible after it.
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- host
// Raises a kernel's dynamic shared memory limit once per (kernel, device), so
// that launches captured in a CUDA graph make no attribute calls.
template <typename Kern>
inline cudaError_t ensure_smem(Kern kern, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(reinterpret_cast<const void*>(kern), dev);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

}  // namespace sas
