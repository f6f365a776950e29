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

// Number of keys of v[0 .. n) above key (v 16-byte aligned, in shared
// memory): eight keys per step, loaded before they are compared, so that
// the loads of a step are in flight together.
__device__ __forceinline__ int count_above(const unsigned long long* v, int n,
                                           unsigned long long key) {
  int c = 0, j = 0;
  for (; j + 8 <= n; j += 8) {
    ulonglong2 w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) w[u] = *reinterpret_cast<const ulonglong2*>(v + j + 2 * u);
#pragma unroll
    for (int u = 0; u < 4; ++u) c += (w[u].x > key) + (w[u].y > key);
  }
  for (; j < n; ++j) c += v[j] > key;
  return c;
}

// Keys of a candidate set that are >= th, compacted into surv (512 keys at
// most) and ranked: each survivor counts the survivors above it, which is
// its rank in the whole set when every key above a survivor also survives
// (th is a lower bound of the k-th key). out[rank] = key for rank < k.
// key_of(e, key) gives candidate e < n (false: no candidate at e). Returns
// false, out untouched, when more than 512 keys survive. *cnt is 0 on entry.
// All threads of the block call it; it ends with a barrier.
template <typename KeyOf>
__device__ inline bool rank_survivors(KeyOf key_of, int n, unsigned long long th, int k,
                                      unsigned long long* out, unsigned long long* surv,
                                      int* cnt) {
  const int lane = threadIdx.x & 31;
  for (int e0 = 0; e0 < n; e0 += blockDim.x) {
    const int e = e0 + (int)threadIdx.x;
    unsigned long long key = 0;
    const bool keep = e < n && key_of(e, key) && key >= th;
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    int base = 0;
    if (lane == 0 && m) base = atomicAdd(cnt, __popc(m));
    base = __shfl_sync(0xffffffffu, base, 0);
    const int at = base + __popc(m & ((1u << lane) - 1u));
    if (keep && at < 512) surv[at] = key;
  }
  __syncthreads();
  const int S = *cnt;
  if (S > 512) return false;
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    const unsigned long long key = surv[i];
    const int rank = count_above(surv, S, key);
    if (rank < k) out[rank] = key;
  }
  __syncthreads();
  return true;
}

// Largest v over the block; every thread gets it. red holds one word per
// warp. All threads of the block call it (it holds one barrier), and red
// must not be rewritten before every thread has returned.
__device__ inline unsigned long long block_max_u64(unsigned long long v, unsigned long long* red) {
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, off);
    v = w > v ? w : v;
  }
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v = red[w] > v ? red[w] : v;
  return v;
}

// The k-th largest key of samp[0 .. ns) (0 marks an empty entry), returned
// by the thread that holds it (0 elsewhere, and everywhere when the sample
// holds fewer than k keys). A k-th largest key of any subset of a set is at
// most the set's k-th largest key, so it is a lower bound for the set.
__device__ inline unsigned long long sample_kth(const unsigned long long* samp, int ns, int k) {
  unsigned long long th = 0;
  for (int i = threadIdx.x; i < ns; i += blockDim.x) {
    const unsigned long long key = samp[i];
    if (key != 0ull && count_above(samp, ns, key) == k - 1) th = key;
  }
  return th;
}

// Number of keys greater than x in the descending lists l < nl, l != skip
// (list l at A + (l << lg); only its first lim[l] <= 2^slg entries are
// searched; lim[l] = 0 for l >= nl). One branch-free binary search per
// list; the searches advance step by step together and every load is
// unconditional (an index past lim reads entry 0 of a valid list and is
// ignored), so that each step's loads are in flight at once.
template <int NL>
__device__ __forceinline__ int count_greater_lists(const unsigned long long* A,
                                                   const int (&lim)[NL], int nl, int lg, int slg,
                                                   int skip, unsigned long long x) {
  int pos[NL];
#pragma unroll
  for (int l = 0; l < NL; ++l) pos[l] = 0;
  for (int step = (1 << slg) >> 1; step >= 1; step >>= 1) {
#pragma unroll
    for (int l = 0; l < NL; ++l) {
      const int i = pos[l] + step - 1;
      const bool in = i < lim[l];
      const unsigned long long v = A[((l < nl ? l : 0) << lg) + (in ? i : 0)];
      pos[l] += (in && v > x) ? step : 0;
    }
  }
  int r = 0;
#pragma unroll
  for (int l = 0; l < NL; ++l) {
    const int i = pos[l];
    const bool in = i < lim[l];
    const unsigned long long v = A[((l < nl ? l : 0) << lg) + (in ? i : 0)];
    pos[l] += (in && v > x) ? 1 : 0;
    r += (l != skip) ? pos[l] : 0;
  }
  return r;
}

// Top-k of nl <= NL descending lists of unique 64-bit keys (list l at
// A[l << lg], len[l] <= 2^lg entries) into out[0 .. min(k, sum len) - 1],
// descending. The rank of the key at position p of list l is p plus, for
// every other list, the number of its keys above it (a binary search), so
// each key finds its place on its own. When the lists hold more slots than
// the block has threads, the keys ranked are first cut to those at or above
// a lower bound of the k-th key: the k-th largest key of the sample made of
// each list's first m entries (m a power of two with nl m >= 2k where the
// lists allow; a k-th largest key of a subset is at most the set's), found
// by the same ranking within the sample. Slots are visited position-major
// (thread t takes list t % NL), so that the few keys above the bound, at the
// head of every list, share the first pass. NL is a power of two. *th_s is 0
// on entry. All threads of the block call it; it ends with a barrier.
template <int NL>
__device__ inline void topk_of_lists(const unsigned long long* A, const int* len, int nl, int lg,
                                     int k, unsigned long long* out, unsigned long long* th_s) {
  static_assert((NL & (NL - 1)) == 0, "NL must be a power of two");
  const int kq = 1 << lg;
  int ln[NL];
#pragma unroll
  for (int l = 0; l < NL; ++l) ln[l] = l < nl ? len[l] : 0;
  unsigned long long th = 0;
  if ((nl << lg) > (int)blockDim.x) {
    int lm = 0;
    while ((nl << lm) < 2 * k && lm < lg && (nl << (lm + 1)) <= (int)blockDim.x) ++lm;
    const int t = threadIdx.x, l = t >> lm, p = t & ((1 << lm) - 1);
    if (t < (nl << lm) && p < len[l]) {
      int lim[NL];
#pragma unroll
      for (int l2 = 0; l2 < NL; ++l2) lim[l2] = min(ln[l2], 1 << lm);
      const unsigned long long x = A[(l << lg) + p];
      if (p + count_greater_lists<NL>(A, lim, nl, lg, lm, l, x) == k - 1) *th_s = x;
    }
    __syncthreads();
    th = *th_s;
  }
  for (int e0 = 0; e0 < NL * kq; e0 += blockDim.x) {
    const int e = e0 + (int)threadIdx.x, l = e & (NL - 1), p = e / NL;
    if (e < NL * kq && l < nl && p < len[l]) {
      const unsigned long long x = A[(l << lg) + p];
      if (x >= th) {
        const int r = p + count_greater_lists<NL>(A, ln, nl, lg, lg, l, x);
        if (r < k) out[r] = x;
      }
    }
  }
  __syncthreads();
}

// Sorts a bitonic sequence of P = 2^lg keys into descending order: P <= 32
// keys one per lane of an aligned group of P lanes (j = lane % P), or
// P = 32 E keys E per lane (key e * 32 + lane in v[e]). Every lane of the
// warp calls it.
template <int EMAX>
__device__ __forceinline__ void bitonic_clean_desc(unsigned long long (&v)[EMAX], int lg) {
  const int P = 1 << lg, lane = threadIdx.x & 31;
  for (int stride = P >> 1; stride > 0; stride >>= 1) {
    if (stride >= 32) {
      const int se = stride >> 5;
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if ((e & se) == 0 && e + se < EMAX) {
          const unsigned long long a = v[e], b = v[e + se];
          v[e] = a > b ? a : b;
          v[e + se] = a > b ? b : a;
        }
    } else {
      const bool lower = (lane & stride) == 0;
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, v[e], stride);
        v[e] = (lower == (v[e] > y)) ? v[e] : y;
      }
    }
  }
}

// Top-k of nl descending lists of unique nonzero 64-bit keys (list l at
// A[l << lg], len[l] <= P = 2^lg keys) into out[0 .. min(k, sum len) - 1],
// descending, by a tree of pairwise merges. The top P keys of two
// descending lists a and b are max(a[i], b[P - 1 - i]), i < P (a bitonic
// sequence; a missing key counts as 0), which log2 P bitonic stages sort.
// For P < 32 a warp holds 32 / P lists, one per group of P lanes: it loads
// twice as many, merges them pairwise, then merges its groups pairwise
// through shuffles, so that each barrier level reduces 64 / P lists to one;
// for P >= 32 a warp merges one pair (P / 32 keys per lane). A and B (B with
// room for ceil(nl / 2) lists) are ping-pong buffers; both are overwritten.
// EMAX >= P / 32. All threads of the block call it; it ends with a barrier.
template <int EMAX>
__device__ inline void merge_tree_topk(unsigned long long* A, int* len, unsigned long long* B,
                                       int* Blen, int nl, int lg, int k,
                                       unsigned long long* out) {
  const int P = 1 << lg, lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  const int U = P < 32 ? 32 / P : 1;  // groups (lists held) per warp
  const int g = lane / (P < 32 ? P : 32), j = P < 32 ? lane % P : lane;
  unsigned long long* src = A;
  unsigned long long* dst = B;
  int* sl = len;
  int* dl = Blen;
  while (nl > 1) {
    const int nout = (nl + 2 * U - 1) / (2 * U);
    for (int o = wid; o < nout; o += nw) {  // output list o from inputs [2 U o, 2 U o + 2 U)
      const int la = 2 * (U * o + g), lb = la + 1;
      const int na = la < nl ? sl[la] : 0, nb = lb < nl ? sl[lb] : 0;
      unsigned long long v[EMAX];
#pragma unroll
      for (int e = 0; e < EMAX; ++e) {
        const int i = e * 32 + j;
        unsigned long long a = 0, b = 0;
        if (i < P) {
          if (i < na) a = src[(la << lg) + i];
          if (P - 1 - i < nb) b = src[(lb << lg) + P - 1 - i];
        }
        v[e] = a > b ? a : b;
      }
      bitonic_clean_desc<EMAX>(v, lg);
      int cnt = min(P, na + nb);
      for (int h = 1; h < U; h <<= 1) {  // merge group g with group g + h (P < 32 only)
        const unsigned long long y =
            __shfl_sync(0xffffffffu, v[0], ((g ^ h) * P) + (P - 1 - j));
        v[0] = v[0] > y ? v[0] : y;
        bitonic_clean_desc<EMAX>(v, lg);
        cnt = min(P, cnt + __shfl_sync(0xffffffffu, cnt, (g ^ h) * P));
      }
      if (g == 0) {
#pragma unroll
        for (int e = 0; e < EMAX; ++e)
          if (e * 32 + j < P) dst[(o << lg) + e * 32 + j] = v[e];
        if (lane == 0) dl[o] = cnt;
      }
    }
    __syncthreads();
    unsigned long long* t = src;
    src = dst;
    dst = t;
    int* tl = sl;
    sl = dl;
    dl = tl;
    nl = nout;
  }
  const int n0 = min(k, nl > 0 ? sl[0] : 0);
  for (int i = threadIdx.x; i < n0; i += blockDim.x) out[i] = src[i];
  __syncthreads();
}

// Sorts 64 keys held two per lane (element 32 j + lane in v[j]) into
// descending order across the warp: a bitonic network, strides below 32
// across lanes by shuffles, stride 32 inside the lane.
__device__ __forceinline__ void warp_sort64_desc(unsigned long long (&v)[2]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride == 32) {
        const unsigned long long a = v[0], b = v[1];
        v[0] = a > b ? a : b;
        v[1] = a > b ? b : a;
      } else {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const unsigned long long y = __shfl_xor_sync(0xffffffffu, v[j], stride);
          const bool keep_max = ((lane & stride) == 0) == (((j * 32 + lane) & size) == 0);
          v[j] = keep_max ? (v[j] > y ? v[j] : y) : (v[j] < y ? v[j] : y);
        }
      }
    }
  }
}

// log2 of the smallest power of two >= max(k, 1).
__host__ __device__ inline int ceil_log2(int k) {
  int lg = 0;
  while ((1 << lg) < k) ++lg;
  return lg;
}

// ---------------------------------------------------------------- PDL
// Programmatic dependent launch: a kernel launched with the programmatic
// stream serialization attribute may be scheduled before its predecessor
// ends, once every CTA of the predecessor has called grid_dep_launch() or
// exited (without a call, at the predecessor's completion). The trigger only
// decides that early scheduling. grid_dep_wait() blocks until the predecessor
// grids have completed and their memory operations are visible, so every
// write of the predecessor, before or after its trigger, is seen after it.
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
