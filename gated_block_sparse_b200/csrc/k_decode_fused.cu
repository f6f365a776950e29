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
// Cluster of CS CTAs (16 when the rows fit the GPU that way, else fewer).
// CTA c of the cluster:
//   1. bulk-copies its contiguous range of the row's block summaries through
//      a four-slot shared-memory ring and scores them against qbar (mean of
//      the group's query heads); the current block's K/V, known before any
//      selection, is copied by the CTA that owns it as soon as the ring is
//      free, under the selection;
//   2. reduces its range to (max, sum exp) and a best-first list of
//      min(k, n) candidates (rank counting for short ranges, per-warp
//      register bitonic sorts and a bitonic merge tree for ranges up to 512,
//      and beyond that the keys at or above the k-th key of a strided sample,
//      ranked among themselves), and stores both into its slot of every CTA
//      of the cluster with asynchronous remote stores that complete on the
//      receiver's mbarrier;
//   3. once all lists have landed, every CTA computes the gate's LSE and the
//      same Top-K with a tree of bitonic merges of the CS sorted lists,
//      giving the kept blocks in score order (CTA 0 also writes them in
//      ascending block order to idx_out);
//   4. streams the K/V blocks of its share of the units (the current block
//      first, then kept blocks in score order) through a ring that reuses
//      the summary ring.
//      Each warp takes 8 keys of every unit and keeps its own online-softmax
//      state (m, l, acc) for every head of the group, so no CTA-wide barrier
//      runs per unit. bf16 caches: the K/V tiles arrive by TMA as 64-column
//      boxes with the 128-byte swizzle, and q.k and p.v are warp MMAs
//      (mma.sync m16n8k16 / m16n8k8, fp32 accumulation) with the group's
//      heads as the rows of the A operand and P reused as the A operand of
//      p.v in the layout the q.k accumulator leaves it; fp32 caches: CUDA
//      cores;
//   5. folds the warp states into one per head and stores head h's state
//      into CTA h (remote stores on CTA h's mbarrier); CTA h < G combines the
//      CS states (exact LSE rescaling) and writes o.
// Data moves between CTAs only by remote stores that complete on the
// receiver's mbarrier, so every read is local. A cluster barrier after the
// barrier initialisation orders the first remote store, and one at exit
// keeps every CTA resident until all stores into it are done. No global
// scratch, atomics or memsets; every wait is bounded.
#include <cooperative_groups.h>
#include <cuda.h>
#include <float.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace sas {

__device__ uint32_t g_decode_fused_err = 0;

namespace {

constexpr int FD_THREADS = 256;
constexpr int FD_WARPS = FD_THREADS / 32;
constexpr int FD_NS = 4;      // summary ring slots
constexpr int FD_MAXKV = 4;   // K/V ring slots at most
constexpr int FD_MAXCS = 16;  // cluster size at most
constexpr int FD_BIG_REGION = 192 * 1024;  // ring region with one CTA per SM
constexpr size_t FD_SMEM_MAX = 226 * 1024; // dynamic shared memory per CTA at most
constexpr unsigned FULL = 0xffffffffu;

struct FdSmem {  // byte offsets into dynamic shared memory
  size_t u, q, qf, qbar, sc, mine, slen, stage, sstat, fin, cst, cml, zp, bars, total;
  size_t wl, wb, samp, surv;                  // list scratch inside region u, after K/V slot 0
  int nkv;                                    // K/V ring slots held by region u
  int subc;                                   // summaries per ring slot
};

__host__ __device__ inline size_t fd_al(size_t x) { return (x + 127) & ~(size_t)127; }

// Region u: the summary ring (FD_NS equal slots over the whole region)
// during the scan; then K/V slot 0 (the current block) followed by the list
// scratch (warp lists, sample, survivors, merge buffer) during selection;
// K/V slots 0 .. nkv-1 afterwards; the per-warp states at the end.
// ub_min: the region's size at least (0: two K/V slots, sized for two CTAs
// per SM; larger when the grid leaves one CTA per SM, for deeper rings).
__host__ __device__ inline FdSmem fd_layout(int D, int G, int es, int per, int kq, int CS,
                                             int ses, size_t ub_min = 0) {
  FdSmem L;
  const size_t kvslot = (size_t)2 * SAS_BLOCK * D * es;
  L.wl = kvslot;
  L.wb = L.wl + (size_t)FD_WARPS * kq * 8;
  L.samp = fd_al(L.wb + (size_t)FD_WARPS * kq * 8);
  L.surv = L.samp + 256 * 8;
  size_t ub = 2 * kvslot;
  if (ub < ub_min) ub = ub_min;
  if (ub < L.surv + 512 * 8) ub = L.surv + 512 * 8;
  const size_t comb = (size_t)FD_WARPS * G * (D + 2) * 4;
  if (ub < comb) ub = comb;
  L.nkv = (int)(ub / kvslot);
  if (L.nkv > FD_MAXKV) L.nkv = FD_MAXKV;
  L.subc = (int)(ub / ((size_t)FD_NS * D * ses));
  size_t o = 0;
  L.u = o; o += fd_al(ub);
  L.q = o; o += fd_al((size_t)G * D * 4);
  L.qf = o; o += fd_al((size_t)(D / 16) * 2 * 32 * 4);  // q as warp-MMA A fragments (bf16)
  L.qbar = o; o += fd_al((size_t)D * 4);
  L.sc = o; o += fd_al((size_t)(per > 0 ? per : 1) * 4);
  L.mine = o; o += fd_al((size_t)kq * 8);
  L.slen = o; o += fd_al((size_t)CS * 4);
  L.stage = o; o += fd_al((size_t)CS * kq * 8);
  L.sstat = o; o += fd_al((size_t)CS * 8);
  L.fin = o; o += fd_al((size_t)kq * 8);
  L.cst = o; o += fd_al((size_t)CS * D * 4);
  L.cml = o; o += fd_al((size_t)CS * 8);
  L.zp = o; o += fd_al((size_t)FD_WARPS * 2 * 8 * G * 4);  // per warp: z and p of its 8 keys
  L.bars = o; o += fd_al((size_t)(FD_NS + 2 * FD_MAXKV + 2) * 8);
  L.total = o;
  return L;
}

// N consecutive elements (N = 2 or 4) as fp32.
template <int N>
__device__ __forceinline__ void loadn(const __nv_bfloat16* p, float (&v)[N]) {
  if constexpr (N == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  } else {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    v[0] = a.x; v[1] = a.y;
  }
}
template <int N>
__device__ __forceinline__ void loadn(const float* p, float (&v)[N]) {
  if constexpr (N == 4) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else {
    const float2 a = *reinterpret_cast<const float2*>(p);
    v[0] = a.x; v[1] = a.y;
  }
}

// G consecutive fp32 values from shared memory (16-byte loads when G % 4 == 0).
template <int G>
__device__ __forceinline__ void loadg(const float* p, float (&v)[G]) {
  if constexpr (G % 4 == 0) {
#pragma unroll
    for (int i = 0; i < G; i += 4) {
      const float4 a = *reinterpret_cast<const float4*>(p + i);
      v[i] = a.x; v[i + 1] = a.y; v[i + 2] = a.z; v[i + 3] = a.w;
    }
  } else if constexpr (G == 2) {
    const float2 a = *reinterpret_cast<const float2*>(p);
    v[0] = a.x; v[1] = a.y;
  } else {
#pragma unroll
    for (int i = 0; i < G; ++i) v[i] = p[i];
  }
}

// (a0, a1) += (x0, x1) * (y0, y1) as one packed fp32x2 FMA (sm_100).
__device__ __forceinline__ void fma2(float& a0, float& a1, float x0, float x1, float y0, float y1) {
  asm("{\n\t.reg .b64 a, x, y;\n\t"
      "mov.b64 a, {%0, %1};\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 y, {%4, %5};\n\t"
      "fma.rn.f32x2 a, x, y, a;\n\t"
      "mov.b64 {%0, %1}, a;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x0), "f"(x1), "f"(y0), "f"(y1));
}

// One stage of a transposing warp reduction over CNT values per lane: lanes
// with bit `o` set keep the upper half of the values, the others the lower
// half, and each adds its partner's copy of the half it keeps.
template <int CNT>
__device__ __forceinline__ void tr_stage(float* v, int lane, int o) {
  constexpr int H = CNT / 2;
  const bool up = (lane & o) != 0;
#pragma unroll
  for (int i = 0; i < H; ++i) {
    const float send = up ? v[i] : v[i + H];
    const float keep = up ? v[i + H] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
  }
}

// Sums NV (8, 16 or 32) values over the warp's 32 lanes at once: lane l
// returns the total of value index l * NV / 32 (NV - 1 shuffles in all;
// with NV < 32 several lanes return the same total).
template <int NV>
__device__ __forceinline__ float transpose_sum(float (&v)[NV], int lane) {
  static_assert(NV == 8 || NV == 16 || NV == 32, "8, 16 or 32 values");
  tr_stage<NV>(v, lane, 16);
  tr_stage<NV / 2>(v, lane, 8);
  tr_stage<NV / 4>(v, lane, 4);
  if constexpr (NV >= 16) tr_stage<NV / 8>(v, lane, 2);
  else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
  if constexpr (NV == 32) tr_stage<2>(v, lane, 1);
  else v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
  return v[0];
}

// A step reads each summary and each kept K/V tile once: its copies carry an
// L2 evict-first policy, so that the streamed bytes do not push out of L2 what
// is reused from step to step (among it the kernel's own instructions).
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void bulk_g2s_once(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(l2_evict_first())
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_once(void* dst, const CUtensorMap* map, int c0,
                                                 int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)),
      "l"(l2_evict_first())
      : "memory");
}

// Warp MMAs on bf16 operands with fp32 accumulation (c += a b).
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
// m16n8k8 with the A operand's rows 8..15 zero: c2, c3 (rows 8..15 of the
// result) pass through unchanged, so every call can share one zero pair.
__device__ __forceinline__ void mma_1688(float (&c)[2], float& z2, float& z3, uint32_t a0,
                                         uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(z2), "+f"(z3)
      : "r"(a0), "r"(0u), "r"(b0));
}
// Four transposed 8 x 8 bf16 matrices; lane l gives the address of row l % 8
// of matrix l / 8.
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Byte offset of element (row, col) of a bf16 [64][D] tile stored as
// 64-column boxes of [64 rows][128 B] with the 128-byte swizzle (16-byte
// chunk c of row r at chunk c ^ (r % 8)), as the tensor-map loads leave it.
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
  return (uint32_t)((col >> 6) * 8192 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                    (col & 7) * 2);
}

// Combines two (max, sum exp) pairs; an empty pair is (-FLT_MAX, 0).
__device__ __forceinline__ void ms_merge(float& m, float& s, float m2, float s2) {
  const float M = fmaxf(m, m2);
  s = s * __expf(m - M) + s2 * __expf(m2 - M);
  m = M;
}

}  // namespace

// PAGED: the caches are pools of 64-token pages, [npages][Hkv][64][D], the
// summaries [npages][Hkv][D], and bt [B][max_blocks] maps a sequence's
// logical block to its page (Lmax = 64 max_blocks). Otherwise kc, vc are
// [B][Hkv][Lmax][D] and ksum [B][Hkv][Lmax/64][D].
// S: the summaries' element type (float, or bf16 for half the scan bytes).
template <typename T, int D, int G, bool PAGED, typename S>
__global__ void __launch_bounds__(FD_THREADS, 2) k_decode_fused(
    const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
    const S* __restrict__ ksum, int Hkv, int Lmax, const int32_t* __restrict__ lens, int topk,
    int gated, float scale, int per_max, int ub_min, T* __restrict__ o,
    int32_t* __restrict__ idx_out, const int32_t* __restrict__ bt, int npages,
    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap) {
  // bf16 caches: K/V tiles by TMA (swizzled) and warp MMAs; fp32: bulk copies, CUDA cores
  constexpr bool TMA_KV = std::is_same<T, __nv_bfloat16>::value;
  constexpr int TILE = SAS_BLOCK * D;
  constexpr int VEC = Vec16<T>::N;     // elements per 16-byte vector
  constexpr int CPL = D / 32;          // output columns per lane
  constexpr int PER = D / 32;          // summary elements per lane
  extern __shared__ __align__(1024) unsigned char sm[];
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int lg = ceil_log2(topk > 0 ? topk : 1);
  const int kq = 1 << lg;  // list stride (power of two)
  const FdSmem L = fd_layout(D, G, (int)sizeof(T), per_max, kq, CS, (int)sizeof(S), ub_min);
  unsigned char* U = sm + L.u;
  const size_t kvslot = (size_t)2 * TILE * sizeof(T);
  S* ring = reinterpret_cast<S*>(U);
  const int SUBC = L.subc;
  float* q_s = reinterpret_cast<float*>(sm + L.q);
  float* qbar = reinterpret_cast<float*>(sm + L.qbar);
  float* sc = reinterpret_cast<float*>(sm + L.sc);
  unsigned long long* wl = reinterpret_cast<unsigned long long*>(U + L.wl);
  unsigned long long* wb = reinterpret_cast<unsigned long long*>(U + L.wb);
  unsigned long long* samp = reinterpret_cast<unsigned long long*>(U + L.samp);
  unsigned long long* surv = reinterpret_cast<unsigned long long*>(U + L.surv);
  unsigned long long* mine = reinterpret_cast<unsigned long long*>(sm + L.mine);
  int* slen = reinterpret_cast<int*>(sm + L.slen);
  unsigned long long* stage = reinterpret_cast<unsigned long long*>(sm + L.stage);
  float* sstat = reinterpret_cast<float*>(sm + L.sstat);
  unsigned long long* fin = reinterpret_cast<unsigned long long*>(sm + L.fin);
  float* cst = reinterpret_cast<float*>(sm + L.cst);
  float* cml = reinterpret_cast<float*>(sm + L.cml);
  float* zp = reinterpret_cast<float*>(sm + L.zp);
  uint64_t* sum_bar = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* full = sum_bar + FD_NS;
  uint64_t* empty = full + FD_MAXKV;
  uint64_t* list_bar = empty + FD_MAXKV;
  uint64_t* state_bar = list_bar + 1;
  __shared__ float wred_m[FD_WARPS], wred_s[FD_WARPS];
  __shared__ int wlen[FD_WARPS], wlen_b[FD_WARPS];
  __shared__ int loc_cnt;
  __shared__ unsigned long long red8[FD_WARPS];
  __shared__ float cw[FD_MAXCS];                      // combine weights of the CS states
  __shared__ float2 mlw[8 * FD_WARPS];               // (m, l) per (head, warp) for the fold

  const int r = blockIdx.y, b = blockIdx.z;
  const int Hq = Hkv * G;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  // Programmatic dependent launch: the next kernel of the stream may be
  // scheduled now (it waits for this grid's completion before its own first
  // global read), and this grid reads nothing the previous one may still
  // write before that grid has completed.
  if (TMA_KV && (smem_u32(sm) & 1023u) != 0) {  // swizzled tiles need 1024-byte alignment
    if (tid == 0) atomicOr(&g_decode_fused_err, kErrBadIndex);
    return;  // every CTA of the launch sees the same alignment: no cluster barrier is left waiting
  }
  if (TMA_KV && tid == 0) {
    tc::prefetch_map(&kmap);
    tc::prefetch_map(&vmap);
  }
  grid_dep_launch();
  grid_dep_wait();
  // the group's queries and the sequence length first: both loads in flight together
  constexpr int QPT = (G * D + FD_THREADS - 1) / FD_THREADS;
  float qreg[QPT];
#pragma unroll
  for (int j = 0; j < QPT; ++j) {
    const int i = tid + j * FD_THREADS;
    qreg[j] = i < G * D ? to_f(q[((size_t)b * Hq + r * G) * D + i]) : 0.f;
  }
  const size_t row = (size_t)b * Hkv + r;
  const int nblk = Lmax / SAS_BLOCK;
  // This CTA's range of the row's history summaries: a split of the Lmax/64
  // blocks that does not depend on the sequence length, so that the first
  // copies start before the length is read. Blocks at or past C are copied
  // (contiguous caches) but not scored.
  const int per = per_max;
  const int m0 = crank * per;
  const int nstat = max(0, min(nblk, m0 + per) - m0);
  const int nsub_s = (nstat + SUBC - 1) / SUBC;
  const size_t kvrow = row * (size_t)Lmax * D;
  const S* ks_row = ksum + row * (size_t)nblk * D;
  uint32_t* err = &g_decode_fused_err;
  const int32_t* bt_row = PAGED ? bt + (size_t)b * nblk : nullptr;
  // page of logical block m (paged caches); an out-of-range entry is flagged
  // and replaced by page 0, so every copy stays inside the pools
  auto page_of = [&](int m) -> int {
    int p = bt_row[m];
    if (p < 0 || p >= npages) {
      atomicOr(err, kErrBadIndex);
      p = 0;
    }
    return p;
  };
  // K (or V) tile of logical block blk
  auto kv_tile = [&](const T* base, int blk) -> const T* {
    if constexpr (PAGED) return base + ((size_t)page_of(blk) * Hkv + r) * TILE;
    else return base + kvrow + (size_t)blk * TILE;
  };
  // K and V of logical block blk into a K/V slot (2 * TILE elements), both
  // completing on `bar`: TMA boxes (bf16) or two bulk copies (fp32)
  auto issue_kv = [&](unsigned char* dst, int blk, uint64_t* bar) {
    mbar_arrive_expect_tx(bar, (uint32_t)(2 * TILE * sizeof(T)));
    if constexpr (TMA_KV) {
      int plane, row0;
      if constexpr (PAGED) {
        plane = page_of(blk) * Hkv + r;
        row0 = 0;
      } else {
        plane = b * Hkv + r;
        row0 = SAS_BLOCK * blk;
      }
#pragma unroll
      for (int bx = 0; bx < D / 64; ++bx) {
        tma_load_3d_once(dst + bx * 8192, &kmap, 64 * bx, row0, plane, bar);
        tma_load_3d_once(dst + TILE * sizeof(T) + bx * 8192, &vmap, 64 * bx, row0, plane, bar);
      }
    } else {
      bulk_g2s_once(dst, kv_tile(kc, blk), TILE * sizeof(T), bar);
      bulk_g2s_once(dst + TILE * sizeof(T), kv_tile(vc, blk), TILE * sizeof(T), bar);
    }
  };
  // summaries [first, first + cnt) of this CTA's range into ring slot `slot`:
  // one bulk copy (contiguous), or one row copy per lane of warp 0 (paged)
  auto issue_summaries = [&](int slot, int first, int cnt) {
    S* dst = ring + (size_t)slot * SUBC * D;
    if constexpr (PAGED) {
      if (lane == 0) mbar_arrive_expect_tx(&sum_bar[slot], (uint32_t)(cnt * D * sizeof(S)));
      __syncwarp();
      for (int j = lane; j < cnt; j += 32)
        bulk_g2s_once(dst + (size_t)j * D, ksum + ((size_t)page_of(m0 + first + j) * Hkv + r) * D,
                 (uint32_t)(D * sizeof(S)), &sum_bar[slot]);
    } else {
      mbar_arrive_expect_tx(&sum_bar[slot], (uint32_t)(cnt * D * sizeof(S)));
      bulk_g2s_once(dst, ks_row + (size_t)(m0 + first) * D, (uint32_t)(cnt * D * sizeof(S)),
                    &sum_bar[slot]);
    }
  };


  if (tid == 0) {
    for (int i = 0; i < FD_NS; ++i) mbar_init(&sum_bar[i], 1);
    fence_mbar_init();
    if constexpr (!PAGED)
      for (int i = 0; i < min(FD_NS, nsub_s); ++i)
        issue_summaries(i, i * SUBC, min(SUBC, nstat - i * SUBC));
  }

  const int n = min(max(lens[b], 1), Lmax);
  const int t = (n - 1) / SAS_BLOCK;  // current block; C = t history blocks
  const int C = t;
  const int ncur = n - t * SAS_BLOCK;
  const int kk = min(topk, C);
  const int units = kk + 1;
  const int nmine = max(0, min(C, m0 + per) - m0);  // blocks this CTA scores
  const int upc = (units + CS - 1) / CS;  // units attended by each CTA
  const int u0 = min(units, crank * upc), u1 = min(units, u0 + upc), nu = u1 - u0;
  const bool own_cur = (kk >= u0 && kk < u1);
  const int nsub = (nmine + SUBC - 1) / SUBC;
  // chunks to wait for: the scored ones and, for contiguous caches, every
  // chunk copied before the length was known
  const int nwait = PAGED ? nsub : max(nsub, min(FD_NS, nsub_s));
  const int NKV = L.nkv;

  // ---- 0. barriers, expected remote bytes, first copies, q and qbar
  if (tid < CS) {
    const int nm = min(C, (tid + 1) * per) - min(C, tid * per);
    slen[tid] = topk > 0 ? min(topk, nm) : 0;
  }
  if (tid == 0) {
    for (int i = 0; i < FD_MAXKV; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], FD_WARPS);
    }
    mbar_init(list_bar, 1);
    mbar_init(state_bar, 1);
    fence_mbar_init();
    loc_cnt = 0;
    uint32_t lb = 0;  // every CTA's list and (max, sum exp)
    for (int c = 0; c < CS; ++c) {
      const int nm = min(C, (c + 1) * per) - min(C, c * per);
      lb += 8u * (uint32_t)(topk > 0 ? min(topk, nm) : 0) + 8u;
    }
    mbar_arrive_expect_tx(list_bar, lb);
    if (crank < G) mbar_arrive_expect_tx(state_bar, (uint32_t)CS * (D * 4 + 8));
  }
  if constexpr (PAGED) {
    if (wid == 0) {
      __syncwarp();  // lane 0 initialised the barriers
      for (int i = 0; i < min(FD_NS, nsub); ++i)
        issue_summaries(i, i * SUBC, min(SUBC, nmine - i * SUBC));
    }
  }
  // Barriers are initialised and fenced (fence.mbarrier_init.release.cluster
  // above): other CTAs may store into this one once every thread of the
  // cluster has arrived. A relaxed arrive does not wait for this thread's
  // loads in flight. A remote store that lands before the local expect_tx
  // only drives the transaction count below zero for a while; the phase
  // cannot complete before the local arrival.
  cluster_arrive_relaxed();
#pragma unroll
  for (int j = 0; j < QPT; ++j) {
    const int i = tid + j * FD_THREADS;
    if (i < G * D) q_s[i] = qreg[j];
  }
  __syncthreads();
  for (int i = tid; i < D; i += FD_THREADS) {
    float a = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) a += q_s[g * D + i];
    qbar[i] = a / (float)G;
  }
  __syncthreads();

  // ---- 1. score this CTA's range of history blocks. A quarter-warp takes
  // one summary: its 8 lanes read 16-byte chunks p, p + 8, ... so that each
  // quarter reads 128 contiguous bytes per load, and the dot product ends in
  // three shuffle levels (a warp reduces 4 summaries with one chain).
  {
    constexpr int SV = Vec16<S>::N;    // summary elements per 16-byte chunk
    constexpr int NCL = D / (8 * SV);  // chunks per lane
    const int qw = lane >> 3, p8 = lane & 7;
    float qv[NCL * SV];
#pragma unroll
    for (int c = 0; c < NCL; ++c)
#pragma unroll
      for (int e = 0; e < SV; ++e) qv[c * SV + e] = qbar[(c * 8 + p8) * SV + e];
    for (int i = 0; i < nwait; ++i) {
      const int slot = i % FD_NS;
      const int cnt_i = max(0, min(SUBC, nmine - i * SUBC));
      mbar_wait_data(&sum_bar[slot], (uint32_t)((i / FD_NS) & 1), err);
      const S* sb = ring + (size_t)slot * SUBC * D;
#pragma unroll 2
      for (int j0 = wid * 4; j0 < cnt_i; j0 += 4 * FD_WARPS) {
        const int j = j0 + qw;
        float a0 = 0.f, a1 = 0.f;
        if (j < cnt_i) {
#pragma unroll
          for (int c = 0; c < NCL; ++c) {
            float x[SV];
            Vec16<S>::load(sb + (size_t)j * D + (c * 8 + p8) * SV, x);
#pragma unroll
            for (int e = 0; e < SV; e += 2) {
              a0 = fmaf(x[e], qv[c * SV + e], a0);
              a1 = fmaf(x[e + 1], qv[c * SV + e + 1], a1);
            }
          }
        }
        float a = a0 + a1;
        a += __shfl_xor_sync(FULL, a, 4);
        a += __shfl_xor_sync(FULL, a, 2);
        a += __shfl_xor_sync(FULL, a, 1);
        if (p8 == 0 && j < cnt_i) sc[i * SUBC + j] = a * scale + 0.0f;
      }
      __syncthreads();  // slot consumed
      if ((PAGED ? wid == 0 : tid == 0) && i + FD_NS < nsub)
        issue_summaries(slot, (i + FD_NS) * SUBC, min(SUBC, nmine - (i + FD_NS) * SUBC));
    }
  }
  // The ring is consumed (the scan's last barrier): K/V slot 0 takes the
  // current block, unit 0 of this CTA's order when it owns it; the copy
  // overlaps the selection below.
  if (tid == 0 && own_cur) issue_kv(U, t, &full[0]);

  // ---- 2. this range's (max, sum exp) and best-first list
  {
    float lm = -FLT_MAX, ls = 0.f;
    for (int j = tid; j < nmine; j += FD_THREADS) ms_merge(lm, ls, sc[j], 1.f);
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      const float m2 = __shfl_xor_sync(FULL, lm, off), s2 = __shfl_xor_sync(FULL, ls, off);
      ms_merge(lm, ls, m2, s2);
    }
    if (lane == 0) {
      wred_m[wid] = lm;
      wred_s[wid] = ls;
    }
  }
  // Top-k of nl descending lists of stride kq (a tree of bitonic merges;
  // the buffers and length arrays are overwritten)
  auto merge_lists = [&](unsigned long long* A, int* len, unsigned long long* B, int* Blen,
                         int nl, unsigned long long* out) {
    if (lg <= 5) merge_tree_topk<1>(A, len, B, Blen, nl, lg, topk, out);
    else if (lg == 6) merge_tree_topk<2>(A, len, B, Blen, nl, lg, topk, out);
    else merge_tree_topk<4>(A, len, B, Blen, nl, lg, topk, out);
  };
  const int my_len = topk > 0 ? min(topk, nmine) : 0;
  const unsigned long long* mylist = mine;
  if (topk > 0 && nmine <= 64) {
    // small range: each key counts the keys above it, four threads per key
    // (a quarter of the range each)
    const int c = tid >> 2, qd = tid & 3;
    float sj = 0.f;
    int rk = 0;
    if (c < nmine) {
      sj = sc[c];
      const int x1 = min(nmine, qd * 16 + 16);
#pragma unroll 4
      for (int x = qd * 16; x < x1; ++x) {
        const float sx = sc[x];
        rk += (sx > sj) || (sx == sj && x < c);
      }
    }
    rk += __shfl_xor_sync(FULL, rk, 1);
    rk += __shfl_xor_sync(FULL, rk, 2);
    if (c < nmine && qd == 0 && rk < topk) mine[rk] = cand_key(sj, m0 + c);
  } else if (topk > 0 && nmine <= 64 * FD_WARPS) {
    // each warp sorts its share (at most 64 keys) in registers; the 8
    // sorted lists are merged by rank
    const int pw = (nmine + FD_WARPS - 1) / FD_WARPS;
    const int a0 = min(nmine, wid * pw), cnt = min(nmine, a0 + pw) - a0;
    unsigned long long v[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int i = j * 32 + lane;
      v[j] = i < cnt ? cand_key(sc[a0 + i], m0 + a0 + i) : 0ull;
    }
    warp_sort64_desc(v);
    const int wlen_w = min(topk, cnt);
#pragma unroll
    for (int j = 0; j < 2; ++j)
      if (j * 32 + lane < wlen_w) wl[wid * kq + j * 32 + lane] = v[j];
    if (lane == 0) wlen[wid] = wlen_w;
    __syncthreads();
    merge_lists(wl, wlen, wb, wlen_b, FD_WARPS, mine);
  } else if (topk > 0) {
    // A lower bound of the k-th key: the k-th key of a strided sample of at
    // most 256 of the range's keys. The keys at or above it are ranked.
    const int st = (nmine + 255) / 256;
    const int ns = (nmine + st - 1) / st;
    for (int i = tid; i < ns; i += FD_THREADS) samp[i] = cand_key(sc[i * st], m0 + i * st);
    __syncthreads();
    const unsigned long long th_loc = block_max_u64(sample_kth(samp, ns, topk), red8);
    auto key_of = [&](int e, unsigned long long& key) -> bool {
      key = cand_key(sc[e], m0 + e);
      return true;
    };
    if (!rank_survivors(key_of, nmine, th_loc, topk, mine, surv, &loc_cnt)) {
      // more than 512 keys at or above the bound: each warp ranks its
      // contiguous share, then one merge of the 8 lists
      const int pw = (nmine + FD_WARPS - 1) / FD_WARPS;
      const int a0 = min(nmine, wid * pw), a1 = min(nmine, a0 + pw);
      for (int j = a0 + lane; j < a1; j += 32) {
        const float sj = sc[j];
        int rk = 0;
        for (int x = a0; x < a1; ++x) {
          const float sx = sc[x];
          rk += (sx > sj) || (sx == sj && x < j);
        }
        if (rk < topk) wl[wid * kq + rk] = cand_key(sj, m0 + j);
      }
      if (lane == 0) wlen[wid] = min(topk, a1 - a0);
      __syncthreads();
      mylist = tree_merge(wl, wlen, wb, wlen_b, FD_WARPS, lg, topk) ? wb : wl;
    }
  }
  __syncthreads();
  // The head of this CTA's list (its first ceil(k/CS) keys, the share a
  // CTA holds when the kept blocks spread evenly) is likely among the kept
  // blocks: its K/V starts towards L2 now, under the exchange and the merge
  // (the CTA that attends a block after the merge may be another one).
  if (tid < min(my_len, (topk + CS - 1) / CS)) {
    const int blk = key_block(mylist[tid]);
    if (blk >= 0 && blk < nblk) {
      bulk_prefetch_l2(kv_tile(kc, blk), TILE * sizeof(T));
      bulk_prefetch_l2(kv_tile(vc, blk), TILE * sizeof(T));
    }
  }

  // ---- push this CTA's list and (max, sum exp) into its slot of every CTA
  cluster_wait_acquire();  // every CTA of the cluster has initialised its barriers
  {
    const uint32_t lst = smem_u32(stage) + (uint32_t)(crank * kq * 8);
    const uint32_t sst = smem_u32(sstat) + (uint32_t)(crank * 8);
    const uint32_t lbar = smem_u32(list_bar);
    for (int e = tid; e < CS * (my_len + 1); e += FD_THREADS) {
      const int c = e / (my_len + 1), p = e - c * (my_len + 1);
      if (p < my_len) {
        st_async_u64(mapa(lst + 8u * p, c), mylist[p], mapa(lbar, c));
      } else {
        float m4[4], s4[4];  // tree over the 8 warp pairs
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          m4[w] = wred_m[w];
          s4[w] = wred_s[w];
          ms_merge(m4[w], s4[w], wred_m[w + 4], wred_s[w + 4]);
        }
        ms_merge(m4[0], s4[0], m4[2], s4[2]);
        ms_merge(m4[1], s4[1], m4[3], s4[3]);
        ms_merge(m4[0], s4[0], m4[1], s4[1]);
        const float M = m4[0], Z = s4[0];
        st_async_f32x2(mapa(sst, c), M, Z, mapa(lbar, c));
      }
    }
  }

  // ---- 3. merge the CS lists (every CTA, identically) and the LSE
  mbar_wait_cluster(list_bar, 0, err);
  float lse;
  {  // every warp computes the same value
    const float mx = lane < CS ? sstat[2 * lane] : -FLT_MAX;
    const float se = lane < CS ? sstat[2 * lane + 1] : 0.f;
    const float M = warp_max(mx);
    const float Z = warp_sum(se > 0.f ? se * __expf(mx - M) : 0.f);
    lse = (C > 0) ? M + __logf(Z) : 0.f;
  }
  // Units are taken in score order (fin[u], best first): a CTA knows its
  // blocks as soon as the merge ends. Ascending block order is needed only
  // for idx_out, which CTA 0 writes.
  if (topk > 0 && kk > 0)
    merge_lists(stage, slen, wl, wlen_b, CS, fin);

  // ---- 4. attention over this CTA's units: the current block first when
  // owned (already in flight in slot 0), then its kept blocks in score order.
  auto unit_of = [&](int i) -> int {
    if (own_cur) return i == 0 ? kk : u0 + i - 1;
    return u0 + i;
  };
  auto issue_unit = [&](int i) {
    const int u = unit_of(i);
    int blk = (u == kk) ? t : key_block(fin[u]);
    if (blk < 0 || blk >= nblk) {
      atomicOr(err, kErrBadIndex);
      blk = t;
    }
    const int slot = i % NKV;
    issue_kv(U + (size_t)slot * kvslot, blk, &full[slot]);
  };
  if (tid == 0) {
    fence_proxy_async_smem();  // the list scratch written above becomes K/V slots
    for (int i = own_cur ? 1 : 0; i < min(NKV, nu); ++i) issue_unit(i);
  }
  if (crank == 0 && idx_out != nullptr && topk > 0) {  // kept blocks, ascending, -1 padded
    for (int i = tid; i < topk; i += FD_THREADS) {
      if (i >= kk) {
        idx_out[row * topk + i] = -1;
        continue;
      }
      const int mi = key_block(fin[i]);
      int pos = 0;
#pragma unroll 8
      for (int j = 0; j < kk; ++j) pos += key_block(fin[j]) < mi;
      idx_out[row * topk + pos] = mi;
    }
  }
  float* wst = reinterpret_cast<float*>(U);  // [warp][head][D] acc, once the units are done
  if constexpr (TMA_KV) {
    // Warp MMAs. Per unit, warp w takes keys 8w .. 8w+7: S = Q K^T as one
    // m16n8k16 chain over d (A: the group's heads as rows 0..G-1 of 16, q in
    // registers; B: K rows from the swizzled tile), leaving lane (g, t) =
    // (lane / 4, lane % 4) with head g's scores of keys 8w + 2t and 8w + 2t + 1;
    // the online softmax per head reduces over the four lanes of a head; P
    // in bf16 is then the A operand of O += P V (m16n8k8 over the 8 keys, V
    // by transposing ldmatrix), one per 8-column tile of O.
    constexpr int KS = D / 16;  // k-steps of q.k
    constexpr int NT = D / 8;   // 8-column tiles of O
    const int g = lane >> 2, t4 = lane & 3;
    // q as the A fragments of every k-step (lane-major in shared memory, read
    // back conflict-free each unit): head g's columns 16ks + 2t4 (+1) and
    // 16ks + 2t4 + 8 (+9); rows g >= G are zero
    uint32_t* qf = reinterpret_cast<uint32_t*>(sm + L.qf);
    if (wid == 0) {
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int c = ks * 16 + 2 * t4;
        qf[(2 * ks) * 32 + lane] = g < G ? pack_bf16(q_s[g * D + c], q_s[g * D + c + 1]) : 0u;
        qf[(2 * ks + 1) * 32 + lane] =
            g < G ? pack_bf16(q_s[g * D + c + 8], q_s[g * D + c + 9]) : 0u;
      }
    }
    __syncthreads();
    float acc[NT][2];  // O[head g][8n + 2t4], O[g][8n + 2t4 + 1]
    float z2 = 0.f, z3 = 0.f;  // rows 8..15 of every O tile: always zero
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = 0.f;
    float m_h = -INFINITY, l_h = 0.f;  // head g's running max and sum (this warp)
    const int key0 = wid * 8 + 2 * t4;  // this lane's two keys of the unit
    for (int i = 0; i < nu; ++i) {
      const int slot = i % NKV;
      const int u = unit_of(i);
      const bool cur = (u == kk);
      const float bias = (!cur && gated) ? key_score(fin[u]) - lse : 0.f;
      mbar_wait_data(&full[slot], (uint32_t)((i / NKV) & 1), err);
      const uint32_t kt = smem_u32(U + (size_t)slot * kvslot);
      const uint32_t vt = kt + TILE * sizeof(T);
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t b0, b1;
        const int c = ks * 16 + 2 * t4;
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b0) : "r"(kt + sw_off(wid * 8 + g, c)));
        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b1) : "r"(kt + sw_off(wid * 8 + g, c + 8)));
        mma_16816(sc, qf[(2 * ks) * 32 + lane], qf[(2 * ks + 1) * 32 + lane], b0, b1);
      }
      const float z0 = (cur && key0 >= ncur) ? -INFINITY : sc[0] * scale + bias;
      const float z1 = (cur && key0 + 1 >= ncur) ? -INFINITY : sc[1] * scale + bias;
      float zmax = fmaxf(z0, z1);
      zmax = fmaxf(zmax, __shfl_xor_sync(FULL, zmax, 1));
      zmax = fmaxf(zmax, __shfl_xor_sync(FULL, zmax, 2));
      const float mn = fmaxf(m_h, zmax);
      float p0, p1, alpha;
      if (mn == -INFINITY) {  // every key seen so far is masked
        p0 = p1 = 0.f;
        alpha = 1.f;
      } else {
        p0 = __expf(z0 - mn);
        p1 = __expf(z1 - mn);
        alpha = __expf(m_h - mn);
      }
      m_h = mn;
      float ps = p0 + p1;
      ps += __shfl_xor_sync(FULL, ps, 1);
      ps += __shfl_xor_sync(FULL, ps, 2);
      l_h = l_h * alpha + ps;
      const uint32_t pa = pack_bf16(p0, p1);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        acc[n][0] *= alpha;
        acc[n][1] *= alpha;
      }
#pragma unroll
      for (int nq = 0; nq < NT / 4; ++nq) {
        uint32_t vb[4];
        ldsm_x4_t(vb, vt + sw_off(wid * 8 + (lane & 7), (nq * 4 + (lane >> 3)) * 8));
#pragma unroll
        for (int mm = 0; mm < 4; ++mm) mma_1688(acc[nq * 4 + mm], z2, z3, pa, vb[mm]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (tid == 0 && i + NKV < nu) {  // refill the slot once every warp is done with it
        mbar_wait(&empty[slot], (uint32_t)((i / NKV) & 1), err);
        issue_unit(i + NKV);
      }
    }
    __syncthreads();  // every warp left the loop and every copy was consumed: region u is free
    if (g < G) {  // this warp's state of head g: (m, l) and acc, into [warp][head][D]
      float* w = wst + (size_t)(wid * G + g) * D;
#pragma unroll
      for (int n = 0; n < NT; ++n)
        *reinterpret_cast<float2*>(w + n * 8 + 2 * t4) = make_float2(acc[n][0], acc[n][1]);
      if (t4 == 0) mlw[g * FD_WARPS + wid] = make_float2(m_h, l_h);
    }
  } else {
    // Each warp takes 8 keys of every unit (keys wid*8 .. wid*8+7) and keeps
    // its own online-softmax state per head. Lane l holds columns
    // [l*CPL, l*CPL + CPL) of q and of the accumulators of every head. The
    // q.k partial sums of the warp's 8 keys x GP heads (one pass per group of
    // at most 4 heads) are summed over the lanes by a transposing reduction:
    // each shuffle stage halves the values a lane carries, so 8*GP sums cost
    // fewer than 8*GP shuffles and lane l ends with the sum of key l/4 and
    // head (l%4)/(4/GP) of the pass (lanes holding the same pair agree).
    constexpr int GP = G < 4 ? G : 4;  // heads per pass
    constexpr int HP = G / GP;         // passes
    constexpr int NV = 8 * GP;         // partial sums per lane per pass
    float qr[G][CPL], acc[G][CPL], m_p[HP], l_p[HP];
  #pragma unroll
    for (int h = 0; h < G; ++h) {
  #pragma unroll
      for (int c = 0; c < CPL; ++c) {
        qr[h][c] = q_s[h * D + lane * CPL + c];
        acc[h][c] = 0.f;
      }
    }
  #pragma unroll
    for (int p = 0; p < HP; ++p) {
      m_p[p] = -INFINITY;
      l_p[p] = 0.f;
    }
    const int jj = lane >> 2;                                  // this lane's key of the 8
    const int hp = (lane & 3) / (4 / GP);                      // and head within a pass
    const bool uniq = (lane & (4 / GP - 1)) == 0;              // first lane holding the pair
    float* pw = zp + wid * (2 * 8 * G);                        // [8 keys][G] p of this warp
    float* aw = pw + 8 * G;                                    // [G] rescale factors
    for (int i = 0; i < nu; ++i) {
      const int slot = i % NKV;
      const int u = unit_of(i);
      const bool cur = (u == kk);
      const float bias = (!cur && gated) ? key_score(fin[u]) - lse : 0.f;
      mbar_wait_data(&full[slot], (uint32_t)((i / NKV) & 1), err);
      const T* kt = reinterpret_cast<const T*>(U + (size_t)slot * kvslot) + (size_t)wid * 8 * D;
      const T* vt = kt + TILE;
      const bool masked = cur && (wid * 8 + jj >= ncur);
  #pragma unroll
      for (int p = 0; p < HP; ++p) {
        float part[NV];
  #pragma unroll
        for (int k8 = 0; k8 < 8; ++k8) {
          float kv[CPL];
          loadn<CPL>(kt + (size_t)k8 * D + lane * CPL, kv);
  #pragma unroll
          for (int g = 0; g < GP; ++g) {
            float a = 0.f;
  #pragma unroll
            for (int c = 0; c < CPL; ++c) a = fmaf(qr[p * GP + g][c], kv[c], a);
            part[k8 * GP + g] = a;
          }
        }
        const float dot = transpose_sum<NV>(part, lane);
        const float z = masked ? -INFINITY : dot * scale + bias;
        float zmax = z;
        zmax = fmaxf(zmax, __shfl_xor_sync(FULL, zmax, 4));
        zmax = fmaxf(zmax, __shfl_xor_sync(FULL, zmax, 8));
        zmax = fmaxf(zmax, __shfl_xor_sync(FULL, zmax, 16));
        const float mn = fmaxf(m_p[p], zmax);
        float pr, alpha;
        if (mn == -INFINITY) {  // every key seen so far is masked
          pr = 0.f;
          alpha = 1.f;
        } else {
          pr = __expf(z - mn);
          alpha = __expf(m_p[p] - mn);
        }
        m_p[p] = mn;
        float ps = pr;
        ps += __shfl_xor_sync(FULL, ps, 4);
        ps += __shfl_xor_sync(FULL, ps, 8);
        ps += __shfl_xor_sync(FULL, ps, 16);
        l_p[p] = l_p[p] * alpha + ps;
        const int h = p * GP + hp;
        if (uniq) {
          pw[jj * G + h] = pr;
          if (jj == 0) aw[h] = alpha;
        }
      }
      __syncwarp();
      {
        float al[G];
        loadg<G>(aw, al);
  #pragma unroll
        for (int h = 0; h < G; ++h)
  #pragma unroll
          for (int c = 0; c < CPL; ++c) acc[h][c] *= al[h];
      }
  #pragma unroll
      for (int k8 = 0; k8 < 8; ++k8) {  // this warp's 8 keys
        float pk[G], v[CPL];
        loadg<G>(pw + k8 * G, pk);
        loadn<CPL>(vt + (size_t)k8 * D + lane * CPL, v);
  #pragma unroll
        for (int h = 0; h < G; ++h)
  #pragma unroll
          for (int c = 0; c < CPL; c += 2) fma2(acc[h][c], acc[h][c + 1], pk[h], pk[h], v[c], v[c + 1]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      if (tid == 0 && i + NKV < nu) {  // refill the slot once every warp is done with it
        mbar_wait(&empty[slot], (uint32_t)((i / NKV) & 1), err);
        issue_unit(i + NKV);
      }
    }
    __syncthreads();  // every warp left the loop and every copy was consumed: region u is free
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float* w = wst + (size_t)(wid * G + h) * D;
#pragma unroll
      for (int c = 0; c < CPL; ++c) w[lane * CPL + c] = acc[h][c];
    }
    if (lane < 4 && uniq) {  // the lanes of key 0 hold every head's (m, l) once
#pragma unroll
      for (int p = 0; p < HP; ++p) mlw[(p * GP + hp) * FD_WARPS + wid] = make_float2(m_p[p], l_p[p]);
    }
  }
  // ---- 5. fold the warp states per head; push head h's state into CTA h.
  // Every thread of the fold takes (head, 4 columns) and derives the 8 warp
  // weights itself from the warps' (m, l).
  __syncthreads();
  {
    const uint32_t cst_r = smem_u32(cst) + (uint32_t)(crank * D * 4);
    const uint32_t cml_r = smem_u32(cml) + (uint32_t)(crank * 8);
    const uint32_t sbar = smem_u32(state_bar);
    for (int e = tid; e < G * (D / 4); e += FD_THREADS) {
      const int h = e / (D / 4), c4 = (e % (D / 4)) * 4;
      float2 ml[FD_WARPS];
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < FD_WARPS; ++w) {
        ml[w] = mlw[h * FD_WARPS + w];
        if (ml[w].y > 0.f) M = fmaxf(M, ml[w].x);
      }
      float Ls = 0.f, a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
      for (int w = 0; w < FD_WARPS; ++w) {
        const float f = ml[w].y > 0.f ? __expf(ml[w].x - M) : 0.f;
        const float4 x = *reinterpret_cast<const float4*>(wst + (size_t)(w * G + h) * D + c4);
        Ls += ml[w].y * f;
        a0 += x.x * f;
        a1 += x.y * f;
        a2 += x.z * f;
        a3 += x.w * f;
      }
      st_async_f32x4(mapa(cst_r + 4u * c4, h), a0, a1, a2, a3, mapa(sbar, h));
      if (c4 == 0) st_async_f32x2(mapa(cml_r, h), M, Ls, mapa(sbar, h));
    }
  }
  cluster_arrive_relaxed();  // pairs with the wait at exit; carries no data

  // ---- 6. CTA h < G combines head h (exact LSE rescaling)
  if (crank < G) {
    mbar_wait_cluster(state_bar, 0, err);
    if (wid == 0) {  // weights of the CS states, 1/L folded in
      const bool ok = lane < CS && cml[2 * lane + 1] > 0.f;
      const float m = ok ? cml[2 * lane] : -INFINITY;
      const float M = warp_max(m);
      const float f = ok ? __expf(m - M) : 0.f;
      const float Ls = warp_sum(ok ? cml[2 * lane + 1] * f : 0.f);
      if (lane < CS) cw[lane] = __fdividef(f, Ls);  // Ls >= 1: the max state has f = 1
    }
    __syncthreads();
    const int h = crank;
    for (int col = tid; col < D; col += FD_THREADS) {
      float a = 0.f;
      for (int c = 0; c < CS; ++c) a += cst[c * D + col] * cw[c];
      o[((size_t)b * Hq + r * G + h) * D + col] = from_f<T>(a);
    }
  }
  cluster_wait_acquire();  // no CTA leaves while stores into it may be pending
}

// ------------------------------------------------------------------ host
namespace {

struct FdPick {
  int dev, rows, nblk, kq, CS, ub;
};

// Cluster size and ring region for a shape. Candidates: cluster sizes 16,
// 8, 4, 2, 1 (>= G, since CTA h combines head h), each first with a large
// ring region (when the grid leaves at most one CTA per SM: deeper summary
// and K/V rings) and then with the small one (two CTAs per SM). The first
// whose clusters of all rows are co-resident on the GPU wins; if none is,
// the first that launches. Cached per shape, so repeated launches make no
// occupancy queries.
template <typename T, int D, int G, bool PAGED, typename S>
cudaError_t pick_cluster(int B, int Hkv, int nblk, int kq, int& CS_out, int& ub_out) {
  static std::mutex mu;
  static FdPick cache[32];
  static int ncache = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int rows = B * Hkv;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < ncache; ++i)
      if (cache[i].dev == dev && cache[i].rows == rows && cache[i].nblk == nblk &&
          cache[i].kq == kq) {
        CS_out = cache[i].CS;
        ub_out = cache[i].ub;
        return cudaSuccess;
      }
  }
  int nsm = 0;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  auto kern = k_decode_fused<T, D, G, PAGED, S>;
  int best = 0, best_ub = 0, first = 0, first_ub = 0;
  const int cands[5] = {16, 8, 4, 2, 1};
  for (int ci = 0; ci < 5 && !best; ++ci) {
    const int CS = cands[ci];
    if (CS < G) break;
    for (int big = (rows * CS <= nsm) ? 1 : 0; big >= 0 && !best; --big) {
      const int ub = big ? FD_BIG_REGION : 0;
      const size_t smem =
          fd_layout(D, G, (int)sizeof(T), (nblk + CS - 1) / CS, kq, CS, (int)sizeof(S), ub).total;
      if (smem > FD_SMEM_MAX) continue;
      if (ensure_smem(kern, smem) != cudaSuccess) {
        cudaGetLastError();
        continue;
      }
      if (CS > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                         1) != cudaSuccess) {
        cudaGetLastError();
        continue;
      }
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(CS, Hkv, B);
      cfg.blockDim = dim3(FD_THREADS);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = CS;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int ncl = 0;
      if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        continue;
      }
      if (ncl < 1) continue;
      if (!first) {
        first = CS;
        first_ub = ub;
      }
      if (ncl >= rows) {
        best = CS;
        best_ub = ub;
      }
    }
  }
  CS_out = best ? best : first;
  ub_out = best ? best_ub : first_ub;
  if (!CS_out) return cudaErrorInvalidConfiguration;
  std::lock_guard<std::mutex> lock(mu);
  if (ncache < 32) cache[ncache++] = FdPick{dev, rows, nblk, kq, CS_out, ub_out};
  return cudaSuccess;
}

template <typename T, int D, int G, bool PAGED, typename S>
cudaError_t launch_fused_t(const void* q, const void* kc, const void* vc, const void* ksum, int B,
                           int Hkv, int Lmax, const int32_t* lens, int topk, int gated, float scale,
                           void* o, int32_t* idx_out, const int32_t* bt, int npages,
                           cudaStream_t st) {
  auto kern = k_decode_fused<T, D, G, PAGED, S>;
  const int nblk = Lmax / SAS_BLOCK;
  const int kq = 1 << ceil_log2(topk > 0 ? topk : 1);
  int CS = 0, ub = 0;
  cudaError_t e = pick_cluster<T, D, G, PAGED, S>(B, Hkv, nblk, kq, CS, ub);
  if (e != cudaSuccess) return e;
  const int per_max = (nblk + CS - 1) / CS;
  const size_t smem =
      fd_layout(D, G, (int)sizeof(T), per_max, kq, CS, (int)sizeof(S), ub).total;
  e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, Hkv, B);
  cfg.blockDim = dim3(FD_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // bf16 caches are read by TMA: the caches as 3-D tensors of 64 x 64 boxes
  // (contiguous: planes of Lmax rows per (sequence, kv head); paged: planes of
  // 64 rows per (page, kv head))
  CUtensorMap km = {}, vm = {};
  if (std::is_same<T, __nv_bfloat16>::value) {
    const int rows = PAGED ? SAS_BLOCK : Lmax;
    const int planes = PAGED ? npages * Hkv : B * Hkv;
    if (!make_tma_map_bf16_3d(&km, kc, D, rows, planes) ||
        !make_tma_map_bf16_3d(&vm, vc, D, rows, planes))
      return cudaErrorInvalidValue;
  }
  return cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(q), static_cast<const T*>(kc),
                            static_cast<const T*>(vc), static_cast<const S*>(ksum), Hkv, Lmax,
                            lens, topk, gated, scale, per_max, ub, static_cast<T*>(o), idx_out,
                            bt, npages, km, vm);
}

template <typename T, int D>
cudaError_t launch_fused_g(int G, const void* q, const void* kc, const void* vc, const void* ksum,
                           int sum_bf16, int B, int Hkv, int Lmax, const int32_t* lens, int topk,
                           int gated, float scale, void* o, int32_t* idx_out, const int32_t* bt,
                           int npages, cudaStream_t st) {
#define SAS_FD(GG)                                                                              \
  if (bt && sum_bf16)                                                                           \
    return launch_fused_t<T, D, GG, true, __nv_bfloat16>(q, kc, vc, ksum, B, Hkv, Lmax, lens,   \
                                                         topk, gated, scale, o, idx_out, bt,    \
                                                         npages, st);                           \
  if (bt)                                                                                       \
    return launch_fused_t<T, D, GG, true, float>(q, kc, vc, ksum, B, Hkv, Lmax, lens, topk,     \
                                                 gated, scale, o, idx_out, bt, npages, st);     \
  if (sum_bf16)                                                                                 \
    return launch_fused_t<T, D, GG, false, __nv_bfloat16>(q, kc, vc, ksum, B, Hkv, Lmax, lens,  \
                                                          topk, gated, scale, o, idx_out,       \
                                                          nullptr, 0, st);                      \
  return launch_fused_t<T, D, GG, false, float>(q, kc, vc, ksum, B, Hkv, Lmax, lens, topk,      \
                                                gated, scale, o, idx_out, nullptr, 0, st)
  switch (G) {
    case 1: SAS_FD(1);
    case 2: SAS_FD(2);
    case 4: SAS_FD(4);
    case 8: SAS_FD(8);
    default: return cudaErrorInvalidValue;
  }
#undef SAS_FD
}

cudaError_t launch_fused(const void* q, const void* kc, const void* vc, int bf16, int B, int Hq,
                         int Hkv, int Lmax, int d, const int32_t* lens, const void* ksum,
                         int sum_bf16, int topk, int gated, float scale, void* o,
                         int32_t* idx_out, const int32_t* bt, int npages, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  const int G = Hq / Hkv;
  if (bf16) {
    if (d == 128)
      return launch_fused_g<__nv_bfloat16, 128>(G, q, kc, vc, ksum, sum_bf16, B, Hkv, Lmax, lens,
                                                topk, gated, scale, o, idx_out, bt, npages, st);
    return launch_fused_g<__nv_bfloat16, 64>(G, q, kc, vc, ksum, sum_bf16, B, Hkv, Lmax, lens,
                                             topk, gated, scale, o, idx_out, bt, npages, st);
  }
  if (d == 128)
    return launch_fused_g<float, 128>(G, q, kc, vc, ksum, sum_bf16, B, Hkv, Lmax, lens, topk,
                                      gated, scale, o, idx_out, bt, npages, st);
  return launch_fused_g<float, 64>(G, q, kc, vc, ksum, sum_bf16, B, Hkv, Lmax, lens, topk, gated,
                                   scale, o, idx_out, bt, npages, st);
}

}  // namespace

cudaError_t launch_decode_fused(const void* q, const void* kc, const void* vc, int bf16, int B,
                                int Hq, int Hkv, int Lmax, int d, const int32_t* lens,
                                const float* ksum, int topk, int gated, float scale, void* o,
                                int32_t* idx_out, cudaStream_t st) {
  return launch_fused(q, kc, vc, bf16, B, Hq, Hkv, Lmax, d, lens, ksum, 0, topk, gated, scale, o,
                      idx_out, nullptr, 0, st);
}

cudaError_t launch_decode_fused_ex(const void* q, const void* kc, const void* vc, int bf16, int B,
                                   int Hq, int Hkv, int Lmax, int d, const int32_t* lens,
                                   const void* ksum, int sum_bf16, int topk, int gated,
                                   float scale, void* o, int32_t* idx_out, cudaStream_t st) {
  return launch_fused(q, kc, vc, bf16, B, Hq, Hkv, Lmax, d, lens, ksum, sum_bf16, topk, gated,
                      scale, o, idx_out, nullptr, 0, st);
}

cudaError_t launch_decode_paged(const void* q, const void* kpool, const void* vpool, int bf16,
                                int B, int Hq, int Hkv, int npages, int d,
                                const int32_t* block_table, int max_blocks, const int32_t* lens,
                                const void* kspool, int sum_bf16, int topk, int gated,
                                float scale, void* o, int32_t* idx_out, cudaStream_t st) {
  return launch_fused(q, kpool, vpool, bf16, B, Hq, Hkv, max_blocks * SAS_BLOCK, d, lens, kspool,
                      sum_bf16, topk, gated, scale, o, idx_out, block_table, npages, st);
}

uint32_t* decode_fused_error_word() {
  void* p = nullptr;
  cudaGetSymbolAddress(&p, g_decode_fused_err);
  return static_cast<uint32_t*>(p);
}

}  // namespace sas
