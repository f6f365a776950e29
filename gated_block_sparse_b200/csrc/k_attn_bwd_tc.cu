// Gated sparse attention backward on the 5th-generation tensor cores (bf16,
// d = 128): TMA-fed tcgen05 MMAs with TMEM accumulators.
//
// Definition (SAS close reading, liuzhao09.github.io, sections 2.2 and 2.4,
// eq. 5): with p recomputed from the forward's lse, D_i = dO_i . o_i,
// dp_ij = dO_i . v_j, dz_ij = p_ij (dp_ij - D_i); dq_i = scale sum_j dz_ij k_j,
// dk_j = scale sum_i dz_ij q_i, dv_j = sum_i p_ij dO_i, and
// dlogg[t][slot] = the sum of dz over the slot's keys, the query block's rows
// and the group's heads.
//
// One CTA per (query block t, kv group r, pair of query heads): M = 128 rows.
// For each unit (kept history block, then the current block):
//   S = Q K^T and dP = dO V^T          M128 N64  K128 -> TMEM (lanes = rows)
//   dQ += dS K                          M128 N128 K64  -> TMEM (lanes = rows)
//   dK^T = Q^T dS, dV^T = dO^T P        M128 N64  K128 -> TMEM (lanes = d)
// The softmax warps write P and scale*dS as bf16 into shared memory in the
// 128-byte-swizzled layout; the same buffer is the K-major A operand of dQ
// and the MN-major B operand of dK^T (P likewise for dV^T). dK^T / dV^T are
// double-buffered in TMEM; the softmax warps, which own TMEM lanes = d,
// read them and add them into fp32 accumulators of dk and dv (coalesced
// reductions; a conversion pass writes the output dtype). dlogg is summed
// in-CTA in a fixed order and added once per CTA.
//   warp 4: TMA (Q and dO once; K and V of each unit into a 2-stage ring)
//   warp 5: one thread issues all MMAs
//   warps 0-3: softmax / gradient rows and the reductions
// 512 TMEM columns and about 161 KB of shared memory: one CTA per SM.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tc.cuh"

namespace sas {

__device__ uint32_t g_attn_bwd_tc_err = 0;

namespace {

constexpr int BT_THREADS = 192;
constexpr int D = 128;
constexpr uint32_t TILE128 = 128 * D * 2;            // Q or dO: 32 KB
constexpr uint32_t KV_STAGE = 2 * 64 * D * 2;        // K + V: 32 KB
constexpr uint32_t PT_BYTES = 128 * 64 * 2;          // P or dS: 16 KB
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_DO = OFF_Q + TILE128;
constexpr uint32_t OFF_KV = OFF_DO + TILE128;
constexpr uint32_t OFF_P = OFF_KV + 2 * KV_STAGE;
constexpr uint32_t OFF_DS = OFF_P + PT_BYTES;
constexpr uint32_t OFF_BAR = OFF_DS + PT_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256;
constexpr float LOG2E = 1.4426950408889634f;

enum Bar {
  B_Q = 0,     // Q and dO loaded
  B_KVF = 1,   // [2] K/V stage full
  B_KVE = 3,   // [2] K/V stage empty (all MMAs of its unit done)
  B_SF = 5,    // S and dP of the unit in TMEM
  B_SE = 6,    // S and dP read by the softmax warps (4 arrivals)
  B_PF = 7,    // P and dS written (4 arrivals)
  B_MD = 8,    // all MMAs of the unit done
  B_TE = 9,    // [2] dK^T/dV^T TMEM buffer read (4 arrivals)
  NBAR = 11
};

// TMEM columns
constexpr uint32_t C_S = 0, C_DP = 64, C_DQ = 128, C_DKT = 256, C_DVT = 320, C_BUF = 128;

__device__ __forceinline__ void named_bar_softmax() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

__device__ __forceinline__ void red_add(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

}  // namespace

__global__ void __launch_bounds__(BT_THREADS, 1) k_attn_bwd_tc(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
    const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap domap,
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, int Hq, int Hkv, int N, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ cnt, const float* __restrict__ logg, int topk, float scale,
    __nv_bfloat16* __restrict__ dq, float* __restrict__ dk_acc, float* __restrict__ dv_acc,
    float* __restrict__ dlogg) {
  extern __shared__ __align__(1024) unsigned char sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + NBAR * 8);
  float* red_s = reinterpret_cast<float*>(sm + OFF_BAR + NBAR * 8 + 16);  // [4]
  uint32_t* err = &g_attn_bwd_tc_err;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = Hq / Hkv, pairs = G / 2;
  const int T_ = gridDim.x;
  const int t = T_ - 1 - (int)blockIdx.x;
  const int r = blockIdx.y / pairs, hp = blockIdx.y % pairs, b = blockIdx.z;
  const int h0 = r * G + 2 * hp;
  const size_t srow = ((size_t)b * Hkv + r) * T_ + t;
  const int kk = min(max(cnt[srow], 0), topk);
  const int nunits = kk + 1;
  const int32_t* idx_row = idx + srow * topk;
  const float* logg_row = logg + srow * topk;
  if ((smem_u32(sm) & 1023u) != 0) {
    if (tid == 0) atomicOr(err, kErrBadIndex);
    return;
  }
  auto unit_block = [&](int j) -> int {
    int blk = (j < kk) ? idx_row[j] : t;
    if (blk < 0 || blk >= t) blk = t;
    return blk;
  };
  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i) {
      const bool four = (i == B_SE || i == B_PF || i == B_TE || i == B_TE + 1);
      mbar_init(&bars[i], four ? 4 : 1);
    }
    fence_mbar_init();
  }
  if (warp == 5) tc::tmem_alloc(tmem_slot, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tc::prefetch_map(&qmap);
      tc::prefetch_map(&kmap);
      tc::prefetch_map(&vmap);
      tc::prefetch_map(&domap);
      mbar_arrive_expect_tx(&bars[B_Q], 2 * TILE128);
      for (int c = 0; c < 2; ++c)
        for (int h = 0; h < 2; ++h) {
          tc::tma_load_3d(sm + OFF_Q + c * 16384 + h * 8192, &qmap, 64 * c, 64 * t,
                          b * Hq + h0 + h, &bars[B_Q]);
          tc::tma_load_3d(sm + OFF_DO + c * 16384 + h * 8192, &domap, 64 * c, 64 * t,
                          b * Hq + h0 + h, &bars[B_Q]);
        }
      for (int j = 0; j < nunits; ++j) {
        const int s = j & 1;
        if (j >= 2) mbar_wait(&bars[B_KVE + s], ((j >> 1) - 1) & 1, err);
        const int blk = unit_block(j);
        if (j < kk && blk != idx_row[j]) atomicOr(err, kErrBadIndex);
        unsigned char* st = sm + OFF_KV + s * KV_STAGE;
        mbar_arrive_expect_tx(&bars[B_KVF + s], KV_STAGE);
        const int plane = b * Hkv + r;
        tc::tma_load_3d(st, &kmap, 0, 64 * blk, plane, &bars[B_KVF + s]);
        tc::tma_load_3d(st + 8192, &kmap, 64, 64 * blk, plane, &bars[B_KVF + s]);
        tc::tma_load_3d(st + 16384, &vmap, 0, 64 * blk, plane, &bars[B_KVF + s]);
        tc::tma_load_3d(st + 24576, &vmap, 64, 64 * blk, plane, &bars[B_KVF + s]);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_N64 = tc::idesc_bf16(128, 64, 0, 0);     // S, dP
      constexpr uint32_t ID_DQ = tc::idesc_bf16(128, 128, 0, 1);     // dQ += dS K
      constexpr uint32_t ID_T = tc::idesc_bf16(128, 64, 1, 1);       // dK^T, dV^T
      const uint32_t q_a = smem_u32(sm + OFF_Q), do_a = smem_u32(sm + OFF_DO);
      const uint32_t p_a = smem_u32(sm + OFF_P), ds_a = smem_u32(sm + OFF_DS);
      mbar_wait(&bars[B_Q], 0, err);
      for (int j = 0; j < nunits; ++j) {
        const int s = j & 1;
        const uint32_t k_a = smem_u32(sm + OFF_KV + s * KV_STAGE);
        const uint32_t v_a = k_a + 16384;
        mbar_wait(&bars[B_KVF + s], (j >> 1) & 1, err);
        if (j >= 1) mbar_wait(&bars[B_SE], (j - 1) & 1, err);
        tc::fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // S = Q K^T, dP = dO V^T (K = d)
          const uint32_t c = ks >> 2, off = (ks & 3) * 32;
          tc::mma_bf16(tmem + C_S, tc::sw128_desc(q_a + c * 16384 + off, 16, 1024),
                       tc::sw128_desc(k_a + c * 8192 + off, 16, 1024), ID_N64, ks > 0);
          tc::mma_bf16(tmem + C_DP, tc::sw128_desc(do_a + c * 16384 + off, 16, 1024),
                       tc::sw128_desc(v_a + c * 8192 + off, 16, 1024), ID_N64, ks > 0);
        }
        tc::commit(&bars[B_SF]);
        mbar_wait(&bars[B_PF], j & 1, err);
        if (j >= 2) mbar_wait(&bars[B_TE + s], ((j >> 1) - 1) & 1, err);
        tc::fence_after_sync();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)  // dQ += dS K   (K = keys)
          tc::mma_bf16(tmem + C_DQ, tc::sw128_desc(ds_a + ks * 32, 16, 1024),
                       tc::sw128_desc(k_a + ks * 2048, 8192, 1024), ID_DQ, (j > 0 || ks > 0));
        const uint32_t cb = tmem + s * C_BUF;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // dK^T = Q^T dS, dV^T = dO^T P   (K = rows)
          tc::mma_bf16(cb + C_DKT, tc::sw128_desc(q_a + ks * 2048, 16384, 1024),
                       tc::sw128_desc(ds_a + ks * 2048, 8192, 1024), ID_T, ks > 0);
          tc::mma_bf16(cb + C_DVT, tc::sw128_desc(do_a + ks * 2048, 16384, 1024),
                       tc::sw128_desc(p_a + ks * 2048, 8192, 1024), ID_T, ks > 0);
        }
        tc::commit(&bars[B_MD]);
        tc::commit(&bars[B_KVE + s]);
      }
    }
  } else {
    // ---------------------------------------------------------------- gradient rows
    const int row = tid;  // TMEM lane: query row for S/dP/dQ, head dim d for dK^T/dV^T
    const int hh = row >> 6, qr = row & 63;
    const int pos = 64 * t + qr;
    const bool valid = pos < N;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float c1 = scale * LOG2E;
    const size_t qrow = ((size_t)b * Hq + h0 + hh) * N + (valid ? pos : 0);
    float Di = 0.f, lse2 = 0.f;
    if (valid) {
      const __nv_bfloat16* orow = o + qrow * D;
      const __nv_bfloat16* drow = dout + qrow * D;
      for (int c = 0; c < D; c += 8) {
        float a[8], g[8];
        Vec16<__nv_bfloat16>::load(orow + c, a);
        Vec16<__nv_bfloat16>::load(drow + c, g);
#pragma unroll
        for (int e = 0; e < 8; ++e) Di += a[e] * g[e];
      }
      lse2 = lse[qrow] * LOG2E;
    }
    unsigned char* prow = sm + OFF_P + row * 128;
    unsigned char* dsrow = sm + OFF_DS + row * 128;
    const size_t kvbase = ((size_t)b * Hkv + r) * N * D;
    auto flush_kv = [&](int jj) {  // add unit jj's dK^T / dV^T (lane = d) to the accumulators
      const int blk = unit_block(jj);
      const uint32_t cb = tmem + (jj & 1) * C_BUF + lane_off;
      const int dcol = row;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        float kv[32], vv[32];
        tc::tmem_ld32(cb + C_DKT + 32 * half, kv);
        tc::tmem_ld32(cb + C_DVT + 32 * half, vv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int key = 64 * blk + 32 * half + i;
          if (key < N) {
            red_add(dk_acc + kvbase + (size_t)key * D + dcol, kv[i]);
            red_add(dv_acc + kvbase + (size_t)key * D + dcol, vv[i]);
          }
        }
      }
    };
    for (int j = 0; j < nunits; ++j) {
      const int s = j & 1;
      const bool cur = (j == kk);
      const float bias = cur ? 0.f : logg_row[j] * LOG2E;
      mbar_wait(&bars[B_SF], j & 1, err);
      tc::fence_after_sync();
      float sv[64], dp[64];
      {
        float a0[32], a1[32];
        tc::tmem_ld32(tmem + C_S + lane_off, a0);
        tc::tmem_ld32(tmem + C_S + lane_off + 32, a1);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          sv[i] = a0[i];
          sv[32 + i] = a1[i];
        }
        tc::tmem_ld32(tmem + C_DP + lane_off, a0);
        tc::tmem_ld32(tmem + C_DP + lane_off + 32, a1);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          dp[i] = a0[i];
          dp[32 + i] = a1[i];
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_SE]);
      float dsum = 0.f;
      uint32_t pk[32], dk2[32];
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        float p0 = exp2f(sv[i] * c1 + bias - lse2), p1 = exp2f(sv[i + 1] * c1 + bias - lse2);
        if (!valid || (cur && i > qr)) p0 = 0.f;
        if (!valid || (cur && i + 1 > qr)) p1 = 0.f;
        const float d0 = p0 * (dp[i] - Di), d1 = p1 * (dp[i + 1] - Di);
        dsum += d0 + d1;
        __nv_bfloat162 hp2 = __floats2bfloat162_rn(p0, p1);
        __nv_bfloat162 hd2 = __floats2bfloat162_rn(d0 * scale, d1 * scale);
        pk[i >> 1] = *reinterpret_cast<uint32_t*>(&hp2);
        dk2[i >> 1] = *reinterpret_cast<uint32_t*>(&hd2);
      }
      if (j >= 1) {  // MMAs of the previous unit done: P/dS buffers free, dK^T/dV^T ready
        mbar_wait(&bars[B_MD], (j - 1) & 1, err);
        tc::fence_after_sync();
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int pc = (c ^ (row & 7)) << 4;
        *reinterpret_cast<uint4*>(prow + pc) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(dsrow + pc) =
            make_uint4(dk2[4 * c], dk2[4 * c + 1], dk2[4 * c + 2], dk2[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PF]);
      if (j >= 1) {
        flush_kv(j - 1);
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B_TE + ((j - 1) & 1)]);
      }
      if (!cur) {  // d(log g) of this slot, in a fixed order
        dsum = warp_sum(dsum);
        if (lane == 0) red_s[warp] = dsum;
        named_bar_softmax();
        if (tid == 0) atomicAdd(dlogg + srow * topk + j, red_s[0] + red_s[1] + red_s[2] + red_s[3]);
        named_bar_softmax();
      }
    }
    mbar_wait(&bars[B_MD], (nunits - 1) & 1, err);
    tc::fence_after_sync();
    flush_kv(nunits - 1);
    // dQ (already scaled through dS)
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float qv[32];
      tc::tmem_ld32(tmem + C_DQ + lane_off + 32 * c, qv);
      tc::tmem_wait_ld();
      if (valid) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(qv[8 * g + 2 * e], qv[8 * g + 2 * e + 1]);
            w[e] = *reinterpret_cast<uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(dq + qrow * D + 32 * c + 8 * g) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host
static bool make_map(CUtensorMap* map, const void* base, int rows_per_plane, int planes) {
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows_per_plane, (cuuint64_t)planes};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows_per_plane * D * 2};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return cuTensorMapEncodeTiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                                dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename TT>
__global__ void k_convert_tc(const float* __restrict__ src, TT* __restrict__ dst, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = from_f<TT>(src[i]);
}

cudaError_t launch_attn_bwd_tc(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, int B, int Hq, int Hkv, int N,
                               const float* lse, const int32_t* idx, const int32_t* cnt,
                               const float* logg, int topk, float scale, void* dq, void* dk,
                               void* dv, float* dlogg, void* ws, cudaStream_t st) {
  const int T_ = (N + 63) / 64;
  if (B == 0 || T_ == 0) return cudaSuccess;
  const size_t nkv = (size_t)B * Hkv * N * D;
  float* dk_acc = static_cast<float*>(ws);
  float* dv_acc = dk_acc + nkv;
  cudaError_t e = cudaMemsetAsync(ws, 0, 2 * nkv * sizeof(float), st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(dlogg, 0, (size_t)B * Hkv * T_ * topk * sizeof(float), st);
  if (e != cudaSuccess) return e;
  CUtensorMap qm, km, vm, dom;
  if (!make_map(&qm, q, N, B * Hq) || !make_map(&km, k, N, B * Hkv) ||
      !make_map(&vm, v, N, B * Hkv) || !make_map(&dom, dout, N, B * Hq))
    return cudaErrorInvalidValue;
  e = ensure_smem(k_attn_bwd_tc, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(T_, Hkv * (Hq / Hkv / 2), B);
  k_attn_bwd_tc<<<grid, BT_THREADS, SMEM_BYTES, st>>>(
      qm, km, vm, dom, static_cast<const __nv_bfloat16*>(o),
      static_cast<const __nv_bfloat16*>(dout), lse, Hq, Hkv, N, idx, cnt, logg, topk, scale,
      static_cast<__nv_bfloat16*>(dq), dk_acc, dv_acc, dlogg);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int cgrid = (int)((nkv + 255) / 256 < 8192 ? (nkv + 255) / 256 : 8192);
  k_convert_tc<__nv_bfloat16><<<cgrid, 256, 0, st>>>(dk_acc, static_cast<__nv_bfloat16*>(dk), nkv);
  k_convert_tc<__nv_bfloat16><<<cgrid, 256, 0, st>>>(dv_acc, static_cast<__nv_bfloat16*>(dv), nkv);
  return cudaGetLastError();
}

uint32_t* attn_bwd_tc_error_word() {
  void* p = nullptr;
  cudaGetSymbolAddress(&p, g_attn_bwd_tc_err);
  return static_cast<uint32_t*>(p);
}

}  // namespace sas
