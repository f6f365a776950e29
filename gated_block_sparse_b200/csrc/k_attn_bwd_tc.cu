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
// read them and add them into fp32 accumulators of dk and dv (a conversion
// pass writes the output dtype). dlogg is summed in-CTA in a fixed order and
// added once per CTA.
//   warp 8: TMA (Q and dO once; K and V of each unit into a 2-stage ring)
//   warp 9: one thread issues all MMAs; S/dP of unit j+1 are issued while
//           the gradient warps form unit j's P and dS
//   warps 0-7: gradient rows: warps w and w+4 share the TMEM lanes of rows
//           32(w%4).. and split the 64 key columns, two warps per SM
//           sub-partition to hide instruction latency
//   warps 10-13: flush of dK^T / dV^T (TMEM lanes 32(w%4).. = head dims)
// dK^T / dV^T reach the fp32 accumulators through four flush warps (one per
// TMEM lane quarter): each moves its quarter of unit j's dK^T / dV^T into
// [8 keys][32 d] shared-memory slices, each added by one TMA tensor
// reduce-add (two slices per warp alternate), while the gradient warps
// already work on unit j+1; K/V stream through a three-stage ring; no
// CTA-wide barrier runs inside the unit loop. The reductions (64 KB per
// unit) drain at about 20 bytes per cycle per SM, so the flush warps take
// them off the gradient warps' path.
// 512 TMEM columns and about 213 KB of shared memory: one CTA per SM.
//
// Per-token selection (TOK = true; section 2.4): units are the union of the
// blocks the query block's tokens selected (a bitmask walked in ascending
// order), then the current block; each gradient row adds its token's log g
// where its token selected the unit's block and masks the unit otherwise,
// and adds its logit gradients over the unit's keys into its token's slot of
// dlogg ([B][Hkv][N][topk]).
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tc.cuh"

namespace sas {

__device__ uint32_t g_attn_bwd_tc_err = 0;

namespace {

constexpr int BT_THREADS = 448;  // 8 gradient warps, TMA warp, MMA warp, 4 flush warps
constexpr int NGW = 8;           // gradient warps
constexpr int NFW = 4;           // flush warps (warps 10-13)
constexpr int D = 128;
constexpr uint32_t TILE128 = 128 * D * 2;            // Q or dO: 32 KB
constexpr uint32_t KV_STAGE = 2 * 64 * D * 2;        // K + V: 32 KB
constexpr uint32_t PT_BYTES = 128 * 64 * 2;          // P or dS: 16 KB
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_DO = OFF_Q + TILE128;
constexpr uint32_t OFF_KV = OFF_DO + TILE128;
constexpr int NKV = 3;                                // K/V ring stages
constexpr uint32_t OFF_P = OFF_KV + NKV * KV_STAGE;
constexpr uint32_t OFF_DS = OFF_P + PT_BYTES;
constexpr uint32_t OFF_T = OFF_DS + PT_BYTES;         // fp32 [warp][2][8 keys][32 d] slices
constexpr int FSLOT = 1;         // [32 keys][32 d] slices per flush warp
constexpr uint32_t OFF_DL = OFF_T + NFW * FSLOT * 32 * 32 * 4;  // fp32 [unit][warp] d(log g) partials
constexpr uint32_t OFF_BAR = OFF_DL + 129 * 8 * 4 + 64;
constexpr uint32_t OFF_UM = OFF_BAR + 256;  // per-token mode: union bitmask and its count
constexpr uint32_t SMEM_BYTES = OFF_UM + 128;
constexpr int TOK_UMAX = 512;  // history blocks of a query block at most (per-token mode)
constexpr float LOG2E = 1.4426950408889634f;

enum Bar {
  B_Q = 0,     // Q and dO loaded
  B_KVF = 1,   // [NKV] K/V stage full
  B_KVE = 4,   // [NKV] K/V stage empty (all MMAs of its unit done)
  B_SF = 7,    // S and dP of the unit in TMEM
  B_SE = 8,    // S and dP read by the gradient warps (one arrival per warp)
  B_PF = 9,    // P and dS written (one arrival per warp)
  B_MD = 10,   // all MMAs of the unit done
  B_TE = 11,   // [2] dK^T/dV^T TMEM buffer read (one arrival per flush warp)
  B_KF = 13,   // [2] dK^T/dV^T TMEM buffer written (its unit's MMAs done)
  NBAR = 15
};

// TMEM columns
constexpr uint32_t C_S = 0, C_DP = 64, C_DQ = 128, C_DKT = 256, C_DVT = 320, C_BUF = 128;

__device__ __forceinline__ void named_bar_softmax() {
  asm volatile("bar.sync 1, 256;" ::: "memory");
}


}  // namespace

template <bool TOK>
__global__ void __launch_bounds__(BT_THREADS, 1) k_attn_bwd_tc(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
    const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap domap,
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
    const __grid_constant__ CUtensorMap dkmap, const __grid_constant__ CUtensorMap dvmap,
    const float* __restrict__ lse, int Hq, int Hkv, int N, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ cnt, const float* __restrict__ logg, int topk, float scale,
    __nv_bfloat16* __restrict__ dq, float* __restrict__ dlogg) {
  extern __shared__ __align__(1024) unsigned char sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + NBAR * 8);
  uint32_t* err = &g_attn_bwd_tc_err;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = Hq / Hkv, pairs = G / 2;
  const int T_ = gridDim.x;
  const int t = T_ - 1 - (int)blockIdx.x;
  const int r = blockIdx.y / pairs, hp = blockIdx.y % pairs, b = blockIdx.z;
  const int h0 = r * G + 2 * hp;
  const size_t srow = ((size_t)b * Hkv + r) * T_ + t;
  int kk = TOK ? 0 : min(max(cnt[srow], 0), topk);
  const int32_t* idx_row = idx + (TOK ? 0 : srow * topk);
  const float* logg_row = logg + (TOK ? 0 : srow * topk);
  if ((smem_u32(sm) & 1023u) != 0) {
    if (tid == 0) atomicOr(err, kErrBadIndex);
    return;
  }
  const size_t tok0 = ((size_t)b * Hkv + r) * N + 64 * t;  // first token row of the block
  const int words = (t + 31) / 32;
  uint32_t* umask = reinterpret_cast<uint32_t*>(sm + OFF_UM);  // per-token: TOK_UMAX / 32 words
  if constexpr (TOK) {
    int& ucnt = *reinterpret_cast<int*>(sm + OFF_UM + TOK_UMAX / 8);
    const int nr = min(64, N - 64 * t);
    for (int w = tid; w < words; w += BT_THREADS) umask[w] = 0u;
    __syncthreads();
    for (int e = tid; e < nr * topk; e += BT_THREADS) {
      const int i = e / topk, p = e - i * topk;
      if (p < min(max(cnt[tok0 + i], 0), topk)) {
        const int m = idx[(tok0 + i) * topk + p];
        if (m >= 0 && m < t) atomicOr(&umask[m >> 5], 1u << (m & 31));
        else atomicOr(err, kErrBadIndex);
      }
    }
    __syncthreads();
    if (warp == 0) {
      int c = 0;
      for (int w = lane; w < words; w += 32) c += __popc(umask[w]);
      c = __reduce_add_sync(0xffffffffu, c);
      if (lane == 0) ucnt = c;
    }
    __syncthreads();
    kk = ucnt;
  }
  const int nunits = kk + 1;
  // per-token: smallest selected block >= from (ascending), -1 past the end
  auto next_unit = [&](int from) -> int {
    for (int w = from >> 5; w < words; ++w) {
      const uint32_t word = umask[w] & (w == (from >> 5) ? (~0u << (from & 31)) : ~0u);
      if (word) return w * 32 + __ffs(word) - 1;
    }
    return -1;
  };
  // block of unit j (units in order; per-token mode advances the cursor)
  int ucur = -1;
  auto unit_block = [&](int j) -> int {
    int blk;
    if constexpr (TOK) {
      if (j < kk) ucur = next_unit(ucur + 1);
      blk = (j < kk) ? ucur : t;
    } else {
      blk = (j < kk) ? idx_row[j] : t;
    }
    if (blk < 0 || blk >= t) blk = t;
    return blk;
  };
  if (tid == 0) {
    for (int i = 0; i < NBAR; ++i) {
      const bool grad = (i == B_SE || i == B_PF), flush = (i == B_TE || i == B_TE + 1);
      mbar_init(&bars[i], grad ? NGW : (flush ? NFW : 1));
    }
    fence_mbar_init();
  }
  if (warp == 9) tc::tmem_alloc(tmem_slot, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
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
        const int s = j % NKV;
        if (j >= NKV) mbar_wait_data(&bars[B_KVE + s], ((j / NKV) - 1) & 1, err);
        const int blk = unit_block(j);
        if (!TOK && j < kk && blk != idx_row[j]) atomicOr(err, kErrBadIndex);
        unsigned char* st = sm + OFF_KV + s * KV_STAGE;
        mbar_arrive_expect_tx(&bars[B_KVF + s], KV_STAGE);
        const int plane = b * Hkv + r;
        tc::tma_load_3d(st, &kmap, 0, 64 * blk, plane, &bars[B_KVF + s]);
        tc::tma_load_3d(st + 8192, &kmap, 64, 64 * blk, plane, &bars[B_KVF + s]);
        tc::tma_load_3d(st + 16384, &vmap, 0, 64 * blk, plane, &bars[B_KVF + s]);
        tc::tma_load_3d(st + 24576, &vmap, 64, 64 * blk, plane, &bars[B_KVF + s]);
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_N64 = tc::idesc_bf16(128, 64, 0, 0);     // S, dP
      constexpr uint32_t ID_DQ = tc::idesc_bf16(128, 128, 0, 1);     // dQ += dS K
      constexpr uint32_t ID_T = tc::idesc_bf16(128, 64, 1, 1);       // dK^T, dV^T
      const uint32_t q_a = smem_u32(sm + OFF_Q), do_a = smem_u32(sm + OFF_DO);
      const uint32_t p_a = smem_u32(sm + OFF_P), ds_a = smem_u32(sm + OFF_DS);
      mbar_wait_data(&bars[B_Q], 0, err);
      // S/dP of unit j+1 are issued as soon as the gradient warps have copied
      // S/dP of unit j into registers, so they run while unit j's P and dS are
      // being formed; the dQ / dK^T / dV^T products of unit j follow.
      auto issue_sdp = [&](int j) {
        const int s = j % NKV;
        const uint32_t k_a = smem_u32(sm + OFF_KV + s * KV_STAGE);
        const uint32_t v_a = k_a + 16384;
        mbar_wait_data(&bars[B_KVF + s], (j / NKV) & 1, err);
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
      };
      auto issue_grad = [&](int j) {
        const int s = j & 1;  // dK^T / dV^T TMEM buffer
        const int ks_ = j % NKV;
        const uint32_t k_a = smem_u32(sm + OFF_KV + ks_ * KV_STAGE);
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
        tc::commit(&bars[B_KVE + ks_]);
        tc::commit(&bars[B_KF + s]);
      };
      issue_sdp(0);
      for (int j = 0; j < nunits; ++j) {
        if (j + 1 < nunits) issue_sdp(j + 1);
        issue_grad(j);
      }
    }
  } else if (warp >= 8 + 2) {
    // ---------------------------------------------------------------- flush
    // Warp 10 + i owns TMEM lanes 32((10 + i) % 4).. = head dims of dK^T /
    // dV^T. For each unit, once its MMAs are done, it moves its lane quarter
    // (all 64 keys, both matrices) into [32 keys][32 d] fp32 slices and adds
    // each with one TMA reduce-add (rows past N are clipped by the map; a
    // slice wholly past N is skipped). It releases the unit's TMEM buffer
    // after its last TMEM read. Slices rotate with the count of issued
    // groups: the reduce issued from a slice FSLOT groups earlier must have
    // read it before it is rewritten.
    const int fq = warp & 3;
    const uint32_t lane_off = (uint32_t)(fq * 32) << 16;
    float* tw = reinterpret_cast<float*>(sm + OFF_T) + (warp - 10) * FSLOT * 1024;  // [32][32] slices
    const int plane = b * Hkv + r;
    int ngroups = 0;
    for (int j = 0; j < nunits; ++j) {
      // buffer j & 1 holds unit j: its phase cannot advance again before this
      // warp releases the buffer, so the parity below is never ambiguous
      mbar_wait_data(&bars[B_KF + (j & 1)], (j >> 1) & 1, err);
      tc::fence_after_sync();
      const int blk = unit_block(j);
      const uint32_t cb = tmem + (j & 1) * C_BUF + lane_off;
#pragma unroll 1
      for (int part = 0; part < 4; ++part) {  // (matrix, key half)
        const int m2 = part >> 1, hk = part & 1;
        float kv[32];
        tc::tmem_ld32(cb + (m2 == 0 ? C_DKT : C_DVT) + 32 * hk, kv);
        tc::tmem_wait_ld();
        if (part == 3) {  // the unit's TMEM buffer is no longer read
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[B_TE + (j & 1)]);
        }
        const int key0 = 64 * blk + 32 * hk;
        if (key0 < N) {  // warp-uniform; rows past N are clipped by the map
          float* sl = tw + ((ngroups % FSLOT) << 10);
          if (lane == 0) tc::bulk_wait_read<FSLOT - 1>();
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 32; ++i) sl[i * 32 + lane] = kv[i];
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tc::tma_reduce_add_3d(m2 == 0 ? &dkmap : &dvmap, sl, 32 * fq, key0, plane);
            tc::bulk_commit();
          }
          ++ngroups;
        }
      }
    }
    if (lane == 0) tc::bulk_wait<0>();  // every reduce of this warp has completed
  } else {
    // ---------------------------------------------------------------- gradient rows
    // Warps w and w + 4 share TMEM lanes 32(w%4)..+31 (query rows for S/dP/dQ,
    // head dim for dK^T/dV^T) and split the columns: hc = w / 4 takes keys
    // 32hc..32hc+31 of S/dP/dK^T/dV^T and columns 64hc..64hc+63 of dQ.
    const int wq = warp & 3, hc = warp >> 2;
    const int row = wq * 32 + lane;
    const int hh = row >> 6, qr = row & 63;
    const int pos = 64 * t + qr;
    const bool valid = pos < N;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
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
    } else {
      lse2 = INFINITY;  // rows past N: every p is 2^-inf = 0
    }
    unsigned char* prow = sm + OFF_P + row * 128;
    unsigned char* dsrow = sm + OFF_DS + row * 128;
    const int gtid = hc * 128 + row;  // 0..255 over the gradient warps
    float* dl_s = reinterpret_cast<float*>(sm + OFF_DL);
    // per-token: this row's own list (ascending), walked as the units advance
    const size_t trow = tok0 + (valid ? qr : 0);
    const int tn = (TOK && valid) ? min(max(cnt[trow], 0), topk) : 0;
    const int32_t* tidx = idx + trow * topk;
    const float* tlog = logg + trow * topk;
    int tp = 0;
    for (int j = 0; j < nunits; ++j) {
      const bool cur = (j == kk);
      float bias;
      bool sel = !cur;
      if constexpr (TOK) {
        bias = 0.f;
        if (!cur) {
          const int blk = unit_block(j);
          while (tp < tn && tidx[tp] < blk) ++tp;
          sel = tp < tn && tidx[tp] == blk;
          bias = sel ? tlog[tp] * LOG2E : -INFINITY;
        }
      } else {
        bias = cur ? 0.f : logg_row[j] * LOG2E;
      }
      mbar_wait_data(&bars[B_SF], j & 1, err);
      tc::fence_after_sync();
      float sv[32], dp[32];
      tc::tmem_ld32(tmem + C_S + lane_off + 32 * hc, sv);
      tc::tmem_ld32(tmem + C_DP + lane_off + 32 * hc, dp);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_SE]);
      float dsum = 0.f;
      uint32_t pk[16], dk2[16];
      if (cur) {  // causal mask inside the current block
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (32 * hc + i > qr) sv[i] = -INFINITY;
      }
      const float off = bias - lse2;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float p0 = tc::ex2(fmaf(sv[i], c1, off)), p1 = tc::ex2(fmaf(sv[i + 1], c1, off));
        const float d0 = p0 * (dp[i] - Di), d1 = p1 * (dp[i + 1] - Di);
        dsum += d0 + d1;
        __nv_bfloat162 hp2 = __floats2bfloat162_rn(p0, p1);
        __nv_bfloat162 hd2 = __floats2bfloat162_rn(d0 * scale, d1 * scale);
        pk[i >> 1] = *reinterpret_cast<uint32_t*>(&hp2);
        dk2[i >> 1] = *reinterpret_cast<uint32_t*>(&hd2);
      }
      if (j >= 1) {  // MMAs of the previous unit done: P/dS buffers free, dK^T/dV^T ready
        mbar_wait_data(&bars[B_MD], (j - 1) & 1, err);
        tc::fence_after_sync();
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // 16-byte chunks 4hc..4hc+3 of the row, swizzled
        const int pc = ((4 * hc + c) ^ (row & 7)) << 4;
        *reinterpret_cast<uint4*>(prow + pc) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(dsrow + pc) =
            make_uint4(dk2[4 * c], dk2[4 * c + 1], dk2[4 * c + 2], dk2[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PF]);
      if constexpr (TOK) {  // this row's part (its 32 keys) of its token's slot
        if (sel) atomicAdd(dlogg + trow * topk + tp, dsum);
      } else if (!cur) {  // this warp's part of d(log g) of the slot, summed at the end
        dsum = warp_sum(dsum);
        if (lane == 0) dl_s[j * NGW + warp] = dsum;
      }
    }
    mbar_wait_data(&bars[B_MD], (nunits - 1) & 1, err);
    tc::fence_after_sync();
    named_bar_softmax();
    for (int j = gtid; j < (TOK ? 0 : kk); j += 2 * 128) {  // d(log g): fixed-order sum over the warps
      float a = 0.f;
#pragma unroll
      for (int w = 0; w < NGW; ++w) a += dl_s[j * NGW + w];
      atomicAdd(dlogg + srow * topk + j, a);
    }
    // dQ (already scaled through dS): columns 64hc..64hc+63 of this row
#pragma unroll 1
    for (int c = 2 * hc; c < 2 * hc + 2; ++c) {
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
  if (warp == 9) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host
static bool make_map(CUtensorMap* map, const void* base, int rows_per_plane, int planes) {
  return make_tma_map_bf16_3d(map, base, D, rows_per_plane, planes);
}

template <typename TT>
__global__ void k_convert_tc(const float* __restrict__ src, TT* __restrict__ dst, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = from_f<TT>(src[i]);
}

template <bool TOK>
static cudaError_t launch_bwd_tc(const void* q, const void* k, const void* v, const void* o,
                                 const void* dout, int B, int Hq, int Hkv, int N,
                                 const float* lse, const int32_t* idx, const int32_t* cnt,
                                 const float* logg, int topk, float scale, void* dq, void* dk,
                                 void* dv, float* dlogg, void* ws, cudaStream_t st) {
  const int T_ = (N + 63) / 64;
  if (B == 0 || T_ == 0) return cudaSuccess;
  if (TOK && T_ - 1 > TOK_UMAX) return cudaErrorInvalidValue;
  const size_t nkv = (size_t)B * Hkv * N * D;
  float* dk_acc = static_cast<float*>(ws);
  float* dv_acc = dk_acc + nkv;
  cudaError_t e = cudaMemsetAsync(ws, 0, 2 * nkv * sizeof(float), st);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(dlogg, 0, (size_t)B * Hkv * (TOK ? N : T_) * topk * sizeof(float), st);
  if (e != cudaSuccess) return e;
  CUtensorMap qm, km, vm, dom, dkm, dvm;
  if (!make_map(&qm, q, N, B * Hq) || !make_map(&km, k, N, B * Hkv) ||
      !make_map(&vm, v, N, B * Hkv) || !make_map(&dom, dout, N, B * Hq) ||
      !make_tma_map_f32_3d(&dkm, dk_acc, D, N, B * Hkv, 32, 32) ||
      !make_tma_map_f32_3d(&dvm, dv_acc, D, N, B * Hkv, 32, 32))
    return cudaErrorInvalidValue;
  e = ensure_smem(k_attn_bwd_tc<TOK>, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(T_, Hkv * (Hq / Hkv / 2), B);
  k_attn_bwd_tc<TOK><<<grid, BT_THREADS, SMEM_BYTES, st>>>(
      qm, km, vm, dom, static_cast<const __nv_bfloat16*>(o),
      static_cast<const __nv_bfloat16*>(dout), dkm, dvm, lse, Hq, Hkv, N, idx, cnt, logg, topk,
      scale, static_cast<__nv_bfloat16*>(dq), dlogg);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int cgrid = (int)((nkv + 255) / 256 < 8192 ? (nkv + 255) / 256 : 8192);
  k_convert_tc<__nv_bfloat16><<<cgrid, 256, 0, st>>>(dk_acc, static_cast<__nv_bfloat16*>(dk), nkv);
  k_convert_tc<__nv_bfloat16><<<cgrid, 256, 0, st>>>(dv_acc, static_cast<__nv_bfloat16*>(dv), nkv);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_tc(const void* q, const void* k, const void* v, const void* o,
                               const void* dout, int B, int Hq, int Hkv, int N,
                               const float* lse, const int32_t* idx, const int32_t* cnt,
                               const float* logg, int topk, float scale, void* dq, void* dk,
                               void* dv, float* dlogg, void* ws, cudaStream_t st) {
  return launch_bwd_tc<false>(q, k, v, o, dout, B, Hq, Hkv, N, lse, idx, cnt, logg, topk, scale,
                              dq, dk, dv, dlogg, ws, st);
}

cudaError_t launch_attn_bwd_tc_tokens(const void* q, const void* k, const void* v,
                                      const void* o, const void* dout, int B, int Hq, int Hkv,
                                      int N, const float* lse, const int32_t* idx,
                                      const int32_t* cnt, const float* logg, int topk,
                                      float scale, void* dq, void* dk, void* dv, float* dlogg,
                                      void* ws, cudaStream_t st) {
  return launch_bwd_tc<true>(q, k, v, o, dout, B, Hq, Hkv, N, lse, idx, cnt, logg, topk, scale,
                             dq, dk, dv, dlogg, ws, st);
}

uint32_t* attn_bwd_tc_error_word() {
  void* p = nullptr;
  cudaGetSymbolAddress(&p, g_attn_bwd_tc_err);
  return static_cast<uint32_t*>(p);
}

}  // namespace sas
