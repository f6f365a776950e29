// Gated sparse attention forward on the 5th-generation tensor cores (bf16,
// d = 128): TMA-fed tcgen05 MMAs with TMEM accumulators.
//
// Definition (SAS close reading, liuzhao09.github.io, sections 2.1, 2.2 and
// 2.4; SAS reproduction note, daiwk.github.io, core formula): for query row i
// of block t, z_ij = scale * q_i . k_j + log g of j's block over the kept
// history blocks, and z_ij = scale * q_i . k_j over keys j <= i of the
// current block; o_i = softmax(z) V, lse_i = log sum exp z. The gate is added
// to the QK^T tile before the online-softmax update; unselected blocks are
// never loaded; the score matrix is never materialised.
//
// One CTA per (query block t, kv group r, pair of query heads of the group):
// an M = 128 tile (2 heads x 64 rows) that shares every K/V block it loads.
//   warp 4     TMA producers: lane 0 loads Q once (4 boxes of 64 rows x 64
//              columns, 128-byte swizzle) and then K of each unit, lane 1 V
//              of each unit, each into its own 2-stage ring (a K slot is
//              released when S_j is done, a V slot when PV_j is);
//   warp 5     one elected thread issues tcgen05.mma: S_j = Q K_j^T
//              (M128 N64 K128, two TMEM buffers of 64 columns) and
//              O += P_j V_j (M128 N128 K64, 128 TMEM columns, the A operand
//              P_j read from TMEM); S_j waits until PV_{j-2} has read P_{j-2}
//              from the buffer S_j overwrites;
//   warps 0-3  softmax: thread i owns row i = TMEM lane i; loads S_j,
//              applies scale, bias and the causal mask in the log2 domain,
//              updates the running max lazily (O in TMEM is rescaled only when
//              the max grows by more than 2^8), writes P_j as bf16 (two per
//              column) over the first half of S_j's TMEM buffer; at the end
//              divides O by the row sum and writes o and lse.
// About 97 KB of shared memory and 256 TMEM columns per CTA, so two CTAs
// share an SM and overlap one's softmax with the other's MMAs. Every wait is
// bounded.
//
// Per-token selection (TOK = true; section 2.4: the fused kernel masks, per
// query, the blocks below that query's gate threshold and skips a key tile no
// query of the tile selected): every query token has its own selection row.
// The CTA first builds the union of the blocks its 64 tokens selected
// (ascending); the units are that union, then the current block. For a
// history unit, row i adds its token's log g when its token selected the
// unit's block and masks the whole unit (-inf) otherwise; each row finds that
// by walking its own ascending list as the units advance. MMAs and softmax
// are otherwise the same.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "tc.cuh"

namespace sas {

__device__ uint32_t g_attn_fwd_tc_err = 0;

namespace {

constexpr int FT_THREADS = 192;
constexpr int D = 128;
constexpr uint32_t Q_BYTES = 128 * D * 2;           // 32 KB
constexpr uint32_t KV_STAGE_BYTES = 2 * 64 * D * 2;  // K + V block, 32 KB
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_KV = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_BAR = OFF_KV + 2 * KV_STAGE_BYTES;
constexpr uint32_t OFF_UM = OFF_BAR + 128;  // per-token mode: union bitmask and its count
constexpr uint32_t SMEM_BYTES = OFF_UM + 128;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_LOG2 = 8.0f;  // lazy rescale threshold (log2 units)
constexpr int TOK_UMAX = 512;         // history blocks of a query block at most (per-token mode)

// K_j and V_j have their own full/empty barriers: a K slot is free once S_j is
// done, a V slot once PV_j is done, so the next K load starts a softmax earlier.
enum Bar {
  B_Q = 0, B_KF = 1, B_KE = 3, B_SF = 5, B_PF = 7, B_OD = 8, B_VF = 9, B_VE = 11, NBAR = 13
};
static_assert(NBAR * 8 + 4 <= 128, "barriers and the TMEM address fit their 128 bytes");

// (a0, a1) = (x0, x1) * c + (o, o) as one packed fp32x2 FMA
__device__ __forceinline__ void fma2c(float& a0, float& a1, float x0, float x1, float c, float o) {
  asm("{\n\t.reg .b64 x, c, o, a;\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 c, {%4, %4};\n\t"
      "mov.b64 o, {%5, %5};\n\t"
      "fma.rn.f32x2 a, x, c, o;\n\t"
      "mov.b64 {%0, %1}, a;\n\t}"
      : "=f"(a0), "=f"(a1)
      : "f"(x0), "f"(x1), "f"(c), "f"(o));
}
// (s0, s1) += (x0, x1) as one packed fp32x2 add
__device__ __forceinline__ void add2(float& s0, float& s1, float x0, float x1) {
  asm("{\n\t.reg .b64 s, x;\n\t"
      "mov.b64 s, {%0, %1};\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "add.rn.f32x2 s, s, x;\n\t"
      "mov.b64 {%0, %1}, s;\n\t}"
      : "+f"(s0), "+f"(s1)
      : "f"(x0), "f"(x1));
}

// O += P V with the A operand (P, bf16, 128 lanes x 16 elements packed two
// per 32-bit column) read from TMEM and B from shared memory.
__device__ __forceinline__ void mma_bf16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns from registers (lane of the warp's
// quarter, columns taddr.col .. +31)
__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
      "%10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, "
      "%27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// max(a, b, c) in one instruction
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

}  // namespace

template <bool TOK>
__global__ void __launch_bounds__(FT_THREADS, 2) k_attn_fwd_tc(
    const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
    const __grid_constant__ CUtensorMap vmap, int Hq, int Hkv, int N,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
    const float* __restrict__ logg, int topk, float scale, __nv_bfloat16* __restrict__ o,
    float* __restrict__ lse) {
  extern __shared__ __align__(1024) unsigned char sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + NBAR * 8);
  uint32_t* err = &g_attn_fwd_tc_err;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = Hq / Hkv, pairs = G / 2;
  const int T_ = gridDim.x;
  const int t = T_ - 1 - (int)blockIdx.x;  // longest rows first
  const int r = blockIdx.y / pairs, hp = blockIdx.y % pairs, b = blockIdx.z;
  const int h0 = r * G + 2 * hp;
  const size_t srow = ((size_t)b * Hkv + r) * T_ + t;
  // per query block: kept history blocks; per token: the union of the
  // tokens' blocks (built below); then the current block
  int kk = TOK ? 0 : min(max(cnt[srow], 0), topk);
  const int32_t* idx_row = idx + (TOK ? 0 : srow * topk);
  const float* logg_row = logg + (TOK ? 0 : srow * topk);
  if ((smem_u32(sm) & 1023u) != 0) {  // swizzled tiles need 1024-byte alignment
    if (tid == 0) atomicOr(err, kErrBadIndex);
    return;
  }
  const size_t tok0 = ((size_t)b * Hkv + r) * N + 64 * t;  // first token row of the block
  const int nr = min(64, N - 64 * t);
  // the union as a bitmask over the t history blocks; each consumer walks it
  // in ascending order with its own cursor (next_unit)
  const uint32_t* umask_p = nullptr;
  const int words = (t + 31) / 32;
  if constexpr (TOK) {
    uint32_t* umask = reinterpret_cast<uint32_t*>(sm + OFF_UM);  // TOK_UMAX / 32 words
    int& ucnt = *reinterpret_cast<int*>(sm + OFF_UM + TOK_UMAX / 8);
    umask_p = umask;
    for (int w = tid; w < words; w += FT_THREADS) umask[w] = 0u;
    __syncthreads();
    for (int e = tid; e < nr * topk; e += FT_THREADS) {
      const int i = e / topk, p = e - i * topk;
      if (p < min(max(cnt[tok0 + i], 0), topk)) {
        const int m = idx[(tok0 + i) * topk + p];
        if (m >= 0 && m < t) atomicOr(&umask[m >> 5], 1u << (m & 31));
        else atomicOr(err, kErrBadIndex);
      }
    }
    __syncthreads();
    if (warp == 0) {  // the number of units
      int c = 0;
      for (int w = lane; w < words; w += 32) c += __popc(umask[w]);
      c = __reduce_add_sync(0xffffffffu, c);
      if (lane == 0) ucnt = c;
    }
    __syncthreads();
    kk = ucnt;
  }
  // smallest selected block >= from (the union is ascending), -1 past the end
  auto next_unit = [&](int from) -> int {
    for (int w = from >> 5; w < words; ++w) {
      const uint32_t word = umask_p[w] & (w == (from >> 5) ? (~0u << (from & 31)) : ~0u);
      if (word) return w * 32 + __ffs(word) - 1;
    }
    return -1;
  };
  const int nunits = kk + 1;  // history units, then the current block
  if (tid == 0) {
    // P-full takes one arrival per softmax warp
    for (int i = 0; i < NBAR; ++i)
      mbar_init(&bars[i], i == B_PF ? 4 : 1);
    fence_mbar_init();
  }
  if (warp == 5) tc::tmem_alloc(tmem_slot, 256);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_s[2] = {tmem, tmem + 64};
  const uint32_t tm_o = tmem + 128;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer
    // lane 0: Q, then K of every unit; lane 1: V of every unit
    if (lane < 2) {
      const bool kl = (lane == 0);
      if (kl) {
        tc::prefetch_map(&qmap);
        tc::prefetch_map(&kmap);
        mbar_arrive_expect_tx(&bars[B_Q], Q_BYTES);
        for (int c = 0; c < 2; ++c)
          for (int h = 0; h < 2; ++h)
            tc::tma_load_3d(sm + OFF_Q + c * 16384 + h * 8192, &qmap, 64 * c, 64 * t,
                            b * Hq + h0 + h, &bars[B_Q]);
      } else {
        tc::prefetch_map(&vmap);
      }
      const CUtensorMap* map = kl ? &kmap : &vmap;
      uint64_t* fullb = &bars[kl ? B_KF : B_VF];
      uint64_t* emptyb = &bars[kl ? B_KE : B_VE];
      const uint32_t half = kl ? 0u : 16384u;
      int ucur = -1;  // per-token: the previous unit's block
      for (int j = 0; j < nunits; ++j) {
        const int s = j & 1;
        if (j >= 2) mbar_wait_data(&emptyb[s], ((j >> 1) - 1) & 1, err);
        if (TOK && j < kk) ucur = next_unit(ucur + 1);
        int blk = (j < kk) ? (TOK ? ucur : idx_row[j]) : t;
        if (blk < 0 || blk >= t) {
          if (j < kk && kl) atomicOr(err, kErrBadIndex);
          blk = t;
        }
        unsigned char* st = sm + OFF_KV + s * KV_STAGE_BYTES + half;
        mbar_arrive_expect_tx(&fullb[s], KV_STAGE_BYTES / 2);
        const int plane = b * Hkv + r;
        tc::tma_load_3d(st, map, 0, 64 * blk, plane, &fullb[s]);
        tc::tma_load_3d(st + 8192, map, 64, 64 * blk, plane, &fullb[s]);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_QK = tc::idesc_bf16(128, 64, 0, 0);
      constexpr uint32_t ID_PV = tc::idesc_bf16(128, 128, 0, 1);
      const uint32_t q_addr = smem_u32(sm + OFF_Q);
      mbar_wait_data(&bars[B_Q], 0, err);
      auto pv = [&](int j) {  // O += P_j V_j
        mbar_wait(&bars[B_PF], j & 1, err);
        mbar_wait_data(&bars[B_VF + (j & 1)], (j >> 1) & 1, err);
        tc::fence_after_sync();
        const uint32_t v_addr = smem_u32(sm + OFF_KV + (j & 1) * KV_STAGE_BYTES + 16384);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {  // P_j: columns 8 ks .. 8 ks + 7 of S_j's buffer
          const uint64_t bd = tc::sw128_desc(v_addr + ks * 2048, 8192, 1024);
          mma_bf16_tmem_a(tm_o, tm_s[j & 1] + 8 * ks, bd, ID_PV, (j > 0 || ks > 0) ? 1u : 0u);
        }
        tc::commit(&bars[B_OD]);
        tc::commit(&bars[B_VE + (j & 1)]);
      };
      for (int j = 0; j < nunits; ++j) {
        const int s = j & 1;
        mbar_wait_data(&bars[B_KF + s], (j >> 1) & 1, err);
        // S_j overwrites P_{j-2} (S_{j-2}'s buffer): PV_{j-2} must have read it
        if (j >= 2) mbar_wait(&bars[B_OD], (j - 2) & 1, err);
        tc::fence_after_sync();
        const uint32_t k_addr = smem_u32(sm + OFF_KV + s * KV_STAGE_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // K = 128 in steps of 16 (32 bytes)
          const uint32_t c = ks >> 2, off = (ks & 3) * 32;
          const uint64_t a = tc::sw128_desc(q_addr + c * 16384 + off, 16, 1024);
          const uint64_t bd = tc::sw128_desc(k_addr + c * 8192 + off, 16, 1024);
          tc::mma_bf16(tm_s[s], a, bd, ID_QK, ks > 0 ? 1u : 0u);
        }
        tc::commit(&bars[B_SF + s]);
        tc::commit(&bars[B_KE + s]);
        if (j >= 1) pv(j - 1);
      }
      pv(nunits - 1);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int row = tid;  // 0..127 = TMEM lane
    const int hh = row >> 6, qr = row & 63;
    const int pos = 64 * t + qr;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float c1 = scale * LOG2E;
    float m = -1e30f, l = 0.f;
    // per-token selection: this row's own list (ascending), walked as the
    // units advance; rows past the sequence end select nothing
    const size_t trow = tok0 + (pos < N ? qr : 0);
    const int tn = (TOK && pos < N) ? min(max(cnt[trow], 0), topk) : 0;
    const int32_t* tidx = idx + trow * topk;
    const float* tlog = logg + trow * topk;
    int tp = 0, ucur = -1;
    for (int j = 0; j < nunits; ++j) {
      const int s = j & 1;
      const bool cur = (j == kk);
      float bias;
      if constexpr (TOK) {
        bias = 0.f;
        if (!cur) {
          ucur = next_unit(ucur + 1);
          const int blk = ucur;
          while (tp < tn && tidx[tp] < blk) ++tp;
          bias = (tp < tn && tidx[tp] == blk) ? tlog[tp] * LOG2E : -INFINITY;
        }
      } else {
        bias = cur ? 0.f : logg_row[j] * LOG2E;
      }
      mbar_wait_data(&bars[B_SF + s], (j >> 1) & 1, err);
      tc::fence_after_sync();
      float z[64];
      {
        float a[32], bb[32];
        tc::tmem_ld32(tm_s[s] + lane_off, a);
        tc::tmem_ld32(tm_s[s] + lane_off + 32, bb);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          z[i] = a[i];
          z[32 + i] = bb[i];
        }
      }
      // the row max in the log2 domain: c1 > 0, so max_i (z_i c1 + bias) = c1 max_i z_i + bias
      if (cur) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i > qr) z[i] = -INFINITY;  // causal mask of the current block
      }
      float zm[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) zm[c] = fmaxf(z[2 * c], z[2 * c + 1]);
#pragma unroll
      for (int i = 8; i < 64; i += 8) {
#pragma unroll
        for (int c = 0; c < 4; ++c) zm[c] = max3(zm[c], z[i + 2 * c], z[i + 2 * c + 1]);
      }
      const float mx = max3(zm[0], zm[1], fmaxf(zm[2], zm[3])) * c1 + bias;
      const float mnew = fmaxf(m, mx);
      const bool grow = (j == 0) || (mnew > m + RESCALE_LOG2);
      const float muse = grow ? mnew : m;
      const float off = bias - muse;  // -inf where the row masks the whole unit
      float rs0 = 0.f, rs1 = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float a0, a1;
        fma2c(a0, a1, z[2 * i], z[2 * i + 1], c1, off);
        const float p0 = tc::ex2(a0), p1 = tc::ex2(a1);
        add2(rs0, rs1, p0, p1);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[i] = *reinterpret_cast<uint32_t*>(&h2);
      }
      const float rs = rs0 + rs1;
      if (j > 0) {
        // PV_{j-1} done before O is rescaled. Waiting on every unit also keeps
        // this thread within one phase of the O-done barrier, so that its
        // parity waits (here and at the end) are never a phase behind.
        mbar_wait_data(&bars[B_OD], (j - 1) & 1, err);
        tc::fence_after_sync();
        const float alpha = grow ? tc::ex2(m - muse) : 1.f;
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float ov[32];
            tc::tmem_ld32(tm_o + lane_off + 32 * c, ov);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= alpha;
            tc::tmem_st32(tm_o + lane_off + 32 * c, ov);
          }
          tc::tmem_wait_st();
        }
        l = l * alpha + rs;
      } else {
        l = rs;
      }
      m = muse;
      // P_j (64 bf16, two per column) into the first 32 columns of S_j's
      // buffer, this thread's lane: the A operand of O += P_j V_j
      tmem_st32u(tm_s[s] + lane_off, pk);
      tc::tmem_wait_st();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[B_PF]);
    }
    // epilogue
    mbar_wait_data(&bars[B_OD], (nunits - 1) & 1, err);
    tc::fence_after_sync();
    const float inv = 1.f / l;
    const bool valid = pos < N;
    __nv_bfloat16* orow = o + (((size_t)b * Hq + h0 + hh) * N + (valid ? pos : 0)) * D;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      float ov[32];
      tc::tmem_ld32(tm_o + lane_off + 32 * c, ov);
      tc::tmem_wait_ld();
      if (valid) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(ov[8 * g + 2 * e] * inv,
                                                      ov[8 * g + 2 * e + 1] * inv);
            w[e] = *reinterpret_cast<uint32_t*>(&h2);
          }
          *reinterpret_cast<uint4*>(orow + 32 * c + 8 * g) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    if (valid) lse[((size_t)b * Hq + h0 + hh) * N + pos] = (m + log2f(l)) / LOG2E;
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------ host
static bool make_map(CUtensorMap* map, const void* base, int rows_per_plane, int planes) {
  return make_tma_map_bf16_3d(map, base, D, rows_per_plane, planes);
}

bool attn_fwd_tc_supported(int bf16, int d, int Hq, int Hkv) {
  const int G = Hq / Hkv;
  return bf16 && d == 128 && G >= 2 && (G % 2) == 0;
}

template <bool TOK>
static cudaError_t launch_fwd_tc(const void* q, const void* k, const void* v, int B, int Hq,
                                 int Hkv, int N, const int32_t* idx, const int32_t* cnt,
                                 const float* logg, int topk, float scale, void* o, float* lse,
                                 cudaStream_t st) {
  const int T_ = (N + 63) / 64;
  if (B == 0 || T_ == 0) return cudaSuccess;
  if (TOK && T_ - 1 > TOK_UMAX) return cudaErrorInvalidValue;
  CUtensorMap qm, km, vm;
  if (!make_map(&qm, q, N, B * Hq) || !make_map(&km, k, N, B * Hkv) ||
      !make_map(&vm, v, N, B * Hkv))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem(k_attn_fwd_tc<TOK>, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(T_, Hkv * (Hq / Hkv / 2), B);
  k_attn_fwd_tc<TOK><<<grid, FT_THREADS, SMEM_BYTES, st>>>(
      qm, km, vm, Hq, Hkv, N, idx, cnt, logg, topk, scale, static_cast<__nv_bfloat16*>(o), lse);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_tc(const void* q, const void* k, const void* v, int B, int Hq,
                               int Hkv, int N, const int32_t* idx, const int32_t* cnt,
                               const float* logg, int topk, float scale, void* o, float* lse,
                               cudaStream_t st) {
  return launch_fwd_tc<false>(q, k, v, B, Hq, Hkv, N, idx, cnt, logg, topk, scale, o, lse, st);
}

cudaError_t launch_attn_fwd_tc_tokens(const void* q, const void* k, const void* v, int B, int Hq,
                                      int Hkv, int N, const int32_t* idx, const int32_t* cnt,
                                      const float* logg, int topk, float scale, void* o,
                                      float* lse, cudaStream_t st) {
  return launch_fwd_tc<true>(q, k, v, B, Hq, Hkv, N, idx, cnt, logg, topk, scale, o, lse, st);
}

uint32_t* attn_fwd_tc_error_word() {
  void* p = nullptr;
  cudaGetSymbolAddress(&p, g_attn_fwd_tc_err);
  return static_cast<uint32_t*>(p);
}

}  // namespace sas
