// fp32 SIMT tiles shared by the CUDA-core attention kernels: 64-row tiles in
// shared memory with a row stride of d + 4 floats (the 16-byte row reads of
// a quarter warp fall in distinct banks), a 64 x 64 tile product and the
// half-warp reductions of the thread layout (tr, tc) = (tid / 16, tid % 16).
#pragma once
#include "common.cuh"

namespace sas {

constexpr int AT_THREADS = 256;

template <int D> struct AtShape {
  static constexpr int LD = D + 4;        // fp32 row stride of Q/K/V/dO tiles
  static constexpr int PLD = SAS_BLOCK + 4;
  static constexpr int NG = D / 64;       // float4 column groups per thread
  static constexpr int TILE = SAS_BLOCK * LD;
};

// Loads rows [row0, row0 + 64) of a [N][D] slab (rows >= nvalid become 0)
// into an fp32 tile with stride LD.
template <typename T, int D>
__device__ __forceinline__ void load_tile(float* dst, const T* src, int nvalid) {
  constexpr int VEC = Vec16<T>::N;
  constexpr int PER_ROW = D / VEC;
  for (int e = threadIdx.x; e < SAS_BLOCK * PER_ROW; e += AT_THREADS) {
    const int rr = e / PER_ROW, cc = (e % PER_ROW) * VEC;
    float x[VEC];
    if (rr < nvalid) {
      Vec16<T>::load_nc(src + (size_t)rr * D + cc, x);
    } else {
#pragma unroll
      for (int i = 0; i < VEC; ++i) x[i] = 0.f;
    }
    float* d = dst + rr * AtShape<D>::LD + cc;
#pragma unroll
    for (int i = 0; i < VEC; i += 4)
      *reinterpret_cast<float4*>(d + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
  }
}

// s[ii][jj] = A[tr + 16 ii] . B[tc + 16 jj] over D (fp32 tiles, stride LD).
template <int D>
__device__ __forceinline__ void tile_dot(const float* A, const float* Bt, int tr, int tc,
                                         float s[4][4]) {
  constexpr int LD = AtShape<D>::LD;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) s[i][j] = 0.f;
#pragma unroll 4
  for (int c = 0; c < D; c += 4) {
    float4 a[4], bb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(A + (tr + 16 * i) * LD + c);
#pragma unroll
    for (int j = 0; j < 4; ++j) bb[j] = *reinterpret_cast<const float4*>(Bt + (tc + 16 * j) * LD + c);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        s[i][j] += a[i].x * bb[j].x + a[i].y * bb[j].y + a[i].z * bb[j].z + a[i].w * bb[j].w;
  }
}

// Reductions over the 16 lanes that share tr (one half warp).
__device__ __forceinline__ float half_max(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float half_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace sas
