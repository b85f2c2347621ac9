// k_gemv.cu -- fused trellis decode + GEMV / small-batch product on CUDA cores.
//
// y[t][n] = bf16( sum_k w[n][k] x[t][k] ), w decoded in registers from the resident stream
// (HEPH abstract, first serving mode). HBM-bound in principle: 0.28125 B/weight of stream and
// scales; every CTA stages the activations once in shared memory and then streams rows.
#include <cuda_bf16.h>

#include "tcf4_internal.h"
#include "tcf4_rowdot.cuh"

namespace tcf4 {

// Stage activations x[tok][K] (bf16) for TT token slots into the permuted fp32 layout, 8 values
// (one 16-byte load) per step. Missing token slots are zero.
template <int TT>
__device__ __forceinline__ void stage_x_vec(float2 *xs, const uint16_t *__restrict__ x, int K, const int *tok,
                                            int ntok) {
  const int nb = K >> 5;
  const int groups = K >> 3;  // 8-element groups per token
  for (int idx = threadIdx.x; idx < TT * groups; idx += blockDim.x) {
    const int t = idx / groups, gi = idx - t * groups;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (t < ntok) raw = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)tok[t] * K) + gi);
    const int blk = gi >> 2, u = gi & 3;  // elements 8u..8u+7 of block blk
    const uint32_t r[4] = {raw.x, raw.y, raw.z, raw.w};
    float2 *dst = xs + (size_t)t * nb * 16 + blk * 16 + u;
#pragma unroll
    for (int jj = 0; jj < 4; jj++) {
      // element 8u+jj sits in r[jj/2] half (jj&1); element 8u+4+jj in r[2 + jj/2] half (jj&1)
      const uint32_t lo = r[jj >> 1], hi = r[2 + (jj >> 1)];
      const float a = __uint_as_float((jj & 1) ? (lo & 0xFFFF0000u) : (lo << 16));
      const float b = __uint_as_float((jj & 1) ? (hi & 0xFFFF0000u) : (hi << 16));
      dst[jj * 4] = make_float2(a, b);
    }
  }
}

template <int TT, bool SEG32>
__global__ void __launch_bounds__(256) k_gemv(MatView w, const uint16_t *__restrict__ x, int T,
                                              uint16_t *__restrict__ y) {
  extern __shared__ float4 smem_f4[];
  float2 *xs = reinterpret_cast<float2 *>(smem_f4);
  const int K = w.nbr * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t0 = 0; t0 < T; t0 += TT) {
    const int ntok = min(TT, T - t0);
    int tok[TT];
#pragma unroll
    for (int t = 0; t < TT; t++) tok[t] = t0 + t;
    __syncthreads();
    stage_x_vec<TT>(xs, x, K, tok, ntok);
    __syncthreads();
    for (int r = blockIdx.x * 8 + warp; r < w.rows; r += gridDim.x * 8) {
      float acc[TT];
      row_dot<TT, SEG32>(w.stream + (size_t)r * w.nbr, w.scales + (size_t)r * w.nbr, w.nbr, w.seg_blocks, xs, acc);
      if (lane < ntok) {
        float a = acc[0];
#pragma unroll
        for (int t = 1; t < TT; t++)
          if (lane == t) a = acc[t];
        y[(size_t)(t0 + lane) * w.rows + r] = __bfloat16_as_ushort(__float2bfloat16_rn(a));
      }
    }
  }
}

template <int TT, bool SEG32>
static cudaError_t launch_gemv_t(const MatView &w, const uint16_t *x, int T, uint16_t *y, cudaStream_t s) {
  const size_t smem = (size_t)TT * w.nbr * 32 * sizeof(float);
  static bool attr_set = false;  // benign race: setting the same attribute twice is harmless
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_gemv<TT, SEG32>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int per_sm = smem <= 56 * 1024 ? 4 : (smem <= 110 * 1024 ? 2 : 1);
  int grid = (w.rows + 7) / 8;
  if (grid > nsm * per_sm) grid = nsm * per_sm;
  k_gemv<TT, SEG32><<<grid, 256, smem, s>>>(w, x, T, y);
  return cudaGetLastError();
}

cudaError_t launch_gemv(const MatView &w, const uint16_t *x, int T, uint16_t *y, cudaStream_t s) {
  const int K = w.nbr * 32;
  int TT = T >= 3 ? 4 : T;
  while (TT > 1 && (size_t)TT * K * sizeof(float) > 200 * 1024) TT >>= 1;
  const bool seg32 = w.seg_blocks == 1;
  switch (TT) {
    case 1: return seg32 ? launch_gemv_t<1, true>(w, x, T, y, s) : launch_gemv_t<1, false>(w, x, T, y, s);
    case 2: return seg32 ? launch_gemv_t<2, true>(w, x, T, y, s) : launch_gemv_t<2, false>(w, x, T, y, s);
    default: return seg32 ? launch_gemv_t<4, true>(w, x, T, y, s) : launch_gemv_t<4, false>(w, x, T, y, s);
  }
}

}  // namespace tcf4
