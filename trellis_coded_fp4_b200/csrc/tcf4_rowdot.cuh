// tcf4_rowdot.cuh -- warp-cooperative fused decode + dot product of one trellis-coded row.
//
// HEPH's first serving mode ("HEPH ..." abstract): the compressed stream stays resident and the
// weights are decoded inside the product kernel on every call. A warp owns one row: lane l takes
// the 32-weight blocks l, l+32, ... of the row (coalesced 8-byte loads), decodes each block in
// registers (bit-sliced, tcf4_device.cuh), converts codes to half2 with the hardware E2M1
// conversion, multiplies against fp32 activations staged in shared memory and accumulates in fp32.
// The block's UE8M0 scale (a power of two) is applied once to the block's partial sum, which is
// exact. A warp-shuffle reduction finishes the row.
//
// Activations are staged per 32-weight block in the order the interleaved nibble words produce
// them: entry (jj, u) of a block holds the pair (x[8u+jj], x[8u+4+jj]) as float2, because byte u
// of interleaved word jj holds the codes of weights 8u+jj (low nibble) and 8u+4+jj (high nibble).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "tcf4_device.cuh"

namespace tcf4 {

constexpr unsigned kFull = 0xffffffffu;

// Shared-memory activation layout: xs[t][block][16] float2.
__device__ __forceinline__ int xs_index(int block, int k_in_block) {
  const int u = k_in_block >> 3, h = (k_in_block >> 2) & 1, jj = k_in_block & 3;
  return (block * 16 + jj * 4 + u) * 2 + h;
}

// Stage bf16 activations x[T][K] rows src_tok[0..TT) into xs (zeros for missing tokens).
template <int TT>
__device__ __forceinline__ void stage_x(float *xs, const __nv_bfloat16 *x, int K, const int *tok, int ntok) {
  const int nb = K >> 5;
  for (int idx = threadIdx.x; idx < TT * K; idx += blockDim.x) {
    const int t = idx / K, k = idx - t * K;
    float v = 0.f;
    if (t < ntok) v = __bfloat162float(x[(size_t)tok[t] * K + k]);
    xs[(size_t)t * nb * 32 + xs_index(k >> 5, k & 31)] = v;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Accumulate one decoded block against TT tokens: bsum[t] = sum over the block of code * x.
template <int TT>
__device__ __forceinline__ void block_dot(const Planes &P, const float2 *xb, int tok_stride, float *bsum) {
  uint32_t W[4];
  planes_to_nibbles_interleaved(P, W[0], W[1], W[2], W[3]);
#pragma unroll
  for (int jj = 0; jj < 4; jj++) {
    uint32_t h[4];
    e2m1x8_to_f16x2x4(W[jj], h[0], h[1], h[2], h[3]);
#pragma unroll
    for (int u = 0; u < 4; u++) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h[u]));
#pragma unroll
      for (int t = 0; t < TT; t++) {
        const float2 xv = xb[t * tok_stride + jj * 4 + u];
        bsum[t] = fmaf(f.x, xv.x, bsum[t]);
        bsum[t] = fmaf(f.y, xv.y, bsum[t]);
      }
    }
  }
}

// One row: returns (in every lane) the full dot products acc[t] for t < TT.
// srow/scrow: the row's blocks and scales; nbr blocks; seg_blocks blocks per segment.
// xs: staged activations (TT tokens, stride nbr*16 float2 per token).
template <int TT, bool SEG32>
__device__ __forceinline__ void row_dot(const uint2 *__restrict__ srow, const uint8_t *__restrict__ scrow, int nbr,
                                        int seg_blocks, const float2 *xs, float *acc) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int t = 0; t < TT; t++) acc[t] = 0.f;
  uint32_t cL = 0u, cH = 0u;  // planes of the block before this iteration's lane-0 block
  for (int j0 = 0; j0 < nbr; j0 += 32) {
    const int j = j0 + lane;
    uint2 v = make_uint2(0u, 0u);
    uint32_t E = 127u;
    if (j < nbr) {
      v = __ldg(srow + j);
      E = __ldg(scrow + j);
    }
    Planes P;
    if (SEG32) {
      P = decode_block0(v.x, v.y);
    } else {
      uint32_t pL = __shfl_up_sync(kFull, v.x, 1), pH = __shfl_up_sync(kFull, v.y, 1);
      if (lane == 0) {
        pL = cL;
        pH = cH;
      }
      if (j % seg_blocks == 0) {
        pL = 0u;
        pH = 0u;
      }
      cL = __shfl_sync(kFull, v.x, 31);
      cH = __shfl_sync(kFull, v.y, 31);
      P = decode_block(v.x, v.y, pL, pH);
    }
    if (j < nbr) {
      float bsum[TT];
#pragma unroll
      for (int t = 0; t < TT; t++) bsum[t] = 0.f;
      block_dot<TT>(P, xs + (size_t)j * 16, nbr * 16, bsum);
      const float sc = ue8m0_to_float(E);
#pragma unroll
      for (int t = 0; t < TT; t++) acc[t] = fmaf(bsum[t], sc, acc[t]);
    }
  }
#pragma unroll
  for (int t = 0; t < TT; t++) acc[t] = warp_sum(acc[t]);
}

}  // namespace tcf4
