// tcf4_rowdot.cuh -- warp-cooperative fused decode + dot products of trellis-coded rows.
//
// HEPH's first serving mode ("HEPH ..." abstract): the compressed stream stays resident and the
// weights are decoded inside the product kernel on every call. A warp owns RPW rows of a slab that
// sits in shared memory: lane l takes the 32-weight blocks l, l+32, ... of each row, decodes every
// block in registers (bit-sliced, tcf4_device.cuh), converts the codes to half2 with the hardware
// E2M1 conversion, and multiplies them against fp32 activations staged in shared memory, with fp32
// accumulation. Activations are read once per block and reused for the RPW rows. The block's UE8M0
// scale (a power of two) is applied once to the block's partial sum, which is exact. A warp-shuffle
// reduction finishes each row.
//
// Activations are staged per 32-weight block in the order the interleaved nibble words produce
// them: entry (jj, u) of a block holds the pair (x[8u+jj], x[8u+4+jj]) as float2, because byte u
// of interleaved word jj holds the codes of weights 8u+jj (low nibble) and 8u+4+jj (high nibble).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "tcf4_device.cuh"
#include "tcf4_pipe.cuh"

namespace tcf4 {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Stage bf16 activations (rows tok[0..ntok) of src [*][K]) for TT token slots into the permuted
// fp32 layout, 8 values (one 16-byte load) per step; token slots >= ntok are zero.
template <int TT>
__device__ __forceinline__ void stage_x(float2 *xs, const uint16_t *__restrict__ src, int K, const int *tok,
                                        int ntok) {
  const int nb = K >> 5, groups = K >> 3;
  for (int idx = threadIdx.x; idx < TT * groups; idx += blockDim.x) {
    const int t = idx / groups, gi = idx - t * groups;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (t < ntok) raw = __ldg(reinterpret_cast<const uint4 *>(src + (size_t)tok[t] * K) + gi);
    const int blk = gi >> 2, u = gi & 3;  // elements 8u..8u+7 of block blk
    const uint32_t r[4] = {raw.x, raw.y, raw.z, raw.w};
    float2 *dst = xs + (size_t)t * nb * 16 + blk * 16 + u;
#pragma unroll
    for (int jj = 0; jj < 4; jj++) {
      // element 8u+jj is half (jj&1) of r[jj/2]; element 8u+4+jj is half (jj&1) of r[2+jj/2]
      const uint32_t lo = r[jj >> 1], hi = r[2 + (jj >> 1)];
      const float a = __uint_as_float((jj & 1) ? (lo & 0xFFFF0000u) : (lo << 16));
      const float b = __uint_as_float((jj & 1) ? (hi & 0xFFFF0000u) : (hi << 16));
      dst[jj * 4] = make_float2(a, b);
    }
  }
}

// Dot products of RPW rows held in shared memory with TT staged tokens.
//   st_base / sc_base: shared addresses of row 0's stream words / scales (row stride nbr*8 / nbr);
//   rows: warp-local row indices row_id[q] (q < RPW), valid when row_ok[q];
//   xs_base: shared address of the staged activations (token stride nbr*16 float2).
// Returns in every lane acc[q][t] = full dot product. E5M3: the scale bytes are E5M3 block scales
// (not exact powers of two, so the scaled partial sum is rounded once to fp32).
template <int RPW, int TT, bool SEG32, bool E5M3 = false>
__device__ __forceinline__ void rows_dot_smem(uint32_t st_base, uint32_t sc_base, int nbr, int seg_blocks,
                                              const int *row_id, const bool *row_ok, uint32_t xs_base,
                                              float (&acc)[RPW][TT]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int q = 0; q < RPW; q++)
#pragma unroll
    for (int t = 0; t < TT; t++) acc[q][t] = 0.f;
  uint32_t cL[RPW], cH[RPW];
#pragma unroll
  for (int q = 0; q < RPW; q++) cL[q] = cH[q] = 0u;

  for (int j0 = 0; j0 < nbr; j0 += 32) {
    const int j = j0 + lane;
    const bool vj = j < nbr;
    uint32_t W[RPW][4];
    float sc[RPW];
#pragma unroll
    for (int q = 0; q < RPW; q++) {
      uint2 v = make_uint2(0u, 0u);
      uint32_t E = 127u;
      if (vj && row_ok[q]) {
        v = lds_u2(st_base + ((uint32_t)row_id[q] * nbr + j) * 8u);
        E = lds_u8(sc_base + (uint32_t)row_id[q] * nbr + j);
      }
      Planes P;
      if (SEG32) {
        P = decode_block0(v.x, v.y);
      } else {
        uint32_t pL = __shfl_up_sync(kFull, v.x, 1), pH = __shfl_up_sync(kFull, v.y, 1);
        if (lane == 0) {
          pL = cL[q];
          pH = cH[q];
        }
        if (j % seg_blocks == 0) {
          pL = 0u;
          pH = 0u;
        }
        cL[q] = __shfl_sync(kFull, v.x, 31);
        cH[q] = __shfl_sync(kFull, v.y, 31);
        P = decode_block(v.x, v.y, pL, pH);
      }
      planes_to_nibbles_interleaved(P, W[q][0], W[q][1], W[q][2], W[q][3]);
      sc[q] = E5M3 ? e5m3_to_float(E) : ue8m0_to_float(E);
    }
    if (vj) {
      float bsum[RPW][TT];
#pragma unroll
      for (int q = 0; q < RPW; q++)
#pragma unroll
        for (int t = 0; t < TT; t++) bsum[q][t] = 0.f;
#pragma unroll
      for (int jj = 0; jj < 4; jj++) {
        uint32_t h[RPW][4];
#pragma unroll
        for (int q = 0; q < RPW; q++) e2m1x8_to_f16x2x4(W[q][jj], h[q][0], h[q][1], h[q][2], h[q][3]);
#pragma unroll
        for (int t = 0; t < TT; t++) {
          const uint32_t xa = xs_base + (uint32_t)(((t * nbr + j) * 16 + jj * 4) * 8);
          const float4 x01 = lds_f4(xa), x23 = lds_f4(xa + 16u);
          const float xv[8] = {x01.x, x01.y, x01.z, x01.w, x23.x, x23.y, x23.z, x23.w};
#pragma unroll
          for (int q = 0; q < RPW; q++) {
#pragma unroll
            for (int u = 0; u < 4; u++) {
              const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h[q][u]));
              bsum[q][t] = fmaf(f.x, xv[2 * u], bsum[q][t]);
              bsum[q][t] = fmaf(f.y, xv[2 * u + 1], bsum[q][t]);
            }
          }
        }
      }
#pragma unroll
      for (int q = 0; q < RPW; q++)
#pragma unroll
        for (int t = 0; t < TT; t++) acc[q][t] = fmaf(bsum[q][t], sc[q], acc[q][t]);
    }
  }
#pragma unroll
  for (int q = 0; q < RPW; q++)
#pragma unroll
    for (int t = 0; t < TT; t++) acc[q][t] = warp_sum(acc[q][t]);
}

// Pick acc[q][t] for t == lane (lanes >= TT get acc[q][0]).
template <int RPW, int TT>
__device__ __forceinline__ float lane_token(const float (&acc)[RPW][TT], int q) {
  const int lane = threadIdx.x & 31;
  float a = acc[q][0];
#pragma unroll
  for (int t = 1; t < TT; t++)
    if (lane == t) a = acc[q][t];
  return a;
}

}  // namespace tcf4
