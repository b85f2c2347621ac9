// k_expand.cu -- HEPH's second serving mode: expand a trellis stream into packed MXFP4.
//
// "HEPH: 3-Bit Grid-Aligned Trellis Quantization of MXFP4 Mixture-of-Experts ..." (abstract):
// the ~3-bpw stream can be expanded into a resident 4.25-bpw MXFP4 tensor. Each decoded weight is
// already an E2M1 code under its block's UE8M0 scale, so expansion = decode + nibble packing, and
// the scales are copied unchanged.
//
// HBM-bound streaming kernel: per 32-weight block it reads 8 bytes of stream and writes 16 bytes
// of nibbles (plus one scale byte read and written): 0.8125 B/weight. When the stream and the
// output are 32-byte aligned a thread takes four consecutive blocks (one 32-byte load, two 32-byte
// stores); otherwise pairs of blocks (one 16-byte load, two 16-byte stores). Accesses are
// coalesced across the warp.
#include "tcf4_device.cuh"
#include "tcf4_internal.h"

namespace tcf4 {

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream(uint4 *p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// One 32-byte non-allocating load (four blocks of words; p 32-byte aligned).
__device__ __forceinline__ void ld_stream2(const uint4 *p, uint4 &a, uint4 &b) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
               : "l"(p));
}

// One 32-byte streaming store (both blocks of a pair; p 32-byte aligned).
__device__ __forceinline__ void st_stream2(uint4 *p, uint4 a, uint4 b) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w),
               "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

// SEG32: every block starts a segment (state 0), so no carry between blocks. PT: pairs per thread;
// a CTA covers 256 * PT consecutive pairs, thread t the pairs t, t + 256, ... of them (each round
// coalesced across the warp), and issues all its PT loads before it decodes, so that enough bytes
// are in flight per SM to cover the memory latency.
// V8: the output is 32-byte aligned, so a pair's two blocks go out as one 32-byte store.
template <bool SEG32, int PT, bool V8>
__global__ void __launch_bounds__(256) k_expand(const uint2 *__restrict__ stream, uint32_t nblocks,
                                                uint32_t blocks_per_row, uint32_t seg_blocks,
                                                uint4 *__restrict__ out, const uint8_t *__restrict__ scales,
                                                uint8_t *__restrict__ out_scales, int scales_aligned16) {
  grid_dep_wait();  // out may still be read by the preceding kernel
  // No early release: this kernel writes weights, which a following product kernel may read before
  // its own grid-dependency wait; its dependents start once it has exited.
  const uint32_t npairs = (nblocks + 1u) >> 1;
  const uint32_t base = blockIdx.x * (256u * PT) + threadIdx.x;
  uint4 v[PT];
#pragma unroll
  for (int j = 0; j < PT; j++) {
    const uint32_t pair = base + 256u * (uint32_t)j, g0 = 2u * pair;
    v[j] = make_uint4(0u, 0u, 0u, 0u);
    if (pair < npairs) {
      if (g0 + 1u < nblocks) {
        v[j] = ld_stream(reinterpret_cast<const uint4 *>(stream + g0));
      } else {
        const uint2 t = stream[g0];
        v[j].x = t.x;
        v[j].y = t.y;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < PT; j++) {
    const uint32_t pair = base + 256u * (uint32_t)j, g0 = 2u * pair;
    const bool valid = pair < npairs, has2 = g0 + 1u < nblocks;
    uint4 o;
    if (SEG32) {
      if (valid) {
        planes_to_nibbles_natural(decode_block0(v[j].x, v[j].y), o.x, o.y, o.z, o.w);
        if (V8 && has2) {
          uint4 o2;
          planes_to_nibbles_natural(decode_block0(v[j].z, v[j].w), o2.x, o2.y, o2.z, o2.w);
          st_stream2(out + g0, o, o2);
        } else {
          st_stream(out + g0, o);
          if (has2) {
            planes_to_nibbles_natural(decode_block0(v[j].z, v[j].w), o.x, o.y, o.z, o.w);
            st_stream(out + g0 + 1u, o);
          }
        }
      }
    } else {
      uint32_t pL0 = 0u, pH0 = 0u, pL1 = 0u, pH1 = 0u;  // carries into blocks g0 and g0+1
      // The predecessor of block g0 is the previous thread's second block (the previous lane's, or
      // for lane 0 the one before in memory).
      uint32_t uL = __shfl_up_sync(0xffffffffu, v[j].z, 1), uH = __shfl_up_sync(0xffffffffu, v[j].w, 1);
      if (valid && (g0 % blocks_per_row) % seg_blocks != 0u) {
        if ((threadIdx.x & 31u) == 0u) {
          const uint2 t = stream[g0 - 1u];
          uL = t.x;
          uH = t.y;
        }
        pL0 = uL;
        pH0 = uH;
      }
      if (has2 && ((g0 + 1u) % blocks_per_row) % seg_blocks != 0u) {
        pL1 = v[j].x;
        pH1 = v[j].y;
      }
      if (valid) {
        planes_to_nibbles_natural(decode_block(v[j].x, v[j].y, pL0, pH0), o.x, o.y, o.z, o.w);
        st_stream(out + g0, o);
        if (has2) {
          planes_to_nibbles_natural(decode_block(v[j].z, v[j].w, pL1, pH1), o.x, o.y, o.z, o.w);
          st_stream(out + g0 + 1u, o);
        }
      }
    }
  }

  // Scale bytes are copied verbatim (grid-stride): 16-byte chunks when both pointers allow, then the
  // tail byte by byte.
  const uint32_t tg = blockIdx.x * 256u + threadIdx.x, nth = gridDim.x * 256u;
  const uint32_t nchunk = scales_aligned16 ? nblocks >> 4 : 0u;
  for (uint32_t c = tg; c < nchunk; c += nth)
    reinterpret_cast<uint4 *>(out_scales)[c] = reinterpret_cast<const uint4 *>(scales)[c];
  for (uint32_t b = (nchunk << 4) + tg; b < nblocks; b += nth) out_scales[b] = scales[b];
}

// Pairs of blocks per thread. One: more CTAs in flight beat more loads per thread (measured on the
// 184320 x 2880 gate_up matrix: 77.3 us with one pair, 77.5 with two, 82.5 with four).
constexpr int kExpandPairs = 1;

// Segments of one block with 32-byte aligned stream and output: a thread takes four consecutive
// blocks, one 32-byte load and two 32-byte stores (the last partial quad block by block).
__global__ void __launch_bounds__(256) k_expand_q(const uint2 *__restrict__ stream, uint32_t nblocks,
                                                  uint4 *__restrict__ out, const uint8_t *__restrict__ scales,
                                                  uint8_t *__restrict__ out_scales, int scales_aligned16) {
  grid_dep_wait();  // out may still be read by the preceding kernel
  // No early release: this kernel writes weights, which a following product kernel may read before
  // its own grid-dependency wait; its dependents start once it has exited.
  const uint32_t g0 = 4u * (blockIdx.x * 256u + threadIdx.x);
  if (g0 + 3u < nblocks) {
    uint4 a, b, o0, o1;
    ld_stream2(reinterpret_cast<const uint4 *>(stream + g0), a, b);
    planes_to_nibbles_natural(decode_block0(a.x, a.y), o0.x, o0.y, o0.z, o0.w);
    planes_to_nibbles_natural(decode_block0(a.z, a.w), o1.x, o1.y, o1.z, o1.w);
    st_stream2(out + g0, o0, o1);
    planes_to_nibbles_natural(decode_block0(b.x, b.y), o0.x, o0.y, o0.z, o0.w);
    planes_to_nibbles_natural(decode_block0(b.z, b.w), o1.x, o1.y, o1.z, o1.w);
    st_stream2(out + g0 + 2u, o0, o1);
  } else {
    for (uint32_t g = g0; g < nblocks; g++) {
      const uint2 t = stream[g];
      uint4 o;
      planes_to_nibbles_natural(decode_block0(t.x, t.y), o.x, o.y, o.z, o.w);
      st_stream(out + g, o);
    }
  }
  const uint32_t tg = blockIdx.x * 256u + threadIdx.x, nth = gridDim.x * 256u;
  const uint32_t nchunk = scales_aligned16 ? nblocks >> 4 : 0u;
  for (uint32_t c = tg; c < nchunk; c += nth)
    reinterpret_cast<uint4 *>(out_scales)[c] = reinterpret_cast<const uint4 *>(scales)[c];
  for (uint32_t b = (nchunk << 4) + tg; b < nblocks; b += nth) out_scales[b] = scales[b];
}

cudaError_t launch_expand(const MatView &w, uint8_t *out_nibbles, uint8_t *out_scales, cudaStream_t s) {
  const uint32_t nblocks = (uint32_t)((int64_t)w.rows * w.nbr);
  const bool aligned = ((reinterpret_cast<uintptr_t>(w.scales) | reinterpret_cast<uintptr_t>(out_scales)) & 15u) == 0;
  const uint32_t npairs = (nblocks + 1u) / 2u;
  const uint32_t grid = (npairs + 256u * kExpandPairs - 1u) / (256u * kExpandPairs);
  auto *out = reinterpret_cast<uint4 *>(out_nibbles);
  const bool out32 = (reinterpret_cast<uintptr_t>(out_nibbles) & 31u) == 0;
  if (w.seg_blocks == 1 && out32 && (reinterpret_cast<uintptr_t>(w.stream) & 31u) == 0)
    return launch_dependent(k_expand_q, dim3((nblocks + 1023u) / 1024u), dim3(256), 0, s, w.stream, nblocks, out,
                            w.scales, out_scales, aligned ? 1 : 0);
  if (w.seg_blocks == 1) {
    return out32 ? launch_dependent(k_expand<true, kExpandPairs, true>, dim3(grid), dim3(256), 0, s, w.stream, nblocks,
                                    (uint32_t)w.nbr, 1u, out, w.scales, out_scales, aligned ? 1 : 0)
                 : launch_dependent(k_expand<true, kExpandPairs, false>, dim3(grid), dim3(256), 0, s, w.stream, nblocks,
                                    (uint32_t)w.nbr, 1u, out, w.scales, out_scales, aligned ? 1 : 0);
  } else {
    return launch_dependent(k_expand<false, kExpandPairs, false>, dim3(grid), dim3(256), 0, s, w.stream, nblocks,
                            (uint32_t)w.nbr, (uint32_t)w.seg_blocks, out, w.scales, out_scales, aligned ? 1 : 0);
  }
}

}  // namespace tcf4
