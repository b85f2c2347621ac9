// k_repack.cu -- interleaved stream packing -> the planar words the decoders read.
//
// The XOR-Trellis news page ("XOR-Trellis FP4 decoder" bullet) keys each weight on a 16-bit sliding
// state. A stream may be stored as one bit string per row with two bits per symbol (low bit first,
// LSB-first in 32-bit words), where that state is a window of the string; the decoders here take
// the planar form instead (per 32-weight block, one word of the symbols' low bits and one of their
// high bits), which makes the state's delays whole-word shifts. The two packings are the same
// trellis under a fixed bit permutation, applied by this kernel once, at load time.
//
// HBM-bound streaming kernel: 8 bytes read and 8 written per 32-weight block (0.5 B/weight). A block
// is two words of 16 symbols each; each word is unshuffled (even bits to its low half, odd bits to its
// high half: four delta swaps) and the halves are recombined with two byte permutes. A thread takes
// four blocks (one 32-byte load and store) when both buffers are 32-byte aligned, two when they are
// 16-byte aligned, else one; two such units per thread, both loads issued before either store.
// In place (in == out) is allowed: every thread reads its own blocks before it writes them.
#include "tcf4_internal.h"

namespace tcf4 {

// Even bits of x to bits 0..15, odd bits to bits 16..31.
__device__ __forceinline__ uint32_t unzip_bits(uint32_t x) {
  uint32_t t;
  t = (x ^ (x >> 1)) & 0x22222222u;
  x ^= t ^ (t << 1);
  t = (x ^ (x >> 2)) & 0x0C0C0C0Cu;
  x ^= t ^ (t << 2);
  t = (x ^ (x >> 4)) & 0x00F000F0u;
  x ^= t ^ (t << 4);
  t = (x ^ (x >> 8)) & 0x0000FF00u;
  x ^= t ^ (t << 8);
  return x;
}

// One block: (symbols 0..15, symbols 16..31) interleaved -> (low plane, high plane).
__device__ __forceinline__ uint2 repack_block(uint32_t w0, uint32_t w1) {
  const uint32_t u0 = unzip_bits(w0), u1 = unzip_bits(w1);
  return make_uint2(__byte_perm(u0, u1, 0x5410), __byte_perm(u0, u1, 0x7632));
}

// Coherent loads (the buffer may be the output too) that do not allocate in L1.
__device__ __forceinline__ void ld_unit(const uint2 *p, uint2 (&v)[1]) {
  asm volatile("ld.global.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v[0].x), "=r"(v[0].y) : "l"(p));
}
__device__ __forceinline__ void ld_unit(const uint2 *p, uint2 (&v)[2]) {
  asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v[0].x), "=r"(v[0].y), "=r"(v[1].x), "=r"(v[1].y)
               : "l"(p));
}
__device__ __forceinline__ void ld_unit(const uint2 *p, uint2 (&v)[4]) {
  asm volatile("ld.global.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v[0].x), "=r"(v[0].y), "=r"(v[1].x), "=r"(v[1].y), "=r"(v[2].x), "=r"(v[2].y), "=r"(v[3].x),
                 "=r"(v[3].y)
               : "l"(p));
}
__device__ __forceinline__ void st_unit(uint2 *p, const uint2 (&v)[1]) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v[0].x), "r"(v[0].y) : "memory");
}
__device__ __forceinline__ void st_unit(uint2 *p, const uint2 (&v)[2]) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v[0].x), "r"(v[0].y), "r"(v[1].x),
               "r"(v[1].y)
               : "memory");
}
__device__ __forceinline__ void st_unit(uint2 *p, const uint2 (&v)[4]) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v[0].x), "r"(v[0].y),
               "r"(v[1].x), "r"(v[1].y), "r"(v[2].x), "r"(v[2].y), "r"(v[3].x), "r"(v[3].y)
               : "memory");
}

constexpr int kRepackThreads = 256, kRepackUnits = 2;

// BPU blocks per access unit (4, 2 or 1). Units u and u + 256 of a CTA's 512 go to thread u; the
// last nblocks % BPU blocks go one per thread to the first threads of the last CTA.
template <int BPU>
__global__ void __launch_bounds__(kRepackThreads) k_repack(const uint2 *in, uint2 *out, uint32_t nblocks) {
  grid_dep_wait();  // the input may come from, and the output still be read by, preceding kernels
  // No early release: this kernel writes weights, which a following product kernel may read before
  // its own grid-dependency wait; its dependents start once it has exited.
  const uint32_t nunits = nblocks / BPU;
  const uint32_t u0 = blockIdx.x * (kRepackThreads * kRepackUnits) + threadIdx.x;
  uint2 v[kRepackUnits][BPU];
#pragma unroll
  for (int j = 0; j < kRepackUnits; j++) {
    const uint32_t u = u0 + kRepackThreads * j;
    if (u < nunits) ld_unit(in + (size_t)u * BPU, v[j]);
  }
#pragma unroll
  for (int j = 0; j < kRepackUnits; j++) {
    const uint32_t u = u0 + kRepackThreads * j;
    if (u < nunits) {
#pragma unroll
      for (int i = 0; i < BPU; i++) v[j][i] = repack_block(v[j][i].x, v[j][i].y);
      st_unit(out + (size_t)u * BPU, v[j]);
    }
  }
  if (BPU > 1 && blockIdx.x == gridDim.x - 1 && threadIdx.x < nblocks - nunits * BPU) {
    const uint32_t g = nunits * BPU + threadIdx.x;
    const uint2 w = in[g];
    out[g] = repack_block(w.x, w.y);
  }
}

template <int BPU>
static cudaError_t launch_repack_t(const uint2 *in, uint2 *out, uint32_t nblocks, cudaStream_t s) {
  const uint32_t nunits = nblocks / BPU, per_cta = kRepackThreads * kRepackUnits;
  const uint32_t grid = nunits > 0 ? (nunits + per_cta - 1) / per_cta : 1u;
  return launch_dependent(k_repack<BPU>, dim3(grid), dim3(kRepackThreads), 0, s, in, out, nblocks);
}

cudaError_t launch_repack(const uint32_t *in, uint32_t *out, uint32_t nblocks, cudaStream_t s) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out);
  const uint2 *i2 = reinterpret_cast<const uint2 *>(in);
  uint2 *o2 = reinterpret_cast<uint2 *>(out);
  if ((a & 31u) == 0) return launch_repack_t<4>(i2, o2, nblocks, s);
  if ((a & 15u) == 0) return launch_repack_t<2>(i2, o2, nblocks, s);
  return launch_repack_t<1>(i2, o2, nblocks, s);
}

}  // namespace tcf4
