// k_gemv.cu -- fused trellis decode + GEMV / small-batch product on CUDA cores.
//
// y[t][n] = bf16( sum_k w[n][k] x[t][k] ), w decoded in registers from the resident stream
// (HEPH abstract, first serving mode). Bound by HBM in principle: 0.28125 B/weight of stream and
// scales. Each persistent CTA owns the row slabs s = blockIdx.x + j * gridDim.x (R rows each); one
// thread keeps NS slabs in flight with cp.async.bulk into a shared-memory ring while 8 warps decode
// and multiply the slab at the head of the ring (RPW = R/8 rows per warp, activations reused across
// them). The activations for TT tokens are staged once per pass in shared memory.
#include <cuda_bf16.h>

#include "tcf4_internal.h"
#include "tcf4_rowdot.cuh"

namespace tcf4 {

__device__ unsigned int g_tcf4_timeouts_gemv = 0;

constexpr int kNS = 4;  // slabs in flight per CTA

struct GemvGeom {
  uint32_t xs_bytes, sc_off, stride, smem;
};

__host__ __device__ inline GemvGeom gemv_geom(int nbr, int TT, int R) {
  GemvGeom g;
  g.xs_bytes = round_up((uint32_t)TT * nbr * 32u * 4u, 128u);
  g.sc_off = round_up((uint32_t)R * nbr * 8u, 16u);
  g.stride = round_up(g.sc_off + (uint32_t)R * nbr, 128u);
  g.smem = 128u + g.xs_bytes + kNS * g.stride;
  return g;
}

template <int TT, bool SEG32, int R, bool E5M3>
__global__ void __launch_bounds__(256) k_gemv(MatView w, const uint16_t *__restrict__ x, int T,
                                              uint16_t *__restrict__ y, int bulk_scales) {
  extern __shared__ __align__(128) unsigned char smem[];
  grid_dep_wait();  // x may come from, and y may still be read by, the preceding kernel
  grid_dep_release();
  constexpr int RPW = R / 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbr = w.nbr, K = nbr * 32;
  const GemvGeom geo = gemv_geom(nbr, TT, R);
  SlabRing<kNS> ring;
  ring.full = reinterpret_cast<uint64_t *>(smem);
  ring.buf = smem + 128 + geo.xs_bytes;
  ring.stride = geo.stride;
  ring.sc_off = geo.sc_off;
  ring.st_row = (uint32_t)nbr * 8u;
  ring.sc_row = (uint32_t)nbr;
  ring.bulk_scales = bulk_scales;
  ring.phase_bits = 0u;
  ring.timeouts = &g_tcf4_timeouts_gemv;
  float2 *xs = reinterpret_cast<float2 *>(smem + 128);
  if (tid == 0) {
    for (int b = 0; b < kNS; b++) mbar_init(&ring.full[b], 1);
    mbar_fence_init();
  }
  __syncthreads();

  const int nslab = (w.rows + R - 1) / R;
  const int my_n = (int)blockIdx.x < nslab ? (nslab - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto slab = [&](int j) {
    const int r0 = ((int)blockIdx.x + j * (int)gridDim.x) * R;
    Slab s;
    s.st = reinterpret_cast<const unsigned char *>(w.stream + (size_t)r0 * nbr);
    s.sc = w.scales + (size_t)r0 * nbr;
    s.nrows = (uint32_t)min(R, w.rows - r0);
    return s;
  };

  for (int t0 = 0; t0 < T; t0 += TT) {
    const int ntok = min(TT, T - t0);
    if (tid == 0)
      for (int j = 0; j < kNS && j < my_n; j++) ring.issue(j, slab(j));
    int tok[TT];
#pragma unroll
    for (int t = 0; t < TT; t++) tok[t] = t0 + t;
    stage_x<TT>(xs, x, K, tok, ntok);
    __syncthreads();
    for (int j = 0; j < my_n; j++) {
      const int b = j % kNS;
      const Slab s = slab(j);
      if (ring.acquire(b, s)) {
        const uint32_t st_base = smem_u32(ring.buf + (size_t)b * ring.stride);
        int rid[RPW];
        bool rok[RPW];
#pragma unroll
        for (int q = 0; q < RPW; q++) {
          rid[q] = warp + 8 * q;
          rok[q] = rid[q] < (int)s.nrows;
        }
        float acc[RPW][TT];
        rows_dot_smem<RPW, TT, SEG32, E5M3>(st_base, st_base + ring.sc_off, nbr, w.seg_blocks, rid, rok, smem_u32(xs),
                                      acc);
        const int r0 = ((int)blockIdx.x + j * (int)gridDim.x) * R;
#pragma unroll
        for (int q = 0; q < RPW; q++) {
          const float a = lane_token<RPW, TT>(acc, q);
          if (rok[q] && lane < ntok)
            y[(size_t)(t0 + lane) * w.rows + r0 + rid[q]] = __bfloat16_as_ushort(__float2bfloat16_rn(a));
        }
      }
      __syncthreads();
      if (tid == 0 && j + kNS < my_n) ring.issue(b, slab(j + kNS));
    }
  }
}

template <int TT, bool SEG32, int R, bool E5M3>
static cudaError_t launch_gemv_t(const MatView &w, const uint16_t *x, int T, uint16_t *y, cudaStream_t s) {
  const GemvGeom geo = gemv_geom(w.nbr, TT, R);
  static unsigned long long attr_done = 0;  // benign race: setting the same attribute twice is harmless
  cudaError_t e = ensure_max_dynamic_smem(k_gemv<TT, SEG32, R, E5M3>, attr_done);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 148, occ = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_gemv<TT, SEG32, R, E5M3>, 256, geo.smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  const int nslab = (w.rows + R - 1) / R;
  const int grid = nslab < nsm * occ ? nslab : nsm * occ;
  const int bulk_scales = ((reinterpret_cast<uintptr_t>(w.scales) & 15u) == 0 && (R * w.nbr) % 16 == 0) ? 1 : 0;
  return launch_dependent(k_gemv<TT, SEG32, R, E5M3>, dim3(grid), dim3(256), geo.smem, s, w, x, T, y, bulk_scales);
}

template <int TT, bool SEG32, bool E5M3>
static cudaError_t launch_gemv_r(const MatView &w, const uint16_t *x, int T, uint16_t *y, cudaStream_t s) {
  // 16 rows per slab while a slab stays within ~36 KB, else 8
  if ((size_t)16 * w.nbr * 9 <= 36 * 1024) return launch_gemv_t<TT, SEG32, 16, E5M3>(w, x, T, y, s);
  return launch_gemv_t<TT, SEG32, 8, E5M3>(w, x, T, y, s);
}

template <bool E5M3>
static cudaError_t launch_gemv_f(const MatView &w, const uint16_t *x, int T, uint16_t *y, cudaStream_t s) {
  const int K = w.nbr * 32;
  int TT = T >= 3 ? 4 : T;
  // activations of TT tokens plus 4 slab buffers must fit in shared memory
  while (TT > 1 && gemv_geom(w.nbr, TT, 16 * w.nbr * 9 <= 36 * 1024 ? 16 : 8).smem > 220u * 1024u) TT >>= 1;
  (void)K;
  const bool seg32 = w.seg_blocks == 1;
  switch (TT) {
    case 1: return seg32 ? launch_gemv_r<1, true, E5M3>(w, x, T, y, s) : launch_gemv_r<1, false, E5M3>(w, x, T, y, s);
    case 2: return seg32 ? launch_gemv_r<2, true, E5M3>(w, x, T, y, s) : launch_gemv_r<2, false, E5M3>(w, x, T, y, s);
    default: return seg32 ? launch_gemv_r<4, true, E5M3>(w, x, T, y, s) : launch_gemv_r<4, false, E5M3>(w, x, T, y, s);
  }
}

cudaError_t launch_gemv(const MatView &w, const uint16_t *x, int T, uint16_t *y, cudaStream_t s, bool e5m3) {
  return e5m3 ? launch_gemv_f<true>(w, x, T, y, s) : launch_gemv_f<false>(w, x, T, y, s);
}

unsigned int take_timeouts_gemv() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_tcf4_timeouts_gemv, sizeof v) != cudaSuccess) return 0;
  cudaMemcpyToSymbol(g_tcf4_timeouts_gemv, &zero, sizeof zero);
  return v;
}

}  // namespace tcf4
