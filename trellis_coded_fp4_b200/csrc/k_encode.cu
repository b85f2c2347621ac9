// k_encode.cu -- the upstream step: D-weighted Viterbi encoding of weights into a trellis stream.
//
// "XOR-Trellis: Hadamard-free FP4 LLM quantization" news page, bullet "Curvature-aware Viterbi
// objective": the stream of a segment is the path through the trellis that minimises the additive
// distortion sum_k D_k (w_k - w_hat_k)^2, with D the diagonal weighting and w_hat_k the decoded
// value (palette entry times the block's UE8M0 scale) of the state after symbol k. Offline work,
// compute-bound: per weight, every one of the 2^14 windows of the previous 7 symbols takes the
// cheapest of its 4 predecessors (the oldest symbol slides out) under each of the 4 new symbols.
//
// One segment per CTA (persistent over segments), 1024 threads:
//  * the 16384 path costs of the current step live in shared memory (fp64, 128 KB). Thread t owns
//    the predecessor groups g = t + 1024 i (i < 4): windows 4g..4g+3 feed the new windows
//    g + 4096 b (b = the new symbol), so each step is a butterfly: read 4 old costs, write 4 new;
//  * the E2M1 code of the full 16-bit state (window, new symbol) is fixed per window: each thread
//    derives its 64 codes once from the decoder (bit 7 of the planes of a block whose first eight
//    symbols are the state), and each step needs only the 16 distortions D_k (t_k - v_c s_k)^2, one
//    per E2M1 code c, computed for 256 steps at a time by all threads;
//  * the chosen predecessor of every new window (2 bits) goes to a per-CTA workspace in global
//    memory (4 KB per step); after the last step one thread walks the path back from the cheapest
//    final window (lowest index on ties) and writes the planar stream words.
// Every fp64 operation is written out (__dmul_rn, __dsub_rn, __dadd_rn), with no contraction, so
// costs, ties and hence symbols are exactly those of a plain IEEE evaluation of the objective in
// source order.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "tcf4_device.cuh"
#include "tcf4_internal.h"

namespace tcf4 {

constexpr int kEncThreads = 1024;
constexpr int kWindows = 1 << 14;
constexpr int kEncChunk = 256;  // steps whose 16 distortions are computed ahead, all at once
// shared memory: costs | distortions of a chunk [step][E2M1 code] | codes of every thread's groups |
// reduction scratch
constexpr size_t kEncSmem = sizeof(double) * kWindows + sizeof(double) * 16 * kEncChunk +
                            sizeof(uint64_t) * 4 * kEncThreads + 1024;

// E2M1 code of the state s (symbol m of the window at bits 2m, 2m+1; the newest at bits 14-15):
// weight 7 of a segment-start block whose first eight symbols are those of s.
__device__ __forceinline__ uint32_t state_code_dev(uint32_t s) {
  uint32_t L = 0u, H = 0u;
#pragma unroll
  for (int m = 0; m < 8; m++) {
    L |= ((s >> (2 * m)) & 1u) << m;
    H |= ((s >> (2 * m + 1)) & 1u) << m;
  }
  const Planes p = decode_block0(L, H);
  return ((p.n0 >> 7) & 1u) | (((p.n1 >> 7) & 1u) << 1) | (((p.n2 >> 7) & 1u) << 2) | (((p.n3 >> 7) & 1u) << 3);
}

// Exact value of an E2M1 code as fp64.
__device__ __forceinline__ double e2m1_f64(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  const double mag = e == 0u ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
  return (c & 8u) ? -mag : mag;
}

__global__ void __launch_bounds__(kEncThreads, 1)
    k_encode(const double *__restrict__ target, const double *__restrict__ Dw, const uint8_t *__restrict__ scales,
             int rows, int cols, int seg, uint32_t *__restrict__ out_stream, double *__restrict__ out_cost,
             uint32_t *__restrict__ back) {
  extern __shared__ __align__(16) unsigned char smem[];
  double *cost = reinterpret_cast<double *>(smem);
  double *dist = cost + kWindows;                                       // [kEncChunk][16]
  uint64_t *codes_s = reinterpret_cast<uint64_t *>(dist + 16 * kEncChunk);  // [4][1024]
  double *red_c = reinterpret_cast<double *>(codes_s + 4 * kEncThreads);  // 32 warp minima
  int *red_w = reinterpret_cast<int *>(red_c + 32);
  grid_dep_wait();  // the inputs may come from, and the outputs still be read by, preceding kernels
  // No early release: this kernel writes weights, which a following product kernel may read before
  // its own grid-dependency wait; its dependents start once it has exited.
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int segs_per_row = cols / seg, nseg = rows * segs_per_row, nbr = cols / 32;
  uint32_t *my_back = back + (size_t)blockIdx.x * seg * kEncThreads;

  // codes_s[i][t] holds the 16 codes (4 bits each, index 4 b + r) of group g = t + 1024 i; each
  // thread reads only its own (no barrier needed before the first use)
  for (int i = 0; i < 4; i++) {
    const uint32_t g = (uint32_t)t + 1024u * (uint32_t)i;
    uint64_t c = 0;
    for (uint32_t b = 0; b < 4; b++)
      for (uint32_t r = 0; r < 4; r++)
        c |= (uint64_t)state_code_dev(((g << 2) | r) | (b << 14)) << (4 * (4 * b + r));
    codes_s[i * kEncThreads + t] = c;
  }

  for (int sg = blockIdx.x; sg < nseg; sg += gridDim.x) {
    const int row = sg / segs_per_row, k0 = (sg - row * segs_per_row) * seg;
    for (int w = t; w < kWindows; w += kEncThreads) cost[w] = w == 0 ? 0.0 : INFINITY;
    for (int kc = 0; kc < seg; kc += kEncChunk) {
      const int n = seg - kc < kEncChunk ? seg - kc : kEncChunk;
      __syncthreads();  // the previous chunk's distortions are no longer read
      for (int j = t; j < 16 * n; j += kEncThreads) {
        const int kk = j >> 4, c = j & 15, k = k0 + kc + kk;
        const size_t at = (size_t)row * cols + k;
        const uint32_t E = scales[(size_t)row * nbr + k / 32];
        const double sc = E == 255u ? __longlong_as_double(0x7FF8000000000000ll) : ldexp(1.0, (int)E - 127);
        const double d = __dsub_rn(target[at], __dmul_rn(e2m1_f64((uint32_t)c), sc));
        dist[j] = __dmul_rn(__dmul_rn(Dw[at], d), d);
      }
      for (int kk = 0; kk < n; kk++) {
        const int k = k0 + kc + kk;
        const double *dk = dist + 16 * kk;
        __syncthreads();  // distortions ready; the previous step's costs written
        double oc[4][4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const double2 v0 = *reinterpret_cast<const double2 *>(cost + 4 * (t + 1024 * i));
          const double2 v1 = *reinterpret_cast<const double2 *>(cost + 4 * (t + 1024 * i) + 2);
          oc[i][0] = v0.x;
          oc[i][1] = v0.y;
          oc[i][2] = v1.x;
          oc[i][3] = v1.y;
        }
        __syncthreads();  // every old cost read
        uint32_t bp = 0;
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const uint32_t g = (uint32_t)t + 1024u * (uint32_t)i;
          const uint64_t codes = codes_s[i * kEncThreads + t];
#pragma unroll
          for (int b = 0; b < 4; b++) {
            double best = INFINITY;
            uint32_t br = 0;
#pragma unroll
            for (int r = 0; r < 4; r++) {  // predecessors in increasing order: the first minimum wins
              const double c = __dadd_rn(oc[i][r], dk[(codes >> (4 * (4 * b + r))) & 15u]);
              if (c < best) {
                best = c;
                br = (uint32_t)r;
              }
            }
            cost[g | ((uint32_t)b << 12)] = best;
            bp |= br << (2 * (4 * i + b));
          }
        }
        my_back[(size_t)(k - k0) * kEncThreads + t] = bp;
      }
    }
    __syncthreads();  // the last step's costs and back pointers are complete
    // cheapest final window, lowest index on ties
    double bc = INFINITY;
    int bw = kWindows;
    for (int w = t; w < kWindows; w += kEncThreads)
      if (cost[w] < bc) {
        bc = cost[w];
        bw = w;
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double oc2 = __shfl_xor_sync(0xffffffffu, bc, o);
      const int ow = __shfl_xor_sync(0xffffffffu, bw, o);
      if (oc2 < bc || (oc2 == bc && ow < bw)) {
        bc = oc2;
        bw = ow;
      }
    }
    if (lane == 0) {
      red_c[warp] = bc;
      red_w[warp] = bw;
    }
    __syncthreads();
    if (t == 0) {
      for (int w = 1; w < 32; w++)
        if (red_c[w] < bc || (red_c[w] == bc && red_w[w] < bw)) {
          bc = red_c[w];
          bw = red_w[w];
        }
      if (bw >= kWindows) bw = 0;  // every path infinite: the all-zero window
      if (out_cost != nullptr) out_cost[sg] = bc;
      // walk back: symbol k is the newest symbol of the window after step k
      uint32_t wn = (uint32_t)bw, lo = 0u, hi = 0u;
      for (int k = seg - 1; k >= 0; k--) {
        const uint32_t b = wn >> 12, g = wn & 0xFFFu;
        const int kg = k0 + k;
        lo |= (b & 1u) << (kg & 31);
        hi |= (b >> 1) << (kg & 31);
        if ((kg & 31) == 0) {  // a whole 32-symbol block: its planar words
          const size_t wi = ((size_t)row * nbr + kg / 32) * 2;
          out_stream[wi] = lo;
          out_stream[wi + 1] = hi;
          lo = hi = 0u;
        }
        const uint32_t bp = __ldcg(my_back + (size_t)k * kEncThreads + (g & 1023u));
        wn = (g << 2) | ((bp >> (2 * (4 * (g >> 10) + b))) & 3u);
      }
    }
    __syncthreads();  // the walk is done before the next segment reuses the back pointers
  }
}

static int encode_sm_count() {
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  return nsm;
}

// Back pointers of one CTA: 4 KB per step of a segment.
size_t encode_cta_bytes(int seg) { return (size_t)seg * kEncThreads * sizeof(uint32_t); }

// The workspace for one segment per SM (fewer bytes run fewer segments at a time).
size_t encode_workspace(int rows, int cols, int seg) {
  const int nseg = seg > 0 ? rows * (cols / seg) : 0, nsm = encode_sm_count();
  return (size_t)(nseg < nsm ? nseg : nsm) * encode_cta_bytes(seg);
}

cudaError_t launch_encode(const double *target, const double *D, const uint8_t *scales, int rows, int cols, int seg,
                          uint32_t *out_stream, double *out_cost, void *ws, size_t ws_bytes, cudaStream_t s) {
  const int nseg = rows * (cols / seg), nsm = encode_sm_count();
  const size_t fit = ws_bytes / encode_cta_bytes(seg);
  int grid = nseg < nsm ? nseg : nsm;
  if ((size_t)grid > fit) grid = (int)fit;
  if (grid < 1) return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k_encode, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kEncSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_dependent(k_encode, dim3(grid), dim3(kEncThreads), kEncSmem, s, target, D, scales, rows, cols, seg,
                          out_stream, out_cost, static_cast<uint32_t *>(ws));
}

}  // namespace tcf4
