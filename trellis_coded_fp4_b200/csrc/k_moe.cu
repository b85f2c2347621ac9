// k_moe.cu -- routed MoE layer on trellis-coded experts, decoded in-kernel.
//
// HEPH abstract, first serving mode applied to a "fused grouped-MoE" layer: for every token t and
// selected expert e: g,u = gate_up_e . x_t; h = bf16(silu(g) * u); y = down_e . h;
// out[t] = bf16(sum_j w[t][j] * y_j) with fp32 combine. Tokens routed to the same expert share one
// decode of that expert's rows.
//
// Launches (one stream, no host synchronisation, no device-wide barrier):
//   1. k_moe_plan      one CTA: per-expert token lists and the list of active experts;
//   2. k_moe_gateup    work items (active expert, 64 gate rows): gate and up rows decoded once
//                      for the expert's tokens, SwiGLU epilogue, h -> workspace (bf16);
//   3. k_moe_down      work items (active expert, 64 output rows): down rows against h -> y (fp32);
//   4. k_moe_combine   out[t][n] = bf16(sum_j w[t][j] * y[t*k+j][n]).
#include <cuda_bf16.h>

#include "tcf4_internal.h"
#include "tcf4_rowdot.cuh"

namespace tcf4 {

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

MoeWorkspace moe_workspace_layout(int E, int T, int k, int H, int I) {
  MoeWorkspace L;
  const size_t P = (size_t)T * k;
  size_t off = 0;
  L.counts = off;   off = align256(off + sizeof(int) * E);
  L.offsets = off;  off = align256(off + sizeof(int) * E);
  L.active = off;   off = align256(off + sizeof(int) * E);
  L.list = off;     off = align256(off + sizeof(int) * P);
  L.n_active = off; off = align256(off + sizeof(int));
  L.hidden = off;   off = align256(off + sizeof(uint16_t) * P * I);
  L.y = off;        off = align256(off + sizeof(float) * P * H);
  L.total = off;
  return L;
}

struct MoePlan {
  int *counts, *offsets, *active, *list, *n_active;
};

// Build per-expert token lists in (t, j) order. Pairs p = t*k + j with an expert id outside
// [0, E) are dropped. Deterministic: ranks are counted, not taken from atomics.
__global__ void __launch_bounds__(256) k_moe_plan(const int32_t *__restrict__ ids, int P, int E, MoePlan plan) {
  __shared__ int s_cnt[kMaxExperts];
  __shared__ int s_off[kMaxExperts];
  __shared__ int s_ids[kMaxTokens * kMaxTopK];
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) s_cnt[e] = 0;
  for (int p = tid; p < P; p += blockDim.x) s_ids[p] = ids[p];
  __syncthreads();
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = s_ids[p];
    if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int off = 0, na = 0;
    for (int e = 0; e < E; e++) {
      s_off[e] = off;
      off += s_cnt[e];
      if (s_cnt[e] > 0) plan.active[na++] = e;
    }
    *plan.n_active = na;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    plan.counts[e] = s_cnt[e];
    plan.offsets[e] = s_off[e];
  }
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = s_ids[p];
    if (e < 0 || e >= E) continue;
    int rank = 0;
    for (int q = 0; q < p; q++) rank += (s_ids[q] == e);
    plan.list[s_off[e] + rank] = p;
  }
}

constexpr int kRowsPerItem = 64;  // rows per work item: 8 warps x 8 rows

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

template <int TT>
__device__ __forceinline__ void stage_tokens_bf16(float2 *xs, const uint16_t *__restrict__ src, int K,
                                                  const int *rows, int nrow) {
  // rows[i] is the row of src ([*][K] bf16) that goes to token slot i; zeros beyond nrow
  const int nb = K >> 5, groups = K >> 3;
  for (int idx = threadIdx.x; idx < TT * groups; idx += blockDim.x) {
    const int t = idx / groups, gi = idx - t * groups;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (t < nrow) raw = __ldg(reinterpret_cast<const uint4 *>(src + (size_t)rows[t] * K) + gi);
    const int blk = gi >> 2, u = gi & 3;
    const uint32_t r[4] = {raw.x, raw.y, raw.z, raw.w};
    float2 *dst = xs + (size_t)t * nb * 16 + blk * 16 + u;
#pragma unroll
    for (int jj = 0; jj < 4; jj++) {
      const uint32_t lo = r[jj >> 1], hi = r[2 + (jj >> 1)];
      const float a = __uint_as_float((jj & 1) ? (lo & 0xFFFF0000u) : (lo << 16));
      const float b = __uint_as_float((jj & 1) ? (hi & 0xFFFF0000u) : (hi << 16));
      dst[jj * 4] = make_float2(a, b);
    }
  }
}

// gate_up + SwiGLU. xs holds TT tokens of H activations.
template <int MAXE, int TT, bool SEG32>
__global__ void __launch_bounds__(256) k_moe_gateup(const __grid_constant__ MoeTable<MAXE> tab, MoePlan plan, int H,
                                                    int I, int k, int gu_seg_blocks, const uint16_t *__restrict__ x,
                                                    uint16_t *__restrict__ hidden) {
  extern __shared__ float4 smem_f4[];
  float2 *xs = reinterpret_cast<float2 *>(smem_f4);
  __shared__ int s_tok[TT], s_pair[TT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbr = H >> 5;
  const int chunks = (I + kRowsPerItem - 1) / kRowsPerItem;
  const int items = *plan.n_active * chunks;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int a = item / chunks, c = item - a * chunks;
    const int e = plan.active[a];
    const int cnt = plan.counts[e], off = plan.offsets[e];
    const uint2 *st = tab.gu[e];
    const uint8_t *sc = tab.gus[e];
    for (int t0 = 0; t0 < cnt; t0 += TT) {
      const int ntok = min(TT, cnt - t0);
      __syncthreads();
      if (threadIdx.x < TT) {
        const int p = threadIdx.x < ntok ? plan.list[off + t0 + threadIdx.x] : 0;
        s_pair[threadIdx.x] = p;
        s_tok[threadIdx.x] = p / k;
      }
      __syncthreads();
      stage_tokens_bf16<TT>(xs, x, H, s_tok, ntok);
      __syncthreads();
      for (int rr = warp; rr < kRowsPerItem; rr += 8) {
        const int i = c * kRowsPerItem + rr;
        if (i >= I) break;
        float g[TT], u[TT];
        row_dot<TT, SEG32>(st + (size_t)i * nbr, sc + (size_t)i * nbr, nbr, gu_seg_blocks, xs, g);
        row_dot<TT, SEG32>(st + (size_t)(I + i) * nbr, sc + (size_t)(I + i) * nbr, nbr, gu_seg_blocks, xs, u);
        if (lane < ntok) {
          float gv = g[0], uv = u[0];
#pragma unroll
          for (int t = 1; t < TT; t++)
            if (lane == t) {
              gv = g[t];
              uv = u[t];
            }
          hidden[(size_t)s_pair[lane] * I + i] = __bfloat16_as_ushort(__float2bfloat16_rn(silu_f(gv) * uv));
        }
      }
    }
  }
}

// down: y[p][n] = down_e[n] . h[p] in fp32.
template <int MAXE, int TT, bool SEG32>
__global__ void __launch_bounds__(256) k_moe_down(const __grid_constant__ MoeTable<MAXE> tab, MoePlan plan, int H,
                                                  int I, int dn_seg_blocks, const uint16_t *__restrict__ hidden,
                                                  float *__restrict__ yws) {
  extern __shared__ float4 smem_f4[];
  float2 *xs = reinterpret_cast<float2 *>(smem_f4);
  __shared__ int s_pair[TT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbr = I >> 5;
  const int chunks = (H + kRowsPerItem - 1) / kRowsPerItem;
  const int items = *plan.n_active * chunks;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int a = item / chunks, c = item - a * chunks;
    const int e = plan.active[a];
    const int cnt = plan.counts[e], off = plan.offsets[e];
    const uint2 *st = tab.dn[e];
    const uint8_t *sc = tab.dns[e];
    for (int t0 = 0; t0 < cnt; t0 += TT) {
      const int ntok = min(TT, cnt - t0);
      __syncthreads();
      if (threadIdx.x < TT) s_pair[threadIdx.x] = threadIdx.x < ntok ? plan.list[off + t0 + threadIdx.x] : 0;
      __syncthreads();
      stage_tokens_bf16<TT>(xs, hidden, I, s_pair, ntok);
      __syncthreads();
      for (int rr = warp; rr < kRowsPerItem; rr += 8) {
        const int n = c * kRowsPerItem + rr;
        if (n >= H) break;
        float acc[TT];
        row_dot<TT, SEG32>(st + (size_t)n * nbr, sc + (size_t)n * nbr, nbr, dn_seg_blocks, xs, acc);
        if (lane < ntok) {
          float v = acc[0];
#pragma unroll
          for (int t = 1; t < TT; t++)
            if (lane == t) v = acc[t];
          yws[(size_t)s_pair[lane] * H + n] = v;
        }
      }
    }
  }
}

// out[t][n] = bf16(sum_j w[t][j] * y[t*k+j][n]); pairs with an invalid expert id contribute 0.
__global__ void __launch_bounds__(256) k_moe_combine(const float *__restrict__ yws, const int32_t *__restrict__ ids,
                                                     const float *__restrict__ wts, int T, int k, int H, int E,
                                                     uint16_t *__restrict__ out) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T * H) return;
  const int t = idx / H, n = idx - t * H;
  float acc = 0.f;
  for (int j = 0; j < k; j++) {
    const int e = ids[t * k + j];
    if (e < 0 || e >= E) continue;
    acc = fmaf(wts[t * k + j], yws[(size_t)(t * k + j) * H + n], acc);
  }
  out[idx] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
}

template <int MAXE, int TT, bool SEGGU, bool SEGDN>
static cudaError_t launch_moe_t(const tcf4_moe &m, int gu_seg, int dn_seg, const uint16_t *x, int T,
                                const int32_t *ids, const float *wts, int k, uint16_t *out, void *ws,
                                cudaStream_t s) {
  MoeTable<MAXE> tab;
  for (int e = 0; e < MAXE; e++) {
    const bool ok = e < m.E;
    tab.gu[e] = ok ? reinterpret_cast<const uint2 *>(m.gate_up[e].stream) : nullptr;
    tab.gus[e] = ok ? m.gate_up[e].scales : nullptr;
    tab.dn[e] = ok ? reinterpret_cast<const uint2 *>(m.down[e].stream) : nullptr;
    tab.dns[e] = ok ? m.down[e].scales : nullptr;
  }
  const MoeWorkspace L = moe_workspace_layout(m.E, T, k, m.H, m.I);
  char *base = static_cast<char *>(ws);
  MoePlan plan{reinterpret_cast<int *>(base + L.counts), reinterpret_cast<int *>(base + L.offsets),
               reinterpret_cast<int *>(base + L.active), reinterpret_cast<int *>(base + L.list),
               reinterpret_cast<int *>(base + L.n_active)};
  uint16_t *hidden = reinterpret_cast<uint16_t *>(base + L.hidden);
  float *yws = reinterpret_cast<float *>(base + L.y);

  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e1 = cudaFuncSetAttribute(k_moe_gateup<MAXE, TT, SEGGU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          227 * 1024);
    cudaError_t e2 = cudaFuncSetAttribute(k_moe_down<MAXE, TT, SEGDN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          227 * 1024);
    if (e1 != cudaSuccess) return e1;
    if (e2 != cudaSuccess) return e2;
    attr_set = true;
  }
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);

  k_moe_plan<<<1, 256, 0, s>>>(ids, T * k, m.E, plan);
  const size_t smem_gu = (size_t)TT * m.H * sizeof(float);
  const size_t smem_dn = (size_t)TT * m.I * sizeof(float);
  const int grid_gu = nsm * (smem_gu <= 56 * 1024 ? 4 : (smem_gu <= 110 * 1024 ? 2 : 1));
  const int grid_dn = nsm * (smem_dn <= 56 * 1024 ? 4 : (smem_dn <= 110 * 1024 ? 2 : 1));
  k_moe_gateup<MAXE, TT, SEGGU><<<grid_gu, 256, smem_gu, s>>>(tab, plan, m.H, m.I, k, gu_seg, x, hidden);
  k_moe_down<MAXE, TT, SEGDN><<<grid_dn, 256, smem_dn, s>>>(tab, plan, m.H, m.I, dn_seg, hidden, yws);
  k_moe_combine<<<(T * m.H + 255) / 256, 256, 0, s>>>(yws, ids, wts, T, k, m.H, m.E, out);
  return cudaGetLastError();
}

template <int MAXE, int TT>
static cudaError_t launch_moe_segs(const tcf4_moe &m, int gu_seg, int dn_seg, const uint16_t *x, int T,
                                   const int32_t *ids, const float *wts, int k, uint16_t *out, void *ws,
                                   cudaStream_t s) {
  const bool a = gu_seg == 1, b = dn_seg == 1;
  if (a && b) return launch_moe_t<MAXE, TT, true, true>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
  if (a) return launch_moe_t<MAXE, TT, true, false>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
  if (b) return launch_moe_t<MAXE, TT, false, true>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
  return launch_moe_t<MAXE, TT, false, false>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
}

cudaError_t launch_moe(const tcf4_moe &m, int gu_seg, int dn_seg, const uint16_t *x, int T, const int32_t *ids,
                       const float *wts, int k, uint16_t *out, void *ws, cudaStream_t s) {
  // tokens per decode pass: as many as fit (4 max) in shared memory for the longer K
  const int K = m.H > m.I ? m.H : m.I;
  int TT = 4;
  while (TT > 1 && (size_t)TT * K * sizeof(float) > 200 * 1024) TT >>= 1;
  if (T == 1) TT = 1;
  if (m.E <= 32) {
    if (TT == 1) return launch_moe_segs<32, 1>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
    if (TT == 2) return launch_moe_segs<32, 2>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
    return launch_moe_segs<32, 4>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
  }
  if (TT == 1) return launch_moe_segs<256, 1>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
  if (TT == 2) return launch_moe_segs<256, 2>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
  return launch_moe_segs<256, 4>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
}

}  // namespace tcf4
