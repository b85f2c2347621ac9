// k_moe.cu -- routed MoE layer on trellis-coded experts, decoded in-kernel.
//
// HEPH abstract, first serving mode applied to a "fused grouped-MoE" layer: for every token t and
// selected expert e: g,u = gate_up_e . x_t; h = bf16(silu(g) * u); y = down_e . h;
// out[t] = bf16(sum_j w[t][j] * y_j) with fp32 combine. Tokens routed to the same expert share one
// decode of that expert's rows.
//
// Two launches on one stream, no host synchronisation, no grid-wide barrier:
//   k_moe_gateup  every CTA builds the routing plan (per-expert token lists, active experts) in
//                 shared memory from topk_ids; work items are (active expert, R gate rows), taken in
//                 contiguous ranges per CTA so a CTA restages activations only when the expert
//                 changes; each item's R gate rows and R up rows arrive as one double slab through
//                 the bulk-copy ring; SwiGLU epilogue writes h (bf16) to the workspace.
//   k_moe_down    same plan; work items (active expert, R output rows); y (fp32) per (t, j) goes to
//                 the workspace; the last item to finish a row chunk (counted with an atomic after a
//                 fence) combines out[t][n] = bf16(sum_j w[t][j] y[t*k+j][n]) in fixed j order.
#include <cuda_bf16.h>

#include "tcf4_internal.h"
#include "tcf4_rowdot.cuh"

namespace tcf4 {

__device__ unsigned int g_tcf4_timeouts_moe = 0;

constexpr int kMoeNS = 4;     // slabs in flight per CTA
constexpr int kMoeRMin = 8;   // fewest rows per work item (sizes the counter array)

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

MoeWorkspace moe_workspace_layout(int E, int T, int k, int H, int I) {
  (void)E;
  MoeWorkspace L;
  const size_t P = (size_t)T * k;
  size_t off = 0;
  L.counters = off; off = align256(off + sizeof(int) * ((H + kMoeRMin - 1) / kMoeRMin));
  L.hidden = off;   off = align256(off + sizeof(uint16_t) * P * I);
  L.y = off;        off = align256(off + sizeof(float) * P * H);
  L.total = off;
  return L;
}

// Routing plan in shared memory: per expert the pairs p = t*k + j routed to it, in p order.
struct PlanSmem {
  int cnt[kMaxExperts];
  int off[kMaxExperts];
  int act[kMaxExperts];
  int list[kMaxTokens * kMaxTopK];
  int ids[kMaxTokens * kMaxTopK];
  int n_active;
};

// All threads of the CTA. Pairs whose expert id is outside [0, E) are dropped. Deterministic.
__device__ void build_plan(PlanSmem &pl, const int32_t *__restrict__ ids, int P, int E) {
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) pl.cnt[e] = 0;
  for (int p = tid; p < P; p += blockDim.x) pl.ids[p] = ids[p];
  __syncthreads();
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = pl.ids[p];
    if (e >= 0 && e < E) atomicAdd(&pl.cnt[e], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int o = 0, na = 0;
    for (int e = 0; e < E; e++) {
      pl.off[e] = o;
      o += pl.cnt[e];
      if (pl.cnt[e] > 0) pl.act[na++] = e;
    }
    pl.n_active = na;
  }
  __syncthreads();
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = pl.ids[p];
    if (e < 0 || e >= E) continue;
    int rank = 0;
    for (int q = 0; q < p; q++) rank += (pl.ids[q] == e);
    pl.list[pl.off[e] + rank] = p;
  }
  __syncthreads();
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

struct MoeGeom {
  uint32_t xs_bytes, sc_off, stride, smem;
};

// Buffer of one item: `parts` row groups of R rows (stream words), then their scales.
__host__ __device__ inline MoeGeom moe_geom(int nbr, int TT, int parts, int R) {
  MoeGeom g;
  g.xs_bytes = round_up((uint32_t)TT * nbr * 32u * 4u, 128u);
  g.sc_off = round_up((uint32_t)(parts * R) * nbr * 8u, 16u);
  g.stride = round_up(g.sc_off + (uint32_t)(parts * R) * nbr, 128u);
  g.smem = 128u + (uint32_t)round_up(sizeof(PlanSmem), 128u) + g.xs_bytes + kMoeNS * g.stride;
  return g;
}

// Contiguous range of work items for this CTA.
__device__ __forceinline__ void item_range(int items, int &beg, int &end) {
  beg = (int)(((long long)items * blockIdx.x) / gridDim.x);
  end = (int)(((long long)items * (blockIdx.x + 1)) / gridDim.x);
}

template <int MAXE, int TT, bool SEG32, int R>
__global__ void __launch_bounds__(256) k_moe_gateup(const __grid_constant__ MoeTable<MAXE> tab,
                                                    const int32_t *__restrict__ ids, int P, int E, int k, int H, int I,
                                                    int seg_blocks, const uint16_t *__restrict__ x,
                                                    uint16_t *__restrict__ hidden, int *__restrict__ counters,
                                                    int n_counters, int bulk_scales) {
  extern __shared__ __align__(128) unsigned char smem[];
  grid_dep_wait();  // inputs and workspace come from, or are still read by, the preceding kernel
  grid_dep_release();
  constexpr int RPW = R / 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbr = H >> 5;
  const MoeGeom geo = moe_geom(nbr, TT, 2, R);
  PlanSmem &pl = *reinterpret_cast<PlanSmem *>(smem + 128);
  float2 *xs = reinterpret_cast<float2 *>(smem + 128 + round_up(sizeof(PlanSmem), 128u));
  SlabRing<kMoeNS> ring;
  ring.full = reinterpret_cast<uint64_t *>(smem);
  ring.buf = reinterpret_cast<unsigned char *>(xs) + geo.xs_bytes;
  ring.stride = geo.stride;
  ring.sc_off = geo.sc_off;
  ring.st_row = (uint32_t)nbr * 8u;
  ring.sc_row = (uint32_t)nbr;
  ring.bulk_scales = bulk_scales;
  ring.phase_bits = 0u;
  ring.timeouts = &g_tcf4_timeouts_moe;
  if (tid == 0) {
    for (int b = 0; b < kMoeNS; b++) mbar_init(&ring.full[b], 1);
    mbar_fence_init();
  }
  if (blockIdx.x == 0)  // the down kernel's chunk counters start at zero
    for (int c = tid; c < n_counters; c += blockDim.x) counters[c] = 0;
  build_plan(pl, ids, P, E);

  const int nch = (I + R - 1) / R;
  const int items = pl.n_active * nch;
  int beg, end;
  item_range(items, beg, end);
  // An item is the double slab (gate rows i0.., up rows I+i0..) of one expert.
  auto issue = [&](int item, int b) {
    const int a = item / nch, c = item - a * nch, e = pl.act[a];
    const int i0 = c * R, nr = min(R, I - i0);
    Slab g, u;
    g.st = reinterpret_cast<const unsigned char *>(tab.gu[e] + (size_t)i0 * nbr);
    g.sc = tab.gus[e] + (size_t)i0 * nbr;
    u.st = reinterpret_cast<const unsigned char *>(tab.gu[e] + (size_t)(I + i0) * nbr);
    u.sc = tab.gus[e] + (size_t)(I + i0) * nbr;
    g.nrows = u.nrows = (uint32_t)nr;
    ring.issue2(b, g, u, R);
  };
  if (tid == 0)
    for (int it = beg; it < end && it < beg + kMoeNS; it++) issue(it, (it - beg) % kMoeNS);

  int staged_e = -1, staged_t0 = -1;
  for (int it = beg; it < end; it++) {
    const int j = it - beg, b = j % kMoeNS;
    const int a = it / nch, c = it - a * nch, e = pl.act[a];
    const int i0 = c * R, nr = min(R, I - i0);
    Slab g, u;
    g.st = reinterpret_cast<const unsigned char *>(tab.gu[e] + (size_t)i0 * nbr);
    g.sc = tab.gus[e] + (size_t)i0 * nbr;
    u.st = reinterpret_cast<const unsigned char *>(tab.gu[e] + (size_t)(I + i0) * nbr);
    u.sc = tab.gus[e] + (size_t)(I + i0) * nbr;
    g.nrows = u.nrows = (uint32_t)nr;
    const bool ok = ring.acquire2(b, g, u, R);
    const int cnt = pl.cnt[e], off = pl.off[e];
    for (int t0 = 0; t0 < cnt; t0 += TT) {
      const int ntok = min(TT, cnt - t0);
      if (e != staged_e || t0 != staged_t0) {
        __syncthreads();
        int tok[TT];
#pragma unroll
        for (int t = 0; t < TT; t++) tok[t] = t < ntok ? pl.list[off + t0 + t] / k : 0;
        stage_x<TT>(xs, x, H, tok, ntok);
        __syncthreads();
        staged_e = e;
        staged_t0 = t0;
      }
      if (ok) {
        const uint32_t st_base = smem_u32(ring.buf + (size_t)b * ring.stride);
        int rid[2 * RPW];
        bool rok[2 * RPW];
#pragma unroll
        for (int q = 0; q < RPW; q++) {
          rid[q] = warp + 8 * q;            // gate row
          rid[RPW + q] = R + warp + 8 * q;  // its up row
          rok[q] = rok[RPW + q] = warp + 8 * q < nr;
        }
        float acc[2 * RPW][TT];
        rows_dot_smem<2 * RPW, TT, SEG32>(st_base, st_base + ring.sc_off, nbr, seg_blocks, rid, rok, smem_u32(xs),
                                          acc);
#pragma unroll
        for (int q = 0; q < RPW; q++) {
          const float gv = lane_token<2 * RPW, TT>(acc, q), uv = lane_token<2 * RPW, TT>(acc, RPW + q);
          if (rok[q] && lane < ntok) {
            const int p = pl.list[off + t0 + lane];
            hidden[(size_t)p * I + i0 + rid[q]] = __bfloat16_as_ushort(__float2bfloat16_rn(silu_f(gv) * uv));
          }
        }
      }
    }
    __syncthreads();
    if (tid == 0 && it + kMoeNS < end) issue(it + kMoeNS, b);
  }
}

template <int MAXE, int TT, bool SEG32, int R>
__global__ void __launch_bounds__(256) k_moe_down(const __grid_constant__ MoeTable<MAXE> tab,
                                                  const int32_t *__restrict__ ids, const float *__restrict__ wts, int P,
                                                  int E, int k, int T, int H, int I, int seg_blocks,
                                                  const uint16_t *__restrict__ hidden, float *__restrict__ yws,
                                                  int *__restrict__ counters, uint16_t *__restrict__ out,
                                                  int bulk_scales) {
  extern __shared__ __align__(128) unsigned char smem[];
  grid_dep_wait();  // inputs and workspace come from, or are still read by, the preceding kernel
  grid_dep_release();
  constexpr int RPW = R / 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbr = I >> 5;
  const MoeGeom geo = moe_geom(nbr, TT, 1, R);
  PlanSmem &pl = *reinterpret_cast<PlanSmem *>(smem + 128);
  float2 *xs = reinterpret_cast<float2 *>(smem + 128 + round_up(sizeof(PlanSmem), 128u));
  __shared__ int s_last;
  SlabRing<kMoeNS> ring;
  ring.full = reinterpret_cast<uint64_t *>(smem);
  ring.buf = reinterpret_cast<unsigned char *>(xs) + geo.xs_bytes;
  ring.stride = geo.stride;
  ring.sc_off = geo.sc_off;
  ring.st_row = (uint32_t)nbr * 8u;
  ring.sc_row = (uint32_t)nbr;
  ring.bulk_scales = bulk_scales;
  ring.phase_bits = 0u;
  ring.timeouts = &g_tcf4_timeouts_moe;
  if (tid == 0) {
    for (int b = 0; b < kMoeNS; b++) mbar_init(&ring.full[b], 1);
    mbar_fence_init();
  }
  build_plan(pl, ids, P, E);
  if (pl.n_active == 0) {  // nothing routed anywhere: the layer output is zero
    for (int i = blockIdx.x * blockDim.x + tid; i < T * H; i += gridDim.x * blockDim.x) out[i] = 0;
    return;
  }

  const int nch = (H + R - 1) / R;
  const int items = pl.n_active * nch;
  int beg, end;
  item_range(items, beg, end);
  auto slab_of = [&](int item) {
    const int a = item / nch, c = item - a * nch, e = pl.act[a];
    const int n0 = c * R;
    Slab s;
    s.st = reinterpret_cast<const unsigned char *>(tab.dn[e] + (size_t)n0 * nbr);
    s.sc = tab.dns[e] + (size_t)n0 * nbr;
    s.nrows = (uint32_t)min(R, H - n0);
    return s;
  };
  if (tid == 0)
    for (int it = beg; it < end && it < beg + kMoeNS; it++) ring.issue((it - beg) % kMoeNS, slab_of(it));

  int staged_e = -1, staged_t0 = -1;
  for (int it = beg; it < end; it++) {
    const int j = it - beg, b = j % kMoeNS;
    const int a = it / nch, c = it - a * nch, e = pl.act[a];
    const int n0 = c * R;
    const Slab s = slab_of(it);
    const bool ok = ring.acquire(b, s);
    const int cnt = pl.cnt[e], off = pl.off[e];
    for (int t0 = 0; t0 < cnt; t0 += TT) {
      const int ntok = min(TT, cnt - t0);
      if (e != staged_e || t0 != staged_t0) {
        __syncthreads();
        int tok[TT];
#pragma unroll
        for (int t = 0; t < TT; t++) tok[t] = t < ntok ? pl.list[off + t0 + t] : 0;  // rows of h are pairs
        stage_x<TT>(xs, hidden, I, tok, ntok);
        __syncthreads();
        staged_e = e;
        staged_t0 = t0;
      }
      if (ok) {
        const uint32_t st_base = smem_u32(ring.buf + (size_t)b * ring.stride);
        int rid[RPW];
        bool rok[RPW];
#pragma unroll
        for (int q = 0; q < RPW; q++) {
          rid[q] = warp + 8 * q;
          rok[q] = rid[q] < (int)s.nrows;
        }
        float acc[RPW][TT];
        rows_dot_smem<RPW, TT, SEG32>(st_base, st_base + ring.sc_off, nbr, seg_blocks, rid, rok, smem_u32(xs), acc);
#pragma unroll
        for (int q = 0; q < RPW; q++) {
          const float v = lane_token<RPW, TT>(acc, q);
          if (rok[q] && lane < ntok) yws[(size_t)pl.list[off + t0 + lane] * H + n0 + rid[q]] = v;
        }
      }
    }
    // Publish this item's y, count it for its row chunk; the last of the chunk's n_active items
    // combines the chunk.
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&counters[c], 1) == pl.n_active - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      const int nr = min(R, H - n0);
      for (int i = tid; i < T * nr; i += blockDim.x) {
        const int t = i / nr, n = n0 + (i - t * nr);
        float acc = 0.f;
        for (int jj = 0; jj < k; jj++) {
          const int p = t * k + jj, ee = pl.ids[p];
          if (ee < 0 || ee >= E) continue;
          acc = fmaf(__ldg(wts + p), __ldcg(yws + (size_t)p * H + n), acc);
        }
        out[(size_t)t * H + n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
      }
    }
    __syncthreads();
    if (tid == 0 && it + kMoeNS < end) ring.issue(b, slab_of(it + kMoeNS));
  }
}

// Pointer table and host-side facts shared by the two launches.
template <int MAXE>
struct MoeLaunch {
  MoeTable<MAXE> tab;
  bool scales_aligned = true;
  int nsm = 148;
  int *counters;
  uint16_t *hidden;
  float *yws;
};

// Rows per work item: 16 while a slab of `parts` row groups stays within ~40 KB, else 8.
static int moe_rows(int nbr, int parts) { return (size_t)parts * 16 * nbr * 9 <= 40 * 1024 ? 16 : 8; }

// Tokens per decode pass: as many (up to 4, never more than T) as fit next to the slab ring.
static int moe_tt(int T, int nbr, int parts) {
  int TT = T == 1 ? 1 : (T == 2 ? 2 : 4);
  while (TT > 1 && moe_geom(nbr, TT, parts, moe_rows(nbr, parts)).smem > 220u * 1024u) TT >>= 1;
  return TT;
}

template <int MAXE, int TT, bool SEG32, int R>
static cudaError_t launch_gateup(const MoeLaunch<MAXE> &ml, const tcf4_moe &m, int seg, const uint16_t *x, int T,
                                 const int32_t *ids, int k, cudaStream_t s) {
  static unsigned long long attr = 0;
  cudaError_t e = ensure_max_dynamic_smem(k_moe_gateup<MAXE, TT, SEG32, R>, attr);
  if (e != cudaSuccess) return e;
  const int nbr = m.H / 32;
  const MoeGeom g = moe_geom(nbr, TT, 2, R);
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_moe_gateup<MAXE, TT, SEG32, R>, 256, g.smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  const int max_active = T * k < m.E ? T * k : m.E;
  int grid = ml.nsm * occ;
  const int items = max_active * ((m.I + R - 1) / R);
  if (grid > items) grid = items;
  const int bulk = ml.scales_aligned && (R * nbr) % 16 == 0 && ((size_t)m.I * nbr) % 16 == 0;
  const int n_counters = (m.H + kMoeRMin - 1) / kMoeRMin;
  return launch_dependent(k_moe_gateup<MAXE, TT, SEG32, R>, dim3(grid), dim3(256), g.smem, s, ml.tab, ids, T * k, m.E,
                          k, m.H, m.I, seg, x, ml.hidden, ml.counters, n_counters, bulk);
}

template <int MAXE, int TT, bool SEG32, int R>
static cudaError_t launch_down(const MoeLaunch<MAXE> &ml, const tcf4_moe &m, int seg, int T, const int32_t *ids,
                               const float *wts, int k, uint16_t *out, cudaStream_t s) {
  static unsigned long long attr = 0;
  cudaError_t e = ensure_max_dynamic_smem(k_moe_down<MAXE, TT, SEG32, R>, attr);
  if (e != cudaSuccess) return e;
  const int nbr = m.I / 32;
  const MoeGeom g = moe_geom(nbr, TT, 1, R);
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_moe_down<MAXE, TT, SEG32, R>, 256, g.smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  const int max_active = T * k < m.E ? T * k : m.E;
  int grid = ml.nsm * occ;
  const int items = max_active * ((m.H + R - 1) / R);
  if (grid > items) grid = items;
  const int bulk = ml.scales_aligned && (R * nbr) % 16 == 0;
  return launch_dependent(k_moe_down<MAXE, TT, SEG32, R>, dim3(grid), dim3(256), g.smem, s, ml.tab, ids, wts, T * k,
                          m.E, k, T, m.H, m.I, seg, (const uint16_t *)ml.hidden, ml.yws, ml.counters, out, bulk);
}

// Dispatch (TT, seg_len == 32, R) to a compiled instance.
template <int MAXE, template <int, int, bool, int> class F, class... A>
static cudaError_t dispatch(int TT, bool seg32, int R, A &&...a) {
#define TCF4_CASE(TTv, SEGv, Rv) \
  if (TT == TTv && seg32 == SEGv && R == Rv) return F<MAXE, TTv, SEGv, Rv>::run(a...);
  TCF4_CASE(1, true, 16) TCF4_CASE(1, true, 8) TCF4_CASE(1, false, 16) TCF4_CASE(1, false, 8)
  TCF4_CASE(2, true, 16) TCF4_CASE(2, true, 8) TCF4_CASE(2, false, 16) TCF4_CASE(2, false, 8)
  TCF4_CASE(4, true, 16) TCF4_CASE(4, true, 8) TCF4_CASE(4, false, 16) TCF4_CASE(4, false, 8)
#undef TCF4_CASE
  return cudaErrorInvalidConfiguration;
}

template <int MAXE, int TT, bool SEG32, int R>
struct GateupF {
  static cudaError_t run(const MoeLaunch<MAXE> &ml, const tcf4_moe &m, int seg, const uint16_t *x, int T,
                         const int32_t *ids, int k, cudaStream_t s) {
    return launch_gateup<MAXE, TT, SEG32, R>(ml, m, seg, x, T, ids, k, s);
  }
};
template <int MAXE, int TT, bool SEG32, int R>
struct DownF {
  static cudaError_t run(const MoeLaunch<MAXE> &ml, const tcf4_moe &m, int seg, int T, const int32_t *ids,
                         const float *wts, int k, uint16_t *out, cudaStream_t s) {
    return launch_down<MAXE, TT, SEG32, R>(ml, m, seg, T, ids, wts, k, out, s);
  }
};

template <int MAXE>
static cudaError_t launch_moe_e(const tcf4_moe &m, int gu_seg, int dn_seg, const uint16_t *x, int T,
                                const int32_t *ids, const float *wts, int k, uint16_t *out, void *ws, cudaStream_t s) {
  MoeLaunch<MAXE> ml;
  for (int e = 0; e < MAXE; e++) {
    const bool ok = e < m.E;
    ml.tab.gu[e] = ok ? reinterpret_cast<const uint2 *>(m.gate_up[e].stream) : nullptr;
    ml.tab.gus[e] = ok ? m.gate_up[e].scales : nullptr;
    ml.tab.dn[e] = ok ? reinterpret_cast<const uint2 *>(m.down[e].stream) : nullptr;
    ml.tab.dns[e] = ok ? m.down[e].scales : nullptr;
    if (ok && ((reinterpret_cast<uintptr_t>(ml.tab.gus[e]) | reinterpret_cast<uintptr_t>(ml.tab.dns[e])) & 15u))
      ml.scales_aligned = false;
  }
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&ml.nsm, cudaDevAttrMultiProcessorCount, dev);
  const MoeWorkspace L = moe_workspace_layout(m.E, T, k, m.H, m.I);
  char *base = static_cast<char *>(ws);
  ml.counters = reinterpret_cast<int *>(base + L.counters);
  ml.hidden = reinterpret_cast<uint16_t *>(base + L.hidden);
  ml.yws = reinterpret_cast<float *>(base + L.y);
  const int nbr_gu = m.H / 32, nbr_dn = m.I / 32;
  cudaError_t e = dispatch<MAXE, GateupF>(moe_tt(T, nbr_gu, 2), gu_seg == 1, moe_rows(nbr_gu, 2), ml, m, gu_seg, x,
                                           T, ids, k, s);
  if (e != cudaSuccess) return e;
  return dispatch<MAXE, DownF>(moe_tt(T, nbr_dn, 1), dn_seg == 1, moe_rows(nbr_dn, 1), ml, m, dn_seg, T, ids, wts, k,
                               out, s);
}

cudaError_t launch_moe(const tcf4_moe &m, int gu_seg, int dn_seg, const uint16_t *x, int T, const int32_t *ids,
                       const float *wts, int k, uint16_t *out, void *ws, cudaStream_t s) {
  if (m.E <= 32) return launch_moe_e<32>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
  return launch_moe_e<256>(m, gu_seg, dn_seg, x, T, ids, wts, k, out, ws, s);
}

unsigned int take_timeouts_moe() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_tcf4_timeouts_moe, sizeof v) != cudaSuccess) return 0;
  cudaMemcpyToSymbol(g_tcf4_timeouts_moe, &zero, sizeof zero);
  return v;
}

}  // namespace tcf4
