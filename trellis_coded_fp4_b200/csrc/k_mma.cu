// k_mma.cu -- fused trellis decode + block-scaled tensor-core product (tcgen05, sm_100a).
//
// HEPH abstract, first serving mode: the compressed stream stays resident and is decoded inside the
// product. The product runs on the 5th-generation tensor cores: the decoded weights are already
// MXFP4 elements (E2M1 codes with a UE8M0 scale per 32 weights), so they feed a block-scaled
// kind::mxf8f6f4 MMA directly as the A operand (E2M1, scale factors = the weights' own UE8M0
// bytes). The bf16 activations are the B operand, split exactly into two E4M3 terms per element
// (hi + lo, each 32-block with its own UE8M0 scale): B column 2t holds token t's hi term and column
// 2t+1 its lo term, so y[t] = D[:, 2t] + D[:, 2t+1] in fp32.
//
// One persistent CTA per SM: 8 decode warps + 1 control warp, over 128-row tiles ("jobs"):
//  * decode thread (warp w, lane l) owns tile row 32(w%4)+l and K-blocks 4(w/4)..4(w/4)+3 of each
//    256-wide K stage. It keeps kPref stages of its 32 bytes of trellis words in flight with
//    cp.async, decodes them in registers (bit-sliced) into E2M1 codes in the shared A stage, and
//    stages its row's 4 scale bytes; one stage later warps 0-3 move the stage's A and B scale
//    factors into TMEM (tcgen05.st) and release it.
//  * the control thread streams the pre-split activations (B) with bulk copies kNB stages ahead
//    and issues the stage's 8 MMAs (K = 32 each) into a double-buffered TMEM accumulator.
//  * the epilogue of job i (tcgen05.ld, then the GEMV output, the SwiGLU of gate/up rows, or the MoE
//    down rows and their combine) runs in warps 0-3 during job i+1.
// Every mbarrier wait is bounded; a wait that gives up raises a shared abort flag that all decode
// threads read after the per-stage named barrier, so the CTA leaves together and frees its TMEM.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "tcf4_device.cuh"
#include "tcf4_internal.h"
#include "tcf4_pipe.cuh"
#include "tcf4_tc.cuh"

namespace tcf4 {

__device__ unsigned int g_tcf4_timeouts_mma = 0;

constexpr int kKS = 256;              // K elements per stage (8 blocks of 32)
constexpr int kNA = 3;                // A stages (E2M1 tile + scale-factor TMEM slot)
constexpr int kNB = 4;                // B stages (activation split)
constexpr int kPref = 4;              // trellis-word stages in flight per decode thread
constexpr int kDec = 256;             // decode threads
constexpr int kMmaThreads = kDec + 32;
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kSfaCol = 64, kSfbCol = 88;  // scale-factor slots: 8 and 4 TMEM columns per stage
constexpr uint32_t kSboA = 2048;      // 16 K chunks x 128 B per 8-row group of a stage
constexpr int kMaxGroups = kMaxTokens * kMaxTopK + kMaxExperts / 2;

enum MmaMode { kModeGemv = 0, kModeGateUp = 1, kModeDown = 2 };

// K position (0..31) inside a 32-block of the MMA that holds weight i of the block: the decoder's
// interleaved nibble words put weight 4v+j in nibble v of word j, and word j fills bytes 4j..4j+3
// of the block's 16 data bytes (16-element chunk j/2, elements 8(j%2)..8(j%2)+7).
__host__ __device__ constexpr int kpos_of_weight(int i) { return 16 * ((i & 3) >> 1) + 8 * (i & 1) + (i >> 2); }

// Byte offset of element (n, k), k < 256, in a K-major no-swizzle stage of 8-bit containers:
// core matrices of 8 rows x 16 bytes, LBO = 128 (K chunks), SBO = 2048 (8-row groups).
__host__ __device__ constexpr uint32_t kmajor_off(uint32_t n, uint32_t k) {
  return (n >> 3) * kSboA + (k >> 4) * 128u + (n & 7u) * 16u + (k & 15u);
}

// ------------------------------------------------------------------------------- routing groups
// MoE work is split into groups: an active expert with its routed pairs, at most gmax per group.
struct GroupPlan {
  int cnt[kMaxExperts];
  int off[kMaxExperts];
  int list[kMaxTokens * kMaxTopK];  // pairs p = t*k + j per expert, in p order
  int ids[kMaxTokens * kMaxTopK];
  int g_e[kMaxGroups];              // expert of group g
  int g_first[kMaxGroups];          // first index into list[] of group g
  int g_cnt[kMaxGroups];            // pairs in group g (<= gmax)
  int n_groups;
};

// All threads of the CTA. Pairs whose expert id is outside [0, E) are dropped. Deterministic.
__device__ void build_groups(GroupPlan &pl, const int32_t *__restrict__ ids, int P, int E, int gmax) {
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
    int o = 0, ng = 0;
    for (int e = 0; e < E; e++) {
      pl.off[e] = o;
      for (int f = 0; f < pl.cnt[e]; f += gmax) {
        pl.g_e[ng] = e;
        pl.g_first[ng] = o + f;
        pl.g_cnt[ng] = pl.cnt[e] - f < gmax ? pl.cnt[e] - f : gmax;
        ng++;
      }
      o += pl.cnt[e];
    }
    pl.n_groups = ng;
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

// ------------------------------------------------------------------------------- activation split
// One 32-element block of one source row -> hi/lo E4M3 terms. hi = E4M3(x / 2^Eh) with
// Eh = floor(log2 max|x|) - 7 over the block (so max|x|/2^Eh lies in [128, 256)); lo the same for
// the residual x - hi*2^Eh, exact in fp32. hi*2^Eh + lo*2^El reproduces every bf16 x of the block
// except elements more than ~17 binades below the block maximum.
__device__ __forceinline__ void split_e4m3(float v, float mx, uint8_t &q, uint32_t &sf, float &back) {
  if (!(mx > 0.f)) {
    q = 0;
    sf = 127u;
    back = 0.f;
    return;
  }
  int e = ilogbf(mx) - 7;
  e = e < -126 ? -126 : (e > 127 ? 127 : e);
  q = (uint8_t)__nv_cvt_float_to_fp8(scalbnf(v, -e), __NV_SATFINITE, __NV_E4M3);
  const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)q, __NV_E4M3);
  back = scalbnf(__half2float(__half(hr)), e);
  sf = (uint32_t)(e + 127);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Per group: Bg [S stages][NMAX*256 bytes] (one K-major B stage each) and Bsf [S][32 lanes][4
// words], word 2g+c of a lane = UE8M0 bytes of B column 32c+lane for K-blocks 4g..4g+3.
__host__ __device__ inline size_t bsplit_group_bytes(int S, int NMAX) { return (size_t)S * NMAX * 256; }
__host__ __device__ inline size_t bsf_group_words(int S) { return (size_t)S * 32 * 4; }

// Write the split of one block (p = token slot, kb = 32-block) into one group's B stages.
template <int NMAX>
__device__ __forceinline__ void bsplit_block(float v, int p, int kb, uint8_t *Bg_g, uint32_t *Bsf_g) {
  const int lane = threadIdx.x & 31;
  uint8_t qh, ql;
  uint32_t sfh, sfl;
  float bh, bl;
  split_e4m3(v, warp_max(fabsf(v)), qh, sfh, bh);
  const float res = v - bh;
  split_e4m3(res, warp_max(fabsf(res)), ql, sfl, bl);
  const int s = kb >> 3, kin = (kb & 7) * 32 + kpos_of_weight(lane);
  uint8_t *stage = Bg_g + (size_t)s * NMAX * 256;
  stage[kmajor_off(2 * p, kin)] = qh;
  stage[kmajor_off(2 * p + 1, kin)] = ql;
  if (lane < 2) {
    const int n = 2 * p + lane, g = (kb & 7) >> 2;
    uint8_t *sfb = reinterpret_cast<uint8_t *>(Bsf_g + ((size_t)s * 32 + (n & 31)) * 4 + 2 * g + (n >> 5));
    sfb[kb & 3] = (uint8_t)(lane == 0 ? sfh : sfl);
  }
}

// Plain GEMV: one group, token slots 0..T-1 (the other slots up to NMAX/2 are zero columns).
template <int NMAX>
__global__ void __launch_bounds__(256) k_bsplit_gemv(const uint16_t *__restrict__ x, int T, int K,
                                                     uint8_t *__restrict__ Bg, uint32_t *__restrict__ Bsf) {
  const int nb = K >> 5, lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int wi = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; wi < (NMAX / 2) * nb; wi += nwarps) {
    const int p = wi / nb, kb = wi - p * nb;
    const float v = p < T ? __uint_as_float((uint32_t)x[(size_t)p * K + kb * 32 + lane] << 16) : 0.f;
    bsplit_block<NMAX>(v, p, kb, Bg, Bsf);
  }
}

// MoE: group g's token slot i is pair list[g_first + i]; its activation row is src[pair / div]
// (gate_up reads x rows of tokens: div = k; down reads h rows of pairs: div = 1). Block 0 also
// clears the down kernel's chunk counters when `counters` is given.
template <int NMAX>
__global__ void __launch_bounds__(256) k_bsplit_moe(const int32_t *__restrict__ ids, int P, int E, int div,
                                                    const uint16_t *__restrict__ src, int K, uint8_t *__restrict__ Bg,
                                                    uint32_t *__restrict__ Bsf, int *__restrict__ counters,
                                                    int n_counters) {
  __shared__ GroupPlan pl;
  if (counters != nullptr && blockIdx.x == 0)
    for (int c = threadIdx.x; c < n_counters; c += blockDim.x) counters[c] = 0;
  build_groups(pl, ids, P, E, NMAX / 2);
  const int nb = K >> 5, S = (nb + 7) >> 3;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int per_group = (NMAX / 2) * nb;
  for (int wi = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; wi < pl.n_groups * per_group; wi += nwarps) {
    const int g = wi / per_group, r = wi - g * per_group;
    const int p = r / nb, kb = r - p * nb;
    float v = 0.f;
    if (p < pl.g_cnt[g]) {
      const int row = pl.list[pl.g_first[g] + p] / div;
      v = __uint_as_float((uint32_t)src[(size_t)row * K + kb * 32 + lane] << 16);
    }
    bsplit_block<NMAX>(v, p, kb, Bg + (size_t)g * bsplit_group_bytes(S, NMAX), Bsf + (size_t)g * bsf_group_words(S));
  }
}

// ------------------------------------------------------------------------------- geometry

// Shared memory: barriers | A ring | B ring | trellis-word ring | B-scale ring | scale staging
// | gate/up exchange | group plan | two scale slabs.
struct MmaGeom {
  uint32_t off_A, off_B, off_C, off_F, off_X, off_U, off_P, off_S, slab, smem;
};

__host__ __device__ inline MmaGeom mma_geom(int nbr, int NMAX, int mode) {
  MmaGeom g;
  g.off_A = 1024u;
  g.off_B = g.off_A + kNA * 128u * kKS;
  g.off_C = g.off_B + kNB * (uint32_t)NMAX * kKS;
  g.off_F = g.off_C + kPref * kDec * 32u;
  g.off_X = g.off_F + kPref * 128u * 16u;
  g.off_U = g.off_X + kNA * 1024u;
  g.off_P = g.off_U + (mode == kModeGateUp ? 2u * 64u * (uint32_t)(NMAX / 2) * 4u : 0u);
  g.off_S = g.off_P + (mode == kModeGemv ? 0u : round_up((uint32_t)sizeof(GroupPlan), 128u));
  g.slab = round_up(128u * (uint32_t)nbr + 16u, 16u);  // +16: tail reads of a row's 4 scale bytes
  g.smem = g.off_S + 2u * g.slab;
  return g;
}

__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts_u2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t a) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}

__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// ------------------------------------------------------------------------------- kernel arguments

struct MmaArgs {
  MatView w;              // GEMV: the matrix (MoE: rows/stream unused; experts come from the table)
  int nbr;                // 32-blocks per row (K / 32)
  const uint8_t *Bg;      // activation split, per group
  const uint32_t *Bsf;
  int T;                  // GEMV tokens
  uint16_t *y;            // GEMV out [T][rows]
  const int32_t *ids;     // MoE routing [T][k]
  const float *wts;
  int P, E, k, Tm, H, I;
  uint16_t *hidden;       // [P][I] bf16
  float *yws;             // [P][H] fp32
  int *counters;          // per 128-row chunk of H
  uint16_t *out;          // [T][H] bf16
};

// A job is one 128-row tile: rows [0, na) from (st0, sc0) and, when split, rows [64, 64 + nb) from
// (st1, sc1); B group `group`, MMA width ncols; `cnt` tokens starting at list index `first`.
struct JobRows {
  const uint2 *st0, *st1;
  const uint8_t *sc0, *sc1;
  int na, nb, split, group, ncols, row0, chunk, cnt, first;
};

template <int MAXE, int MODE, int NMAX>
__device__ __forceinline__ JobRows job_rows(const MmaArgs &a, const MoeTable<MAXE> &tab, const GroupPlan *pl,
                                            int job) {
  JobRows j;
  j.split = 0;
  j.st1 = nullptr;
  j.sc1 = nullptr;
  j.nb = 0;
  if (MODE == kModeGemv) {
    const int r0 = job * 128;
    j.st0 = a.w.stream + (size_t)r0 * a.nbr;
    j.sc0 = a.w.scales + (size_t)r0 * a.nbr;
    j.na = a.w.rows - r0 < 128 ? a.w.rows - r0 : 128;
    j.group = 0;
    j.ncols = NMAX;
    j.row0 = r0;
    j.chunk = job;
    j.cnt = a.T;
    j.first = 0;
  } else if (MODE == kModeGateUp) {
    const int nch = (a.I + 63) / 64;
    const int g = job / nch, c = job - g * nch, e = pl->g_e[g];
    const int i0 = 64 * c;
    j.split = 1;
    j.st0 = tab.gu[e] + (size_t)i0 * a.nbr;
    j.sc0 = tab.gus[e] + (size_t)i0 * a.nbr;
    j.st1 = tab.gu[e] + (size_t)(a.I + i0) * a.nbr;
    j.sc1 = tab.gus[e] + (size_t)(a.I + i0) * a.nbr;
    j.na = j.nb = a.I - i0 < 64 ? a.I - i0 : 64;
    j.group = g;
    j.cnt = pl->g_cnt[g];
    j.first = pl->g_first[g];
    j.ncols = (2 * j.cnt + 15) / 16 * 16;
    j.row0 = i0;
    j.chunk = c;
  } else {
    const int nch = (a.H + 127) / 128;
    const int g = job / nch, c = job - g * nch, e = pl->g_e[g];
    const int n0 = 128 * c;
    j.st0 = tab.dn[e] + (size_t)n0 * a.nbr;
    j.sc0 = tab.dns[e] + (size_t)n0 * a.nbr;
    j.na = a.H - n0 < 128 ? a.H - n0 : 128;
    j.group = g;
    j.cnt = pl->g_cnt[g];
    j.first = pl->g_first[g];
    j.ncols = (2 * j.cnt + 15) / 16 * 16;
    j.row0 = n0;
    j.chunk = c;
  }
  return j;
}

__device__ __forceinline__ bool row_valid(const JobRows &j, int m) {
  return j.split ? (m < 64 ? m < j.na : m - 64 < j.nb) : m < j.na;
}

// ------------------------------------------------------------------------------- the kernel

template <int MAXE, int MODE, int NMAX>
__global__ void __launch_bounds__(kMmaThreads, 1) k_mma(const __grid_constant__ MmaArgs a,
                                                        const __grid_constant__ MoeTable<MAXE> tab) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbr = a.nbr, S = (nbr + 7) >> 3;
  const MmaGeom geo = mma_geom(nbr, NMAX, MODE);
  uint64_t *a_full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *a_empty = a_full + 4, *b_full = a_full + 8, *b_empty = a_full + 16, *acc_full = a_full + 24,
           *acc_empty = a_full + 26;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 256);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + 260);
  volatile int *s_last = reinterpret_cast<volatile int *>(smem + 264);
  unsigned int *tmo = &g_tcf4_timeouts_mma;
  GroupPlan *pl = reinterpret_cast<GroupPlan *>(smem + geo.off_P);

  if (tid == 0) {
    for (int b = 0; b < kNA; b++) {
      mbar_init(&a_full[b], 8);
      mbar_init(&a_empty[b], 1);
    }
    for (int b = 0; b < kNB; b++) {
      mbar_init(&b_full[b], 1);
      mbar_init(&b_empty[b], 1);
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  int njobs;
  if (MODE == kModeGemv) {
    njobs = (a.w.rows + 127) >> 7;
  } else {
    build_groups(*pl, a.ids, a.P, a.E, NMAX / 2);  // synchronizes the CTA
    njobs = pl->n_groups * (MODE == kModeGateUp ? (a.I + 63) / 64 : (a.H + 127) / 128);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int my_jobs = (int)blockIdx.x < njobs ? (njobs - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int nq = my_jobs * S;
  auto job_of = [&](int jl) { return (int)blockIdx.x + jl * (int)gridDim.x; };

  if (warp < 8) {
    // ---------------------------------------------------------------- decode warps
    const int sp = warp & 3, h = warp >> 2, m = 32 * sp + lane;
    const uint32_t cbase = smem_u32(smem + geo.off_C) + (uint32_t)tid * 32u;
    const uint32_t fbase = smem_u32(smem + geo.off_F) + (uint32_t)tid * 16u;
    const uint32_t xbase = smem_u32(smem + geo.off_X);
    const uint32_t sbase = smem_u32(smem + geo.off_S);
    const int tail_blocks = nbr - 8 * (S - 1) - 4 * h;  // this thread's blocks in the last stage
    const uint32_t tail = tail_blocks <= 0 ? 0u : (tail_blocks >= 4 ? 32u : 8u * (uint32_t)tail_blocks);

    // Prefetch front: job jl_i, stage s_i; src walks this thread's row 64 bytes per stage.
    int jl_i = 0, s_i = 0;
    const uint2 *src_i = a.w.stream;
    bool rv_i = false;
    const uint32_t *bsf_i = a.Bsf;
    JobRows ji{};
    auto start_job_front = [&]() {
      ji = job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl_i));
      rv_i = row_valid(ji, m);
      src_i = rv_i ? (ji.split && m >= 64 ? ji.st1 + (size_t)(m - 64) * nbr : ji.st0 + (size_t)m * nbr) + 4 * h
                   : a.w.stream;
      bsf_i = a.Bsf + (size_t)ji.group * bsf_group_words(S) + (size_t)lane * 4;
    };
    if (my_jobs) start_job_front();
    uint32_t slot_i = 0;  // ring slot of the front (q % kPref)
    auto issue_next = [&](bool live) {
      if (live) {
        const uint32_t bytes = rv_i ? (s_i == S - 1 ? tail : 32u) : 0u;
        const uint32_t dst = cbase + slot_i * (uint32_t)(kDec * 32);
        cp_async16(dst, src_i, bytes > 16u ? 16u : bytes);
        cp_async16(dst + 16u, bytes > 16u ? src_i + 2 : src_i, bytes > 16u ? bytes - 16u : 0u);
        if (warp < 4) cp_async16(fbase + slot_i * (128u * 16u), bsf_i, 16u);
        if (s_i == 0) {  // the job's scale bytes, into slab buffer jl_i % 2
          const uint32_t sdst = sbase + (uint32_t)(jl_i & 1) * geo.slab;
          const uint32_t t0 = (uint32_t)ji.na * (uint32_t)nbr;
          for (uint32_t c = tid; c * 16u < t0; c += kDec)
            cp_async16(sdst + c * 16u, ji.sc0 + c * 16u, t0 - c * 16u < 16u ? t0 - c * 16u : 16u);
          if (ji.split) {
            const uint32_t t1 = (uint32_t)ji.nb * (uint32_t)nbr, o1 = 64u * (uint32_t)nbr;
            for (uint32_t c = tid; c * 16u < t1; c += kDec)
              cp_async16(sdst + o1 + c * 16u, ji.sc1 + c * 16u, t1 - c * 16u < 16u ? t1 - c * 16u : 16u);
          }
        }
        src_i += 8;
        bsf_i += 32 * 4;
        if (++s_i == S) {
          s_i = 0;
          if (++jl_i < my_jobs) start_job_front();
        }
        slot_i = (slot_i + 1) & (kPref - 1);
      }
      cp_async_commit();
    };

    // scale factors of the stage in A buffer bp into TMEM (warps 0-3), then release it to the MMA
    auto publish_scales = [&](uint32_t bp, const uint4 &sfb) {
      const uint32_t lane_addr = tbase + ((uint32_t)(32 * warp) << 16);
      const uint4 x0 = lds_u4(xbase + bp * 1024u + (uint32_t)lane * 32u);
      const uint4 x1 = lds_u4(xbase + bp * 1024u + (uint32_t)lane * 32u + 16u);
      const uint32_t w8[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      tmem_st_x8(lane_addr + kSfaCol + 8u * bp, w8);
      tmem_st_x4(lane_addr + kSfbCol + 4u * bp, sfb.x, sfb.y, sfb.z, sfb.w);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[bp]);
    };

    // epilogue of local job jl (warps 0-3)
    auto epilogue = [&](int jl) {
      const JobRows jr = job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl));
      const int buf = jl & 1;
      if (!mbar_wait(&acc_full[buf], (uint32_t)(jl >> 1) & 1u, tmo)) *abort_flag = 1;
      tc_fence_after();
      float v[NMAX / 2];
#pragma unroll
      for (int c0 = 0; c0 < NMAX; c0 += 16) {
        uint32_t r[16];
        tmem_ld_x16(tbase + ((uint32_t)(32 * warp) << 16) + (uint32_t)(buf * NMAX + c0), r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; j++) v[c0 / 2 + j] = __uint_as_float(r[2 * j]) + __uint_as_float(r[2 * j + 1]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      const int mrow = 32 * warp + lane;
      if (MODE == kModeGemv) {
        if (mrow < jr.na)
#pragma unroll
          for (int t = 0; t < NMAX / 2; t++)
            if (t < a.T)
              a.y[(size_t)t * a.w.rows + jr.row0 + mrow] = __bfloat16_as_ushort(__float2bfloat16_rn(v[t]));
      } else if (MODE == kModeGateUp) {
        float *U = reinterpret_cast<float *>(smem + geo.off_U) + (size_t)buf * 64 * (NMAX / 2);
        if (mrow >= 64)
#pragma unroll
          for (int t = 0; t < NMAX / 2; t++) U[(mrow - 64) * (NMAX / 2) + t] = v[t];
        named_bar(3, 128);
        if (mrow < 64 && mrow < jr.na)
#pragma unroll
          for (int t = 0; t < NMAX / 2; t++)
            if (t < jr.cnt) {
              const float g = v[t], u = U[mrow * (NMAX / 2) + t];
              const int p = pl->list[jr.first + t];
              a.hidden[(size_t)p * a.I + jr.row0 + mrow] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(g / (1.0f + expf(-g)) * u));
            }
      } else {
        if (mrow < jr.na)
#pragma unroll
          for (int t = 0; t < NMAX / 2; t++)
            if (t < jr.cnt) a.yws[(size_t)pl->list[jr.first + t] * a.H + jr.row0 + mrow] = v[t];
        __threadfence();
        named_bar(3, 128);
        // the last group to finish this 128-row chunk combines it: out = sum_j w_j y_j (fixed j order)
        if (tid == 0) *s_last = atomicAdd(&a.counters[jr.chunk], 1) == pl->n_groups - 1;
        named_bar(3, 128);
        if (*s_last) {
          __threadfence();
          for (int i = tid; i < a.Tm * jr.na; i += 128) {
            const int t = i / jr.na, n = jr.row0 + (i - t * jr.na);
            float acc = 0.f;
            for (int jj = 0; jj < a.k; jj++) {
              const int p = t * a.k + jj, ee = pl->ids[p];
              if (ee < 0 || ee >= a.E) continue;
              acc = fmaf(__ldg(a.wts + p), __ldcg(a.yws + (size_t)p * a.H + n), acc);
            }
            a.out[(size_t)t * a.H + n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
          }
        }
      }
    };

    for (int q = 0; q < kPref; q++) issue_next(q < nq);
    uint4 sfb_prev = make_uint4(0u, 0u, 0u, 0u);
    int jl = 0, s = 0, q = 0;
    uint32_t b = 0, bprev = kNA - 1, empty_phase = 0u, slot = 0;  // A buffer, previous, a_empty parities
    uint32_t srow = sbase + (uint32_t)m * (uint32_t)nbr + 4u * (uint32_t)h;  // this row's scale bytes, job 0
    for (; q < nq; q++) {
      cp_async_wait<kPref - 1>();
      named_bar(1, kDec);
      if (*abort_flag) break;
      if (warp < 4 && q >= 1) publish_scales(bprev, sfb_prev);
      const uint4 c0 = lds_u4(cbase + slot * (uint32_t)(kDec * 32)), c1 = lds_u4(cbase + slot * (uint32_t)(kDec * 32) + 16u);
      if (warp < 4) sfb_prev = lds_u4(fbase + slot * (128u * 16u));
      // this row's 4 scale bytes of the stage (two 16-bit reads of the job's slab)
      const uint32_t sa = srow + (uint32_t)(jl & 1) * geo.slab + 8u * (uint32_t)s;
      const uint32_t sfw = lds_u16(sa) | (lds_u16(sa + 2u) << 16);
      issue_next(q + kPref < nq);
      uint32_t W[4][4];
      planes_to_nibbles_interleaved(decode_block0(c0.x, c0.y), W[0][0], W[0][1], W[0][2], W[0][3]);
      planes_to_nibbles_interleaved(decode_block0(c0.z, c0.w), W[1][0], W[1][1], W[1][2], W[1][3]);
      planes_to_nibbles_interleaved(decode_block0(c1.x, c1.y), W[2][0], W[2][1], W[2][2], W[2][3]);
      planes_to_nibbles_interleaved(decode_block0(c1.z, c1.w), W[3][0], W[3][1], W[3][2], W[3][3]);
      if (q >= kNA) {
        if (lane == 0 && !mbar_wait(&a_empty[b], (empty_phase >> b) & 1u, tmo)) *abort_flag = 1;
        empty_phase ^= 1u << b;
        __syncwarp();
      }
      const uint32_t abase = smem_u32(smem + geo.off_A) + b * (128u * kKS) + (uint32_t)(m >> 3) * kSboA +
                             (uint32_t)(m & 7) * 16u + (uint32_t)h * 1024u;
#pragma unroll
      for (int i = 0; i < 4; i++) {
        sts_u2(abase + (uint32_t)(2 * i) * 128u, W[i][0], W[i][1]);
        sts_u2(abase + (uint32_t)(2 * i + 1) * 128u, W[i][2], W[i][3]);
      }
      // scale word of row m (row group sp), K-blocks 4h..4h+3 -> staging word 4h+sp of this lane
      sts_u32(xbase + b * 1024u + (uint32_t)lane * 32u + (uint32_t)(4 * h + sp) * 4u, sfw);
      fence_proxy_async_smem();
      if (warp >= 4) {  // warps 4-7 release the stage now; warps 0-3 after its scales are in TMEM
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[b]);
      }
      if (warp < 4 && jl >= 1 && s == 1) epilogue(jl - 1);
      bprev = b;
      b = b + 1 == kNA ? 0u : b + 1;
      slot = (slot + 1) & (kPref - 1);
      if (++s == S) {
        s = 0;
        ++jl;
      }
    }
    if (q == nq && nq > 0) {
      named_bar(1, kDec);  // the last stage's scale staging is complete
      if (warp < 4) {
        publish_scales(bprev, sfb_prev);
        epilogue(my_jobs - 1);
      }
    }
    cp_async_wait_all();
  } else {
    // ---------------------------------------------------------------- control warp
    if (lane == 0) {
      const uint32_t bstage = (uint32_t)NMAX * kKS;
      int jl_b = 0, s_b = 0;
      const uint8_t *bsrc = a.Bg;
      auto front_group = [&]() {
        bsrc = a.Bg + (size_t)job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl_b)).group * bsplit_group_bytes(S, NMAX);
      };
      if (my_jobs) front_group();
      uint32_t bb_i = 0;
      auto issue_b = [&]() {  // B stage of the prefetch front (jl_b, s_b) into ring slot bb_i
        mbar_arrive_expect_tx(&b_full[bb_i], bstage);
        bulk_g2s(smem + geo.off_B + bb_i * bstage, bsrc, bstage, &b_full[bb_i]);
        bsrc += bstage;
        if (++s_b == S) {
          s_b = 0;
          if (++jl_b < my_jobs) front_group();
        }
        bb_i = bb_i + 1 == kNB ? 0u : bb_i + 1;
      };
      int issued_b = 0;
      for (; issued_b < kNB && issued_b < nq; issued_b++) issue_b();
      // instruction descriptors for the four scale-factor byte positions
      int jl = 0, s = 0;
      uint32_t ncols = (uint32_t)(my_jobs ? job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(0)).ncols : NMAX);
      uint32_t idesc[4];
      for (int i = 0; i < 4; i++) idesc[i] = idesc_mxf8f6f4_e2m1_e4m3(ncols, (uint32_t)i, (uint32_t)i);
      uint32_t b = 0, bb = 0, full_phase = 0u, bfull_phase = 0u, bempty_phase = 0u, acc_phase = 0u;
      const uint32_t a0 = smem_u32(smem + geo.off_A), b0 = smem_u32(smem + geo.off_B);
      for (int q = 0; q < nq; q++) {
        bool ok = mbar_wait(&a_full[b], (full_phase >> b) & 1u, tmo);
        full_phase ^= 1u << b;
        ok = ok && mbar_wait(&b_full[bb], (bfull_phase >> bb) & 1u, tmo);
        bfull_phase ^= 1u << bb;
        if (ok && s == 0 && jl >= 2) {
          ok = mbar_wait(&acc_empty[jl & 1], (acc_phase >> (jl & 1)) & 1u, tmo);
          acc_phase ^= 1u << (jl & 1);
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const int nkb = nbr - 8 * s < 8 ? nbr - 8 * s : 8;
        uint64_t ad = smem_desc(a0 + b * (128u * kKS), 128u, kSboA);
        uint64_t bd = smem_desc(b0 + bb * (uint32_t)NMAX * kKS, 128u, kSboA);
        const uint32_t d_t = tbase + (uint32_t)((jl & 1) * NMAX);
        const uint32_t sfa0 = tbase + kSfaCol + 8u * b, sfb0 = tbase + kSfbCol + 4u * b;
        for (int kb = 0; kb < nkb; kb++) {
          const uint32_t byte = (uint32_t)(kb & 3) << 30;
          mma_mxf8f6f4(d_t, ad, bd, idesc[kb & 3], (sfa0 + 4u * (uint32_t)(kb >> 2)) | byte,
                       (sfb0 + 2u * (uint32_t)(kb >> 2)) | byte, !(s == 0 && kb == 0));
          ad += 16u;  // +256 bytes (descriptor start address counts 16-byte units)
          bd += 16u;
        }
        tc_commit(&a_empty[b]);
        tc_commit(&b_empty[bb]);
        if (s == S - 1) tc_commit(&acc_full[jl & 1]);
        // refill the B slot of stage q-1 once its MMAs are done (stage q-1+kNB)
        if (q >= 1 && issued_b < nq) {
          const uint32_t pb = bb == 0 ? kNB - 1 : bb - 1;
          if (!mbar_wait(&b_empty[pb], (bempty_phase >> pb) & 1u, tmo)) {
            *abort_flag = 1;
            break;
          }
          bempty_phase ^= 1u << pb;
          issue_b();
          issued_b++;
        }
        b = b + 1 == kNA ? 0u : b + 1;
        bb = bb + 1 == kNB ? 0u : bb + 1;
        if (++s == S) {
          s = 0;
          if (++jl < my_jobs) {
            const uint32_t nc = (uint32_t)job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl)).ncols;
            if (nc != ncols) {
              ncols = nc;
              for (int i = 0; i < 4; i++) idesc[i] = idesc_mxf8f6f4_e2m1_e4m3(ncols, (uint32_t)i, (uint32_t)i);
            }
          }
        }
      }
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------------------- host side

static int nmax_for(int tokens_per_group) { return tokens_per_group <= 8 ? 16 : 32; }

static bool mma_fits(int nbr, int NMAX, int mode) {
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
  return mma_geom(nbr, NMAX, mode).smem <= (uint32_t)optin;
}

// The tensor-core path needs at least kPref K stages (K >= 1024), an even number of 32-blocks per
// row (16-byte aligned row starts), 16-byte aligned scales, and its buffers within shared memory.
static bool k_ok(int nbr) { return nbr >= 8 * kPref && nbr % 2 == 0; }

bool gemv_mma_supported(const MatView &w, int T) {
  return k_ok(w.nbr) && (reinterpret_cast<uintptr_t>(w.scales) & 15u) == 0 &&
         mma_fits(w.nbr, nmax_for(T < 16 ? T : 16), kModeGemv);
}

// Tokens beyond 16 run as further passes of at most 16, each with its own split of x.
size_t gemv_mma_workspace(const MatView &w, int T) {
  const int S = (w.nbr + 7) / 8, NMAX = nmax_for(T < 16 ? T : 16);
  return bsplit_group_bytes(S, NMAX) + bsf_group_words(S) * 4;
}

template <int NMAX>
static cudaError_t launch_gemv_pass(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws,
                                    cudaStream_t s) {
  const int S = (w.nbr + 7) / 8;
  uint8_t *Bg = static_cast<uint8_t *>(ws);
  uint32_t *Bsf = reinterpret_cast<uint32_t *>(Bg + bsplit_group_bytes(S, NMAX));
  const int warps = (NMAX / 2) * w.nbr;
  k_bsplit_gemv<NMAX><<<(warps + 7) / 8, 256, 0, s>>>(x, T, w.nbr * 32, Bg, Bsf);
  static unsigned long long attr = 0;
  cudaError_t e = ensure_max_dynamic_smem(k_mma<32, kModeGemv, NMAX>, attr);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = (w.rows + 127) / 128;
  MmaArgs args{};
  args.w = w;
  args.nbr = w.nbr;
  args.Bg = Bg;
  args.Bsf = Bsf;
  args.T = T;
  args.y = y;
  MoeTable<32> none{};
  k_mma<32, kModeGemv, NMAX><<<ntiles < nsm ? ntiles : nsm, kMmaThreads, mma_geom(w.nbr, NMAX, kModeGemv).smem, s>>>(
      args, none);
  return cudaGetLastError();
}

cudaError_t launch_gemv_mma(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s) {
  for (int t0 = 0; t0 < T; t0 += 16) {
    const int n = T - t0 < 16 ? T - t0 : 16;
    const uint16_t *xp = x + (size_t)t0 * w.nbr * 32;
    uint16_t *yp = y + (size_t)t0 * w.rows;
    cudaError_t e = nmax_for(T < 16 ? T : 16) == 16 ? launch_gemv_pass<16>(w, xp, n, yp, ws, s)
                                                    : launch_gemv_pass<32>(w, xp, n, yp, ws, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ----------------------------------------------------------------------------- MoE on the tensor cores

static int moe_groups_max(int E, int P, int gmax) { return (E < P ? E : P) + P / gmax + 1; }

bool moe_mma_supported(const tcf4_moe &m, int gu_seg, int dn_seg, int T) {
  if (gu_seg != 1 || dn_seg != 1) return false;
  const int nbr_gu = m.H / 32, nbr_dn = m.I / 32, NMAX = nmax_for(T);
  if (!k_ok(nbr_gu) || !k_ok(nbr_dn)) return false;
  if (((size_t)m.I * nbr_gu) % 16 != 0) return false;
  for (int e = 0; e < m.E; e++)
    if ((reinterpret_cast<uintptr_t>(m.gate_up[e].scales) | reinterpret_cast<uintptr_t>(m.down[e].scales)) & 15u)
      return false;
  return mma_fits(nbr_gu, NMAX, kModeGateUp) && mma_fits(nbr_dn, NMAX, kModeDown);
}

MoeMmaWorkspace moe_mma_workspace_layout(const tcf4_moe &m, int T, int k) {
  auto a256 = [](size_t v) { return (v + 255) & ~(size_t)255; };
  const int P = T * k, NMAX = nmax_for(T), G = moe_groups_max(m.E, P, NMAX / 2);
  const int S_gu = (m.H / 32 + 7) / 8, S_dn = (m.I / 32 + 7) / 8;
  MoeMmaWorkspace L;
  size_t off = 0;
  L.counters = off; off = a256(off + sizeof(int) * ((m.H + 127) / 128));
  L.hidden = off;   off = a256(off + sizeof(uint16_t) * (size_t)P * m.I);
  L.y = off;        off = a256(off + sizeof(float) * (size_t)P * m.H);
  L.bg_gu = off;    off = a256(off + (size_t)G * bsplit_group_bytes(S_gu, NMAX));
  L.bsf_gu = off;   off = a256(off + (size_t)G * bsf_group_words(S_gu) * 4);
  L.bg_dn = off;    off = a256(off + (size_t)G * bsplit_group_bytes(S_dn, NMAX));
  L.bsf_dn = off;   off = a256(off + (size_t)G * bsf_group_words(S_dn) * 4);
  L.total = off;
  return L;
}

template <int MAXE, int NMAX>
static cudaError_t launch_moe_mma_t(const tcf4_moe &m, const uint16_t *x, int T, const int32_t *ids,
                                    const float *wts, int k, uint16_t *out, void *ws, cudaStream_t s) {
  MoeTable<MAXE> tab;
  for (int e = 0; e < MAXE; e++) {
    const bool ok = e < m.E;
    tab.gu[e] = ok ? reinterpret_cast<const uint2 *>(m.gate_up[e].stream) : nullptr;
    tab.gus[e] = ok ? m.gate_up[e].scales : nullptr;
    tab.dn[e] = ok ? reinterpret_cast<const uint2 *>(m.down[e].stream) : nullptr;
    tab.dns[e] = ok ? m.down[e].scales : nullptr;
  }
  const MoeMmaWorkspace L = moe_mma_workspace_layout(m, T, k);
  char *base = static_cast<char *>(ws);
  MmaArgs args{};
  args.ids = ids;
  args.wts = wts;
  args.P = T * k;
  args.E = m.E;
  args.k = k;
  args.Tm = T;
  args.H = m.H;
  args.I = m.I;
  args.hidden = reinterpret_cast<uint16_t *>(base + L.hidden);
  args.yws = reinterpret_cast<float *>(base + L.y);
  args.counters = reinterpret_cast<int *>(base + L.counters);
  args.out = out;
  args.w.stream = reinterpret_cast<const uint2 *>(base);  // a valid address for zero-byte copies
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int P = T * k, G = moe_groups_max(m.E, P, NMAX / 2);

  // gate_up: split x per group (and clear the down counters), then decode + MMA + SwiGLU
  {
    uint8_t *Bg = reinterpret_cast<uint8_t *>(base + L.bg_gu);
    uint32_t *Bsf = reinterpret_cast<uint32_t *>(base + L.bsf_gu);
    const int nbr = m.H / 32;
    const int warps = G * (NMAX / 2) * nbr;
    k_bsplit_moe<NMAX><<<(warps + 7) / 8 < 4 * nsm ? (warps + 7) / 8 : 4 * nsm, 256, 0, s>>>(
        ids, P, m.E, k, x, m.H, Bg, Bsf, args.counters, (m.H + 127) / 128);
    static unsigned long long attr = 0;
    cudaError_t e = ensure_max_dynamic_smem(k_mma<MAXE, kModeGateUp, NMAX>, attr);
    if (e != cudaSuccess) return e;
    args.nbr = nbr;
    args.Bg = Bg;
    args.Bsf = Bsf;
    const int jobs = G * ((m.I + 63) / 64);
    k_mma<MAXE, kModeGateUp, NMAX><<<jobs < nsm ? jobs : nsm, kMmaThreads, mma_geom(nbr, NMAX, kModeGateUp).smem, s>>>(
        args, tab);
  }
  // down: split h per group, then decode + MMA, y to the workspace, last arriver per chunk combines
  {
    uint8_t *Bg = reinterpret_cast<uint8_t *>(base + L.bg_dn);
    uint32_t *Bsf = reinterpret_cast<uint32_t *>(base + L.bsf_dn);
    const int nbr = m.I / 32;
    const int warps = G * (NMAX / 2) * nbr;
    k_bsplit_moe<NMAX><<<(warps + 7) / 8 < 4 * nsm ? (warps + 7) / 8 : 4 * nsm, 256, 0, s>>>(
        ids, P, m.E, 1, args.hidden, m.I, Bg, Bsf, nullptr, 0);
    static unsigned long long attr = 0;
    cudaError_t e = ensure_max_dynamic_smem(k_mma<MAXE, kModeDown, NMAX>, attr);
    if (e != cudaSuccess) return e;
    args.nbr = nbr;
    args.Bg = Bg;
    args.Bsf = Bsf;
    const int jobs = G * ((m.H + 127) / 128);
    k_mma<MAXE, kModeDown, NMAX><<<jobs < nsm ? jobs : nsm, kMmaThreads, mma_geom(nbr, NMAX, kModeDown).smem, s>>>(
        args, tab);
  }
  return cudaGetLastError();
}

cudaError_t launch_moe_mma(const tcf4_moe &m, const uint16_t *x, int T, const int32_t *ids, const float *wts, int k,
                           uint16_t *out, void *ws, cudaStream_t s) {
  const bool n16 = nmax_for(T) == 16;
  if (m.E <= 32)
    return n16 ? launch_moe_mma_t<32, 16>(m, x, T, ids, wts, k, out, ws, s)
               : launch_moe_mma_t<32, 32>(m, x, T, ids, wts, k, out, ws, s);
  return n16 ? launch_moe_mma_t<256, 16>(m, x, T, ids, wts, k, out, ws, s)
             : launch_moe_mma_t<256, 32>(m, x, T, ids, wts, k, out, ws, s);
}

unsigned int take_timeouts_mma() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_tcf4_timeouts_mma, sizeof v) != cudaSuccess) return 0;
  cudaMemcpyToSymbol(g_tcf4_timeouts_mma, &zero, sizeof zero);
  return v;
}

}  // namespace tcf4
