// k_mma.cu -- fused trellis decode + block-scaled tensor-core product (tcgen05, sm_100a).
//
// HEPH abstract, first serving mode: the compressed stream stays resident and is decoded inside the
// product. The decoded weights are MXFP4 elements (E2M1 codes, one UE8M0 scale per 32 weights), so
// they feed a block-scaled kind::mxf4 MMA (K = 64 per instruction) directly as the A operand, the
// scale factors being the weights' own UE8M0 bytes. The bf16 activations are the B operand,
// written as a sum of kTerms E2M1 terms per 32-block, each term with its own UE8M0 scale (a greedy
// residual expansion, see split_terms): B column kTerms*t + j holds term j of token t, and
// y[t] = sum_j D[:, kTerms*t + j] in fp32.
//
// One persistent CTA per SM, over 128-row tiles ("jobs") of K stages of KB blocks of 32 (KB = 32 for
// up to ten tokens per group with one scale set, else 16):
//  * word loader warp: lane 0 streams each stage's trellis words (128 rows x 8 KB bytes) into a ring
//    of shared-memory slots with 2-D TMA tile loads (128-byte swizzle, no multicast).
//  * KB/2 decode warps: thread (warp w, lane l) owns tile row 32(w%4)+l and the 8 K-blocks 8(w/4)..
//    of a stage. It reads its 64 bytes of trellis words, decodes them in registers (bit-sliced) and
//    stores the blocks' E2M1 codes, packed eight per 32-bit column, into the stage's A operand in
//    TMEM (tcgen05.st into its own lane quarter); with the weights' scales in their stored layout it
//    also stores its row's scale bytes (loaded one stage ahead). The decoded weights never touch
//    shared memory. A stage's A operand is handed over in two halves (the first and last KB/2
//    blocks), each with its own barriers.
//  * B loader warp: lane 0 bulk-copies each stage's activation terms and their scale-factor tiles
//    (and, with scale tiles, the weights' tiles of the stage) into a ring of B slots, ahead of the
//    MMAs; it alone waits for the preceding kernel (the split that wrote the terms).
//  * MMA warp(s): up to 96 B rows two issuer warps, one per half stage, each into its own
//    accumulator (a double-buffered pair at 32 rows, one each at 64 and 96, as TMEM allows); at 192
//    rows one warp issues both halves. An issuer moves the stage's scale-factor tiles into TMEM with
//    tcgen05.cp, then issues its MMAs (A from TMEM, B from shared memory), released with one commit.
//  * 4 epilogue warps (one per TMEM lane quarter): the epilogue of each job (tcgen05.ld, then the
//    GEMV output, the SwiGLU of gate/up rows and its split into the down product's terms, or the MoE
//    down rows and their combine), overlapping the next job's stages where the accumulators are
//    double-buffered.
// Every wait is bounded; a wait that gives up raises a shared abort flag that the other roles see,
// and each role drains its own asynchronous copies and MMAs before the CTA frees its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "tcf4_device.cuh"
#include "tcf4_internal.h"
#include "tcf4_pipe.cuh"
#include "tcf4_tc.cuh"

namespace tcf4 {

__device__ unsigned int g_tcf4_timeouts_mma = 0;

constexpr int kTerms = 6;            // E2M1 terms per activation block
constexpr int kMapSlots = 8;         // per-CTA tensor-map slots of the grouped MoE (> jobs in flight)

constexpr int kSplitThreads = 128;  // activation-split CTAs (see k_bsplit_gemv)

// Sleep between barrier tests of the idle roles. The loaders run stages ahead and the MMA issuers
// have about two stages (~3 us) of slack, so these only bound how soon a completed phase is seen.
constexpr uint32_t kLoaderSleepNs = 200u, kMmaSleepNs = 100u, kEpiSleepNs = 200u;

enum MmaMode { kModeGemv = 0, kModeGateUp = 1, kModeDown = 2 };

// Register split of the NMAX = 32 decode GEMV (see k_mma): registers per thread at launch, of the
// decode warps and of the other warps after the split.
constexpr int kRsLaunchRegs = 80, kRsDecRegs = 96, kRsOtherRegs = 48;

// SETS: sets of UE8M0 scale factors of the weights per block (1; 4 for E5M3 block scales, whose
// significand bits each get a power-of-two set, see k_mma). Four sets need the 16-block stages.
template <int NMAX, int SETS = 1>
struct Cfg {
  static_assert(NMAX <= 256, "B rows of one MMA");
  static_assert(SETS == 1 || SETS == 4, "one or four scale sets");
  static constexpr int kTok = NMAX / kTerms;                   // tokens per group
  static constexpr int kSlots = (NMAX + kTerms - 1) / kTerms;  // token slots the split writes
  static constexpr int kSplitNT = kTok <= 6 ? kTok : 4;        // slots split side by side
  static constexpr int kC = (NMAX + 31) / 32;                  // B scale columns per 4-block group
  static constexpr int kNTile = (kC + 3) / 4;                  // 32 x 16-byte B scale tiles per group
  static constexpr uint32_t kSfbGCols = 4u * kNTile;           // TMEM columns of a group's B scales
  static constexpr int kKB = NMAX <= 64 && SETS == 1 ? 32 : 16;  // 32-blocks per row per stage
  // Warps: kDecWarps decode warps (four per group of 8 blocks of a stage), then the word loader, two
  // MMA issuer slots, the B loader and four epilogue warps.
  static constexpr int kDecWarps = kKB / 2;
  static constexpr int kWLoadWarp = kDecWarps, kMmaWarp = kDecWarps + 1, kBLoadWarp = kDecWarps + 3;
  static constexpr int kEpiWarp0 = kDecWarps + 4, kThreads = 32 * (kDecWarps + 8);
  static constexpr int kNBT = 8;                               // blocks per decode thread per stage
  static constexpr int kNG = kNBT / 4;                         // scale groups per decode thread
  static constexpr int kNW = kKB == 32 ? 3 : (NMAX > 96 ? 5 : 6);  // word stages in flight
  static constexpr int kNA = NMAX <= 64 || SETS > 1 ? 2 : (NMAX > 96 ? 2 : 3);  // A / scale-factor stages (TMEM)
  static constexpr int kNB = NMAX > 96 ? 2 : (NMAX > 32 && NMAX <= 64 ? 3 : 4);  // B stages (shared memory)
  static constexpr int kBoxCols = kKB / 16;                    // 128-byte TMA boxes per 64 rows
  static constexpr uint32_t kWStage = 1024u * kKB;             // 128 rows x 8 KB bytes of words
  static constexpr uint32_t kSbo = 128u * kKB;                 // B: 8 rows x KB chunks x 16 bytes
  static constexpr uint32_t kBStage = NMAX * 16u * kKB;        // NMAX rows x 32 KB E2M1
  // B scale factors of a stage: per 4-block group kNTile tiles of 32 x 16 bytes, row r of tile i =
  // the group's UE8M0 words of B rows 128 i + r, 128 i + 32 + r, ... (spare words past NMAX), the
  // sources of kNTile tcgen05.cp
  static constexpr uint32_t kSfbStage = (kKB / 4) * 512u * kNTile;
  static constexpr uint32_t kBSlot = kBStage + kSfbStage;       // one stage of terms + scales
  // Weights' scales as scale tiles (trellis_gemv_tiled): per 4-block group a 512-byte tile, row r
  // = the group's UE8M0 words of tile rows r, 32 + r, 64 + r, 96 + r; KB/4 tiles per stage.
  static constexpr uint32_t kSfaTile = (kKB / 4) * 512u;
  // MMA issuers: one per half stage, each into its own accumulator, up to 96 B rows (one issuing
  // thread sustains about one MMA per 60 cycles, two in different warps run concurrently, and a
  // single issuer's instructions slow the decode warps of its sub-partition).
  static constexpr int kNI = NMAX <= 96 ? 2 : 1;
  // accumulators per issuer: two (a job's epilogue overlaps the next job's MMAs) at 32 B rows; one
  // each above, so that both issuers fit (at 64 rows: 2 x 64 + 256 A + 64 + 64 scale columns = 512)
  static constexpr int kNAcc = NMAX > 32 ? 1 : 2;
  static constexpr uint32_t kACols = 4u * kKB;                 // TMEM columns of a stage's A
  static constexpr uint32_t kSfbCols = (kKB / 4) * kSfbGCols;  // TMEM columns of a stage's B scales
  static constexpr uint32_t kACol = kNAcc * kNI * NMAX;        // TMEM: accumulators first, then
  static constexpr uint32_t kSfaCol = kACol + kACols * kNA;    // A stages, A scales (KB columns per
  static constexpr uint32_t kSfbCol = kSfaCol + SETS * kKB * kNA;  // stage and set), B scales
  static constexpr uint32_t kUsed = kSfbCol + kSfbCols * kNA;     // (kSfbCols per stage)
  static constexpr uint32_t kTmemCols = kUsed <= 128 ? 128 : (kUsed <= 256 ? 256 : 512);
  static_assert(kUsed <= 512, "TMEM budget");
  // Resident-MXFP4 source (the expanded tensor): the A operand is a shared-memory tile of nibbles
  // (128 rows x 16 KB bytes, 128-byte-swizzled TMA boxes) and TMEM holds only the accumulators and
  // the scale factors.
  static constexpr int kNWX = NMAX <= 32 ? 2 : 3;              // A-tile stages in flight
  static constexpr uint32_t kWStageX = 2048u * kKB;
  static constexpr uint32_t kSfaColX = kNAcc * kNI * NMAX;
  static constexpr uint32_t kSfbColX = kSfaColX + kKB * kNA;
  static constexpr uint32_t kUsedX = kSfbColX + kSfbCols * kNA;
  static constexpr uint32_t kTmemColsX = kUsedX <= 128 ? 128 : (kUsedX <= 256 ? 256 : 512);
  static_assert(kUsedX <= 512, "TMEM budget");
};

// Position (0..31) inside a 32-element chunk of the MMA operand of weight i of the block: the
// decoder's interleaved nibble words put weight 4v+j in nibble v of word j, and word j fills bytes
// 4j..4j+3 of the chunk (element 2b in the low nibble of byte b).
__host__ __device__ constexpr int kpos_of_weight(int i) { return 8 * (i & 3) + (i >> 2); }

// Byte offset of chunk c (0..KB-1) of row n in a K-major, no-swizzle B stage: core matrices of 8
// rows x 16 bytes, LBO = 128 (adjacent chunks), SBO = 128 KB (adjacent 8-row groups). In TMEM the A
// operand holds the same 16-byte chunks, four 32-bit columns each (element e of a column in bits
// 4e..4e+3).
template <int NMAX, int SETS = 1>
__host__ __device__ constexpr uint32_t chunk_off(uint32_t n, uint32_t c) {
  return (n >> 3) * Cfg<NMAX, SETS>::kSbo + c * 128u + (n & 7u) * 16u;
}

// ------------------------------------------------------------------------------- routing groups
// MoE work is split into groups: an active expert with its routed pairs, at most gmax per group.
struct GroupPlan {
  int cnt[kMaxExperts];
  int off[kMaxExperts];
  int list[kMaxTokens * kMaxTopK];  // pairs p = t*k + j per expert, in p order
  int ids[kMaxTokens * kMaxTopK];
  int g_e[kMaxTokens * kMaxTopK];   // expert of group g
  int g_first[kMaxTokens * kMaxTopK];
  int g_cnt[kMaxTokens * kMaxTopK];
  int n_groups;
};

// All threads of the CTA. Pairs whose expert id is outside [0, E) are dropped. Deterministic: groups
// in expert order, the pairs of an expert in p order. The offsets come from one warp's prefix sum
// over the experts (eight per lane), not a serial walk, so the plan costs little more than the load
// of the routing ids.
__device__ void build_groups(GroupPlan &pl, const int32_t *__restrict__ ids, int P, int E, int gmax) {
  static_assert(kMaxExperts == 8 * 32, "eight experts per lane of the planning warp");
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) pl.cnt[e] = 0;
  for (int p = tid; p < P; p += blockDim.x) pl.ids[p] = ids[p];
  __syncthreads();
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = pl.ids[p];
    if (e >= 0 && e < E) atomicAdd(&pl.cnt[e], 1);
  }
  __syncthreads();
  if (tid < 32) {
    int c[8], cs = 0, gs = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const int e = 8 * tid + i;
      c[i] = e < E ? pl.cnt[e] : 0;
      cs += c[i];
      gs += (c[i] + gmax - 1) / gmax;
    }
    // exclusive prefix sums over the lanes
    int ci = cs, gi = gs;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int cu = __shfl_up_sync(0xffffffffu, ci, o), gu = __shfl_up_sync(0xffffffffu, gi, o);
      if (tid >= o) {
        ci += cu;
        gi += gu;
      }
    }
    int o = ci - cs, ng = gi - gs;
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const int e = 8 * tid + i;
      if (e < E) pl.off[e] = o;
      for (int f = 0; f < c[i]; f += gmax) {
        pl.g_e[ng] = e;
        pl.g_first[ng] = o + f;
        pl.g_cnt[ng] = c[i] - f < gmax ? c[i] - f : gmax;
        ng++;
      }
      o += c[i];
    }
    if (tid == 31) pl.n_groups = ng;
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

// ------------------------------------------------------------------------------- activation terms
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// fp32 -> E2M1 code (round to nearest even, saturating at +-6).
__device__ __forceinline__ uint32_t to_e2m1(float v) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(0.f), "f"(v));
  return r & 15u;
}

// E2M1 code (low nibble) -> value, exact (every E2M1 value is a binary16 value).
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  uint32_t h2;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h2) : "r"(c & 15u));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// 2^e for e in [-127, 127], exact.
__device__ __forceinline__ float pow2f(int e) {
  return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// Per group of token slots, the activation terms of each stage, stage after stage ([S][kBSlot]):
// the K-major E2M1 B operand (kBStage bytes), then its scale factors: for each 4-block group g a
// 512-byte tile whose 16-byte row r holds, at word c, the UE8M0 bytes of B row 32c + r for the
// stage's blocks 4g..4g+3 (byte i = block 4g+i). One tcgen05.cp (32x128b, copied to all four lane
// quarters) moves a group's tile to TMEM, where B row 32c + r reads column c of the group.
template <int NMAX, int SETS = 1>
__host__ __device__ inline size_t terms_bytes(int S) {
  return (size_t)S * Cfg<NMAX, SETS>::kBSlot;
}

// One 32-element block kb of NT activation rows (lane = element; v[i] is slot t0 + i) -> kTerms
// E2M1 terms each with UE8M0 scales, written as B rows kTerms*t .. kTerms*t+kTerms-1 of the
// group's terms (layout above). Term j: with m the largest |residual| of the block, scale 2^S with
// S = ceil(log2(m / 6)) puts the block in (3, 6]; each residual is rounded to the E2M1 grid
// (nearest even) and the rounded value removed (exactly: Sterbenz). The largest residual shrinks
// by at least 5x per term, so after kTerms terms |x - sum| <= 5^-6 max|x| over the block.
// The NT slots are split side by side (their dependent chains overlap); slots at or past `nvalid`
// are computed but not stored.
// NAT: natural K order within a block (the MXFP4 tensor's), else the decoder's interleaved order.
template <int NMAX, bool NAT, int NT, int SETS = 1>
__device__ __forceinline__ void split_terms_n(const float *v, int t0, int nvalid, int kb, int S_total,
                                              uint8_t *terms) {
  using C = Cfg<NMAX, SETS>;
  const int lane = threadIdx.x & 31;
  const int s = kb / C::kKB, c = kb - s * C::kKB, h = c >> 2;
  (void)S_total;
  uint8_t *bst = terms + (size_t)s * C::kBSlot;
  uint8_t *sfs = bst + C::kBStage;
  const int kp = NAT ? lane : kpos_of_weight(lane);
  float r[NT];
#pragma unroll
  for (int i = 0; i < NT; i++) r[i] = v[i];
#pragma unroll
  for (int j = 0; j < kTerms; j++) {
    uint32_t code[NT];
    int S[NT];
#pragma unroll
    for (int i = 0; i < NT; i++) {
      // the largest |residual|: for non-negative floats the bit patterns order as the values do
      const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(r[i])));
      // S from m's exponent field: m = 1.f * 2^e, and m / 2^e <= 1.5 iff the fraction <= 0.5.
      // A subnormal or zero m gives S = -127. S <= 126 for any finite m (max|bf16| < 2^128).
      const int e = (int)(mb >> 23) - 127;
      int Si = (mb >> 23) == 0u ? -127 : ((mb & 0x7FFFFFu) <= 0x400000u ? e - 2 : e - 1);
      S[i] = Si < -127 ? -127 : Si;
      code[i] = to_e2m1(r[i] * pow2f(-S[i]));
      r[i] -= e2m1_value(code[i]) * pow2f(S[i]);
    }
#pragma unroll
    for (int i = 0; i < NT; i++) {
      // the element sharing this one's byte: K positions kp and kp ^ 1
      const uint32_t partner = __shfl_xor_sync(0xffffffffu, code[i], NAT ? 1 : 4);
      const int n = kTerms * (t0 + i) + j;
      if (t0 + i < nvalid && n < NMAX) {
        if ((kp & 1) == 0)
          bst[chunk_off<NMAX, SETS>((uint32_t)n, (uint32_t)c) + (kp >> 1)] = (uint8_t)(code[i] | (partner << 4));
        if (lane == 0)
          sfs[((h * C::kNTile + (n >> 7)) * 32 + (n & 31)) * 16 + ((n >> 5) & 3) * 4 + (c & 3)] = (uint8_t)(S[i] + 127);
      }
    }
  }
}

template <int NMAX, bool NAT = false, int SETS = 1>
__device__ __forceinline__ void split_terms(float v, int t, int kb, int S_total, uint8_t *terms) {
  split_terms_n<NMAX, NAT, 1, SETS>(&v, t, t + 1, kb, S_total, terms);
}

// Plain GEMV: one group, token slots 0..T-1. The B rows of the other slots are not written: an MMA
// column depends only on its own B row (and its scale), and no output reads those columns.
// The GEMV's product kernel is launched as a programmatic dependent of this split, released before
// the split's own grid-dependency wait: it starts its TMEM setup, weight tiles and first decodes
// (none of which depend on the split or on the kernels before it) while the preceding kernel still
// runs, and waits for the split's completion only before it reads the activation terms. (The
// library's kernels that write weights release no dependents early, so a product kernel launched
// after one of them finds its weights complete.) CTAs of 128 threads with at most
// 32 registers each (4096) fit beside a resident product CTA (768 threads x 80 registers = 61440 of
// the SM's 65536): the split of the next call can wait on its grid dependency on any SM while the
// current product kernel runs, and it never keeps a product CTA from starting.
template <int NMAX, bool NAT, int SETS = 1>
__global__ void __launch_bounds__(kSplitThreads, 65536 / (32 * kSplitThreads)) k_bsplit_gemv(const uint16_t *__restrict__ x, int T, int K,
                                                     uint8_t *__restrict__ terms) {
  grid_dep_release();  // the product kernel may start; it waits for this grid before reading terms
  grid_dep_wait();     // x may come from, and terms may still be read by, the preceding kernel
  const int nb = K >> 5, S = (nb + Cfg<NMAX, SETS>::kKB - 1) / Cfg<NMAX, SETS>::kKB, lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int wi = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; wi < T * nb; wi += nwarps) {
    const int t = wi / nb, kb = wi - t * nb;
    split_terms<NMAX, NAT, SETS>(__uint_as_float((uint32_t)x[(size_t)t * K + kb * 32 + lane] << 16), t, kb, S,
                                 terms);
  }
}

// MoE: group g's token slot i is pair list[g_first + i]; its activation row is src[pair / div]
// (rows of tokens: div = k, as for x before gate/up; rows of pairs: div = 1). Only the slots that
// hold a pair are split (the B rows of empty slots feed MMA columns nothing reads). The down
// product's terms do not come from here: the gate/up epilogue writes them. Block 0 also clears the
// down kernel's counters when `counters` is given. CTAs of 128 threads with at most 32 registers, so
// that they fit beside a resident product CTA (as k_bsplit_gemv's).
template <int NMAX, bool NAT>
__global__ void __launch_bounds__(kSplitThreads, 65536 / (32 * kSplitThreads)) k_bsplit_moe(const int32_t *__restrict__ ids, int P, int E, int div,
                                                    const uint16_t *__restrict__ src, int K, uint8_t *__restrict__ terms,
                                                    int *__restrict__ counters, int n_counters) {
  __shared__ GroupPlan pl;
  grid_dep_wait();  // every input (routing, x or h) and the workspace come from preceding kernels
  grid_dep_release();
  if (counters != nullptr && blockIdx.x == 0)
    for (int c = threadIdx.x; c < n_counters; c += blockDim.x) counters[c] = 0;
  build_groups(pl, ids, P, E, Cfg<NMAX>::kTok);
  const int nb = K >> 5, S = (nb + Cfg<NMAX>::kKB - 1) / Cfg<NMAX>::kKB;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  // the routed pairs in list order: entry i belongs to the group g with g_first[g] <= i (groups are
  // consecutive runs of the list, in order), as slot i - g_first[g]
  const int npairs = pl.n_groups > 0 ? pl.g_first[pl.n_groups - 1] + pl.g_cnt[pl.n_groups - 1] : 0;
  for (int wi = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; wi < npairs * nb; wi += nwarps) {
    const int i = wi / nb, kb = wi - i * nb;
    int lo = 0, hi = pl.n_groups - 1;  // the last group whose first entry is <= i
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pl.g_first[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const int row = pl.list[i] / div;
    split_terms<NMAX, NAT>(__uint_as_float((uint32_t)src[(size_t)row * K + kb * 32 + lane] << 16), i - pl.g_first[lo],
                           kb, S, terms + (size_t)lo * terms_bytes<NMAX>(S));
  }
}

// ------------------------------------------------------------------------------- geometry

// Shared memory: barriers + tensor-map copy | word ring | B ring (with the weights' scale tiles
// when tiled) | gate/up exchange | group plan.
struct MmaGeom {
  uint32_t off_W, off_B, bslot, off_U, off_P, smem;
};

template <int NMAX, int SETS = 1>
__host__ __device__ inline MmaGeom mma_geom(int mode, bool mx = false, bool tiled = false) {
  using C = Cfg<NMAX, SETS>;
  MmaGeom g;
  g.off_W = 1024u;
  g.off_B = g.off_W + (mx ? C::kNWX * C::kWStageX : C::kNW * C::kWStage);
  g.bslot = C::kBSlot + (tiled ? C::kSfaTile : 0u);
  g.off_U = g.off_B + C::kNB * g.bslot;
  g.off_P = g.off_U + (mode == kModeGateUp ? 2u * 64u * (uint32_t)C::kTok * 4u : 0u);
  g.smem = g.off_P + (mode == kModeGemv ? 0u : round_up((uint32_t)sizeof(GroupPlan), 128u));
  return g;
}

// ------------------------------------------------------------------------------- instructions

__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// One arrival on `bar` for the whole (converged) warp, from one elected lane; no branch.
__device__ __forceinline__ void mbar_arrive_one(uint64_t *bar) {
  asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Non-blocking test of a barrier phase (1 once the phase with the given parity has completed). Its
// result is read later, so the test's latency overlaps other work.
__device__ __forceinline__ uint32_t mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok;
}

// Bounded wait for a warp that has nothing else to do meanwhile (loaders, MMA issuers, the epilogue's
// poller): it tests the barrier and sleeps about `ns` nanoseconds between tests. (A blocking try_wait
// returns every few tens of nanoseconds while it waits, and the polls of several idle warps take
// issue slots from the decode warps on the same SM sub-partitions.)
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t *bar, uint32_t parity, unsigned int *timeouts, uint32_t ns) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  do {
    __nanosleep(ns);
    if (mbar_test(bar, parity)) return true;
  } while (clock64() - t0 < kWaitCycles);
  atomicAdd(timeouts, 1u);
  return false;
}

// Bounded wait executed by the whole warp (one poll instruction serves all lanes; the result is made
// warp-uniform). The shared abort flag is read only on the slow path, so a wait that succeeds at
// once costs a poll and a vote.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, unsigned int *timeouts,
                                          volatile int *abort_flag) {
  bool ok = mbar_try_wait(bar, parity);
  if (!__all_sync(0xffffffffu, ok)) {
    const long long t0 = clock64();
    ok = false;
    while (!ok && !*abort_flag && clock64() - t0 < kWaitCycles) ok = mbar_try_wait(bar, parity);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && (threadIdx.x & 31) == 0 && !*abort_flag) atomicAdd(timeouts, 1u);
  }
  return ok;
}

// True in exactly one active lane of the warp.
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}" : "=r"(e));
  return e != 0;
}

// 2-D TMA tile load (no multicast; the tensor map covers this GPU's memory only).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Warp-wide stores of one / four consecutive TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_st_x1(uint32_t taddr, uint32_t a) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(a) : "memory");
}

template <int NBT>
__device__ __forceinline__ void tmem_st_codes(uint32_t taddr, const uint32_t (&r)[NBT][4]);

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&r)[4][4]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0][0]), "r"(r[0][1]), "r"(r[0][2]), "r"(r[0][3]), "r"(r[1][0]), "r"(r[1][1]), "r"(r[1][2]), "r"(r[1][3]),
      "r"(r[2][0]), "r"(r[2][1]), "r"(r[2][2]), "r"(r[2][3]), "r"(r[3][0]), "r"(r[3][1]), "r"(r[3][2]), "r"(r[3][3])
      : "memory");
}

__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t (&r)[8][4]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0][0]), "r"(r[0][1]), "r"(r[0][2]), "r"(r[0][3]),
      "r"(r[1][0]), "r"(r[1][1]), "r"(r[1][2]), "r"(r[1][3]),
      "r"(r[2][0]), "r"(r[2][1]), "r"(r[2][2]), "r"(r[2][3]),
      "r"(r[3][0]), "r"(r[3][1]), "r"(r[3][2]), "r"(r[3][3]),
      "r"(r[4][0]), "r"(r[4][1]), "r"(r[4][2]), "r"(r[4][3]),
      "r"(r[5][0]), "r"(r[5][1]), "r"(r[5][2]), "r"(r[5][3]),
      "r"(r[6][0]), "r"(r[6][1]), "r"(r[6][2]), "r"(r[6][3]),
      "r"(r[7][0]), "r"(r[7][1]), "r"(r[7][2]), "r"(r[7][3])
      : "memory");
}

template <>
__device__ __forceinline__ void tmem_st_codes<4>(uint32_t taddr, const uint32_t (&r)[4][4]) {
  tmem_st_x16(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_st_codes<8>(uint32_t taddr, const uint32_t (&r)[8][4]) {
  tmem_st_x32(taddr, r);
}

// Instruction descriptor of a block-scaled kind::mxf4 MMA: A = B = E2M1, K-major, UE8M0 scales per
// 32, fp32 accumulation, M = 128, N columns; sf = scale-factor byte pair (0 or 2) of both operands.
__device__ __forceinline__ uint32_t idesc_mxf4(uint32_t N, uint32_t sf) {
  uint32_t d = 0;
  d |= (sf & 3u) << 4;     // B scale-factor id
  d |= 1u << 7;            // A format: E2M1
  d |= 1u << 10;           // B format: E2M1
  d |= (N >> 3) << 17;     // N / 8
  d |= 1u << 23;           // scale format: UE8M0
  d |= (128u >> 4) << 24;  // M / 16
  d |= (sf & 3u) << 29;    // A scale-factor id
  return d;                // bit 31 = 0: K = 64
}

// One thread: D[tmem] (+)= A[tmem] x B[smem], block-scaled. The A scale factors of rows
// 32q..32q+31 are read from lane quarter q at column sfa+q, those of B row n from column sfb + n/32.
__device__ __forceinline__ void mma_mxf4_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], [%1], %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// A 64-bit descriptor from its two words (a register pair, no instruction).
__device__ __forceinline__ uint64_t desc_of(uint32_t lo, uint32_t hi) { return ((uint64_t)hi << 32) | lo; }

// One thread: copy a 32-row x 16-byte shared-memory tile (descriptor desc) into TMEM columns
// taddr..taddr+3 of every lane quarter: row r to lane 32q + r of each quarter q.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

// The same MMA with A from shared memory (descriptor a_desc).
__device__ __forceinline__ void mma_mxf4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Shared-memory descriptor of a K-major operand tile in the 128-byte-swizzled layout a SWIZZLE_128B
// TMA box of 128-byte rows produces (layout type 2; SBO = 1 KB between 8-row groups; LBO unused).
// A K step of 64 E2M1 elements (32 bytes) inside the 128-byte swizzle row advances the start
// address by 32 bytes.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;  // descriptor version for tcgen05
  d |= (uint64_t)2u << 61;  // SWIZZLE_128B
  return d;
}

// Per-job tensor maps of the grouped MoE: lane 0 rewrites the global address of the shared-memory
// copy, then the whole warp publishes it to the CTA's global slot for the TMA unit.
__device__ __forceinline__ void tmap_set_address(uint32_t smap, const void *addr) {
  asm volatile("tensormap.replace.tile.global_address.shared::cta.b1024.b64 [%0], %1;" ::"r"(smap), "l"(addr)
               : "memory");
}
__device__ __forceinline__ void tmap_publish(void *gmap, uint32_t smap) {
  asm volatile(
      "tensormap.cp_fenceproxy.global.shared::cta.tensormap::generic.release.gpu.sync.aligned [%0], [%1], "
      "128;" ::"l"(gmap),
      "r"(smap)
      : "memory");
}
__device__ __forceinline__ void tmap_acquire(const void *gmap) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(gmap) : "memory");
}

// The UE8M0 scale sets of four E5M3 block-scale bytes (one per byte of w, each byte on its own, no
// carries between bytes): for exponent field e and significand bits m2 m1 m0, set 0 holds
// 2^(e-15) (e + 112; 0, i.e. 2^-127, when e = 0; 0xFF, NaN, when e = 31) and set k = 1, 2, 3 holds
// 2^(max(e,1) - 15 - k) when significand bit 3 - k is set, else 0 (2^-127). The sum over the sets
// is the E5M3 value 2^(e-15) (1 + m/8), or m 2^-17 when e = 0.
__device__ __forceinline__ void e5m3_scale_sets(uint32_t w, uint32_t (&st)[4]) {
  const uint32_t e = (w >> 3) & 0x1F1F1F1Fu, m = w & 0x07070707u;
  const uint32_t nz = ((e + 0x7F7F7F7Fu) & 0x80808080u) >> 7;   // 1 in the bytes with e >= 1
  const uint32_t nan = ((e + 0x61616161u) & 0x80808080u) >> 7;  // 1 in the bytes with e == 31
  const uint32_t ee = e | (nz ^ 0x01010101u);                   // max(e, 1)
  st[0] = ((e + 0x70707070u) & (nz * 0xFFu)) | (nan * 0xFFu);
  st[1] = (ee + 0x6F6F6F6Fu) & (((m >> 2) & 0x01010101u) * 0xFFu);
  st[2] = (ee + 0x6E6E6E6Eu) & (((m >> 1) & 0x01010101u) * 0xFFu);
  st[3] = (ee + 0x6D6D6D6Du) & ((m & 0x01010101u) * 0xFFu);
}

// ------------------------------------------------------------------------------- kernel arguments

struct MmaArgs {
  const uint2 *stream;    // GEMV: the matrix's stream words (MoE: from the table)
  int seg_blocks;         // trellis segment length in 32-blocks (carry path: > 1)
  const uint8_t *scales;  // GEMV: the matrix's scales (MoE: from the table)
  int rows;               // GEMV rows
  int nbr;                // 32-blocks per row (K / 32)
  const uint8_t *terms;   // activation terms, per group (terms_bytes each)
  int T;                  // GEMV tokens
  uint16_t *y;            // GEMV out [T][rows]
  const int32_t *ids;     // MoE routing [T][k]
  const float *wts;
  int P, E, k, Tm, H, I;
  uint16_t *hidden;       // [P][I] bf16
  uint8_t *terms_dn;      // gate/up: the down kernel's activation terms, written by its epilogue
  float *yws;             // [P][H] fp32
  int *counters;          // 4 per 128-row chunk of H
  uint16_t *out;          // [T][H] bf16
  unsigned char *maps;    // MoE: per-CTA tensor-map slots [gridDim][kMapSlots][128]
  const uint8_t *sf_tiles;  // tiled GEMV: the weights' scale tiles, sf_groups 512-byte tiles per 128-row tile
  int sf_groups;
};

// A job is one 128-row tile: tile rows [0, 64) are matrix rows y0.., tile rows [64, 128) matrix
// rows y1..; na / nb of them valid. Activation group `group`, MMA width ncols; `cnt` tokens
// starting at list index `first`.
struct JobRows {
  const void *st;     // the matrix stream (MoE: the tensor map's address)
  const uint8_t *sc;  // its scales
  int y0, y1, na, nb, group, ncols, row0, chunk, cnt, first;
};

template <int MAXE, int MODE, int NMAX>
__device__ __forceinline__ JobRows job_rows(const MmaArgs &a, const MoeTable<MAXE> &tab, const GroupPlan *pl,
                                            int job) {
  JobRows j;
  if (MODE == kModeGemv) {
    const int r0 = job * 128;
    j.st = a.stream;
    j.sc = a.scales;
    j.y0 = r0;
    j.y1 = r0 + 64;
    j.na = a.rows - r0 < 64 ? a.rows - r0 : 64;
    j.nb = a.rows - r0 - 64 < 0 ? 0 : (a.rows - r0 - 64 < 64 ? a.rows - r0 - 64 : 64);
    j.group = 0;
    j.cnt = a.T;
    j.first = 0;
    j.row0 = r0;
    j.chunk = job;
  } else if (MODE == kModeGateUp) {
    const int nch = (a.I + 63) / 64;
    const int g = job / nch, c = job - g * nch, e = pl->g_e[g];
    const int i0 = 64 * c;
    j.st = tab.gu[e];
    j.sc = tab.gus[e];
    j.y0 = i0;
    j.y1 = a.I + i0;
    j.na = j.nb = a.I - i0 < 64 ? a.I - i0 : 64;
    j.group = g;
    j.cnt = pl->g_cnt[g];
    j.first = pl->g_first[g];
    j.row0 = i0;
    j.chunk = c;
  } else {
    const int nch = (a.H + 127) / 128;
    const int g = job / nch, c = job - g * nch, e = pl->g_e[g];
    const int n0 = 128 * c;
    j.st = tab.dn[e];
    j.sc = tab.dns[e];
    j.y0 = n0;
    j.y1 = n0 + 64;
    j.na = a.H - n0 < 64 ? a.H - n0 : 64;
    j.nb = a.H - n0 - 64 < 0 ? 0 : (a.H - n0 - 64 < 64 ? a.H - n0 - 64 : 64);
    j.group = g;
    j.cnt = pl->g_cnt[g];
    j.first = pl->g_first[g];
    j.row0 = n0;
    j.chunk = c;
  }
  j.ncols = (kTerms * j.cnt + 15) / 16 * 16;
  return j;
}

// Matrix row of tile row m (0..127), or -1 when the row is outside the tile's valid rows.
__device__ __forceinline__ int tile_row(const JobRows &j, int m) {
  return m < 64 ? (m < j.na ? j.y0 + m : -1) : (m - 64 < j.nb ? j.y1 + m - 64 : -1);
}

// ------------------------------------------------------------------------------- the kernel

// MX: the weights are a resident MXFP4 tensor (nibbles [rows][K/2], scales [rows][K/32]) instead of a
// trellis stream; the word loader then brings 128-byte-swizzled nibble tiles that the MMAs read as
// the A operand straight from shared memory, and four scale-factor warps replace the decode warps.
// CARRY: trellis segments longer than a block (seg_len = 32 * seg_blocks): each block's state
// continues from the previous block of its segment.
// RS: register split. The launch gives every thread the same registers (768 threads x 80 = 61440
// at NMAX = 32); the decode warps, which carry eight blocks' words and codes, take 96 each and the
// eight other warps give theirs down to 48 (16 x 32 x 96 + 8 x 32 x 48 = 61440). Launched only after
// the host has checked that the compiled kernel's registers cover that sum, since a larger request
// than the launch holds would never be granted.
// TILED (plain GEMV only): the weights' scales come as scale tiles; the B loader bulk-copies each
// stage's tiles into its B slot (after the activation terms) and the MMA issuers move them to TMEM
// with tcgen05.cp, so the decode warps handle no scale factors at all. (In the B ring they are
// released with the stage's MMAs; a ring of their own beside the word ring held back the word
// loads, whose slots free up earlier.)
// SETS = 4: the weights' scale bytes are E5M3 block scales ("XOR-Trellis" news page, its grouping
// format), read as s = 2^(e-15) (1 + m/8) (subnormal below e = 1). Such a scale is the sum of at
// most four powers of two, 2^(e-15) for the implicit bit and 2^(e-16), 2^(e-17), 2^(e-18) for the
// significand bits that are set, so the product of a block is four block-scaled MMAs of the same A
// and B, one per power, summed in the accumulator; an absent power takes the smallest UE8M0 scale
// 2^-127 (its contribution is below 2^-124 of |x| per weight) and a NaN scale (e = 31) gives NaN.
template <int MAXE, int MODE, int NMAX, bool MX, bool CARRY, bool RS = false, bool TILED = false, int SETS = 1>
__global__ void __launch_bounds__(Cfg<NMAX, SETS>::kThreads, 1) k_mma(const __grid_constant__ MmaArgs a,
                                                           const __grid_constant__ MoeTable<MAXE> tab,
                                                           const __grid_constant__ CUtensorMap wmap) {
  using C = Cfg<NMAX, SETS>;
  constexpr int kNW = MX ? C::kNWX : C::kNW, kNA = C::kNA, kKB = C::kKB, kNBT = C::kNBT, kNG = C::kNG;
  constexpr uint32_t kWStage = MX ? C::kWStageX : C::kWStage;
  constexpr uint32_t kSfaCol = MX ? C::kSfaColX : C::kSfaCol, kSfbCol = MX ? C::kSfbColX : C::kSfbCol;
  constexpr uint32_t kTmemCols = MX ? C::kTmemColsX : C::kTmemCols;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbr = a.nbr, S = (nbr + kKB - 1) / kKB;
  static_assert(!TILED || (MODE == kModeGemv && !MX), "scale tiles: plain decode GEMV only");
  static_assert(SETS == 1 || (MODE == kModeGemv && !MX && !TILED), "E5M3 scale sets: plain decode GEMV only");
  const MmaGeom geo = mma_geom<NMAX, SETS>(MODE, MX, TILED);
  static_assert((MX ? 2 * kNW : kNW) <= 8 && kNA <= 4 && C::kNB <= 4,
                "barrier block: 8 word slots, 4 A and 4 B slots");
  // 49 barriers in bytes [0, 392). The A operand of a stage is filled and released in two halves
  // (blocks [0, KB/2) and [KB/2, KB), each by half of the decode warps): barrier 2 b + half. With
  // MX the word slots are also split in halves (barrier 2 ws + half), each released by its MMAs.
  uint64_t *w_full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *w_empty = w_full + 8, *a_full = w_full + 16, *a_empty = w_full + 24, *b_full = w_full + 32,
           *b_empty = w_full + 36, *acc_full = w_full + 40, *acc_empty = w_full + 42, *u_full = w_full + 44,
           *u_empty = w_full + 46, *drain = w_full + 48;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 448);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + 452);
  unsigned char *smap = smem + 512;  // shared-memory copy of the tensor map (grouped MoE)
  unsigned int *tmo = &g_tcf4_timeouts_mma;
  GroupPlan *pl = reinterpret_cast<GroupPlan *>(smem + geo.off_P);
  const size_t tbytes = terms_bytes<NMAX, SETS>(S);

  if (tid == 0) {
    for (int i = 0; i < (MX ? 2 * kNW : kNW); i++) {
      mbar_init(&w_full[i], 1);
      mbar_init(&w_empty[i], MX ? 1 : C::kDecWarps);
    }
    for (int i = 0; i < kNA; i++) {
      for (int hh = 0; hh < 2; hh++) {
        mbar_init(&a_full[2 * i + hh], MX ? 4 : C::kDecWarps / 2);
        mbar_init(&a_empty[2 * i + hh], 1);
      }
    }
    for (int i = 0; i < C::kNB; i++) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], C::kNI);  // every issuer releases the slot after its MMAs of the stage
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(&acc_full[i], C::kNI);
      mbar_init(&acc_empty[i], 4);
      mbar_init(&u_full[i], 2);
      mbar_init(&u_empty[i], 2);
    }
    mbar_init(drain, C::kNI);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (MODE != kModeGemv && tid < 32)
    reinterpret_cast<uint32_t *>(smap)[tid] = reinterpret_cast<const uint32_t *>(&wmap)[tid];
  if (warp == C::kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  int njobs;
  if (MODE == kModeGemv) {
    njobs = (a.rows + 127) >> 7;
  } else {
    build_groups(*pl, a.ids, a.P, a.E, C::kTok);  // synchronizes the CTA
    njobs = pl->n_groups * (MODE == kModeGateUp ? (a.I + 63) / 64 : (a.H + 127) / 128);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int my_jobs = (int)blockIdx.x < njobs ? (njobs - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int nq = my_jobs * S;
  auto job_of = [&](int jl) { return (int)blockIdx.x + jl * (int)gridDim.x; };
  if constexpr (RS) {
    static_assert(!MX && C::kThreads == 768 && C::kDecWarps == 16 && C::kDecWarps % 4 == 0 &&
                      C::kDecWarps * 32 * kRsDecRegs + (C::kThreads - C::kDecWarps * 32) * kRsOtherRegs ==
                          C::kThreads * kRsLaunchRegs,
                  "register split: the shares add up to the launch's registers");
    if (warp < C::kDecWarps)
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRsDecRegs));
    else
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRsOtherRegs));
  }

  if (MX && warp < C::kDecWarps) {
    // ---------------------------------------------------------------- scale-factor warps (MX)
    // Warp w < 4 writes, for every stage, the UE8M0 bytes of tile rows 32w..32w+31 (its lane
    // quarter): each row's KB bytes, four per group column. The next stage's bytes are loaded while
    // the current stage's are stored. (The activation terms' scale factors reach TMEM by
    // tcgen05.cp from the MMA issuers.)
    if (warp < 4) {
      constexpr int kG = kKB / 4;  // scale groups per stage
      const int m = 32 * warp + lane;
      const uint32_t tq = tbase + ((uint32_t)(32 * warp) << 16);
      uint32_t pa[kKB / 2];
      int qp = 0, jl_p = 0, s_p = 0;
      const unsigned short *srow = nullptr;
      auto load_sf = [&](uint32_t(&da)[kKB / 2]) {
        if (qp >= nq) return;
        if (s_p == 0) {
          const JobRows jr = job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl_p));
          const int row = tile_row(jr, m);
          srow = reinterpret_cast<const unsigned short *>(jr.sc + (size_t)(row >= 0 ? row : jr.y0) * nbr);
        }
        const int lim = nbr - kKB * s_p;  // blocks of the stage inside the row (even)
        const unsigned short *p = srow + (kKB / 2) * s_p;
#pragma unroll
        for (int i = 0; i < kKB / 2; i++) da[i] = 2 * i < lim ? (uint32_t)__ldg(p + i) : 0u;
        qp++;
        if (++s_p == S) {
          s_p = 0;
          jl_p++;
        }
      };
      load_sf(pa);
      uint32_t b = 0;
      bool ok = true;
#pragma unroll 1
      for (int q = 0; q < nq; q++) {
        uint32_t na[kKB / 2];
        load_sf(na);
        if (q >= kNA) {
          const uint32_t ph = (uint32_t)((q - kNA) / kNA) & 1u;
          if (!(ok = warp_wait(&a_empty[2 * b], ph, tmo, abort_flag) && warp_wait(&a_empty[2 * b + 1], ph, tmo, abort_flag)))
            break;
          tc_fence_after();
        }
#pragma unroll
        for (int g = 0; g < kG; g++)
          tmem_st_x1(tq + kSfaCol + kKB * b + 4u * (uint32_t)g + (uint32_t)warp, pa[2 * g] | (pa[2 * g + 1] << 16));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        mbar_arrive_one(&a_full[2 * b]);
        mbar_arrive_one(&a_full[2 * b + 1]);
#pragma unroll
        for (int i = 0; i < kKB / 2; i++) pa[i] = na[i];
        b = b + 1 == (uint32_t)kNA ? 0u : b + 1;
      }
      if (!ok) *abort_flag = 1;
    }
  } else if (warp < C::kDecWarps) {
    // ---------------------------------------------------------------- decode warps
    // Thread (warp w, lane l) owns tile row m = 32 (w % 4) + l and the kNBT blocks kNBT (w / 4).. of
    // each stage, decoded in chunks of eight (64 bytes of words, four 16-byte reads).
    const int sp = warp & 3, h = warp >> 2, m = 32 * sp + lane;
    const int hf = 2 * kNBT * h / kKB;  // the half of the stage this warp's blocks lie in
    // 16-byte chunk c of box row rb sits at chunk c ^ (rb & 7) (128-byte swizzle). A chunk of eight
    // blocks is 64 bytes at an offset that is a multiple of 64, so its four reads are chunks
    // c0 + i (c0 = 0 or 4) of one box row: at (c0 ^ (sw & 4)) | (i ^ (sw & 3)).
    const uint32_t rb = (uint32_t)(m & 63), sw = rb & 7u;
    const uint32_t wrow = smem_u32(smem + geo.off_W) + (uint32_t)(m >> 6) * C::kBoxCols * 8192u + rb * 128u;
    static_assert(kNBT == 8, "one 8-block chunk (64 bytes of words) per decode thread and stage");
    // this thread's blocks are bytes 64 h .. 64 h + 63 of its stage row: the four reads of a stage
    // at wrd[i] + (slot offset)
    const uint32_t byte0 = (uint32_t)(kNBT * h) * 8u;
    const uint32_t wc0 = wrow + (byte0 >> 7) * 8192u + ((((byte0 >> 4) & 7u) ^ (sw & 4u)) * 16u);
    uint32_t wrd[4];
#pragma unroll
    for (int i = 0; i < 4; i++) wrd[i] = wc0 + ((uint32_t)i ^ (sw & 3u)) * 16u;
    const uint32_t tq = tbase + ((uint32_t)(32 * sp) << 16);  // this warp's TMEM lane quarter
    const uint32_t acol = tq + C::kACol + 4u * (uint32_t)(kNBT * h);  // its A columns in stage 0

    // The UE8M0 bytes of this thread's kNG groups of four blocks (16-bit loads of block pairs),
    // loaded one stage ahead of their use. Rows outside the tile read the job's first row instead
    // (their products are never stored). Only the weights' scales: the activation terms' scale
    // factors reach TMEM by tcgen05.cp from the MMA issuers, so nothing here waits for the
    // preceding kernel.
    uint32_t pa[kNBT / 2];
    int qp = 0, jl_p = 0, s_p = 0;
    const unsigned short *srow = nullptr;  // row m's scales of the front job, from block kNBT h on
    auto load_sf = [&](uint32_t(&da)[kNBT / 2]) {
      if (TILED || qp >= nq) return;
      if (s_p == 0) {
        const JobRows jr = job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl_p));
        const int row = tile_row(jr, m);
        srow = reinterpret_cast<const unsigned short *>(jr.sc + (size_t)(row >= 0 ? row : jr.y0) * nbr + kNBT * h);
      }
      // blocks of this thread's range inside the row (even, so no 16-bit load crosses the row end).
      // Predicated loads, no branch: a branch around them would make the compiler wait for the
      // loads where the paths join, exposing their latency at the start of every stage.
      const int lim = nbr - kKB * s_p - kNBT * h;
      const unsigned short *p = srow + (kKB / 2) * s_p;
#pragma unroll
      for (int i = 0; i < kNBT / 2; i++) da[i] = 2 * i < lim ? (uint32_t)__ldg(p + i) : 0u;
      qp++;
      if (++s_p == S) {
        s_p = 0;
        jl_p++;
      }
    };
    load_sf(pa);

    // Barrier latencies are hidden: the release of this stage's A slot and the arrival of the next
    // stage's words are tested (non-blocking) before a chunk's decode and their results read after
    // it; only a barrier found incomplete costs a blocking wait.
    // ring positions with their barrier phases, advanced as the slots wrap: word slot ws (phase
    // wph of its next fill), A slot b (bph = parity of the uses of slot b so far)
    uint32_t ws = 0, b = 0, wph = 0, bph = 0;
    bool ok = true, wf_ready = false;
    // carry path: this thread's first block of the stage is block kKB s_c + kNBT h of its row, at
    // position r_c of its segment (r_c = 0: a segment starts there); srow_w = the row's words
    const int segb = CARRY ? a.seg_blocks : 1, seg_inc = CARRY ? kKB % segb : 0;
    int s_c = 0, jl_c = 0, r_c = 0;
    const uint2 *srow_w = nullptr;
#pragma unroll 1
    for (int q = 0; q < nq; q++) {
      if (!wf_ready && !(ok = warp_wait(&w_full[ws], wph, tmo, abort_flag))) break;
      uint32_t cL = 0u, cH = 0u, smask = 0xFFu;  // carry into the first block; blocks that start a segment
      if constexpr (CARRY) {
        if (s_c == 0) {
          const JobRows jr = job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl_c));
          const int row = tile_row(jr, m);
          srow_w = row >= 0 ? reinterpret_cast<const uint2 *>(jr.st) + (size_t)row * nbr : nullptr;
          r_c = (kNBT * h) % segb;
        }
        smask = 0u;
        for (int k = r_c == 0 ? 0 : segb - r_c; k < kNBT; k += segb) smask |= 1u << k;
        if (r_c != 0) {
          if (h > 0) {  // the block before this thread's range is in the same tile
            const uint32_t byte = (uint32_t)(kNBT * h - 1) * 8u;
            const uint2 v = lds_u2(wrow + ws * kWStage + (byte >> 7) * 8192u + ((((byte >> 4) & 7u) ^ sw) * 16u) + 8u);
            cL = v.x;
            cH = v.y;
          } else if (srow_w != nullptr) {  // the previous stage's last block of the row
            const uint2 v = __ldg(srow_w + (size_t)kKB * s_c - 1);
            cL = v.x;
            cH = v.y;
          }
        }
      }
      uint32_t na[kNBT / 2];
      load_sf(na);  // the next stage's scale bytes; their latency hides behind this stage
      const uint32_t wa = ws * kWStage;
      const uint32_t ws1 = ws + 1 == (uint32_t)kNW ? 0u : ws + 1, wph1 = ws1 == 0u ? wph ^ 1u : wph;
      uint4 cw[4];
#pragma unroll
      for (int i = 0; i < 4; i++) cw[i] = lds_u4(wrd[i] + wa);
      uint32_t ae = 1u, wf = 0u;
      if (q >= kNA) ae = mbar_test(&a_empty[2 * b + hf], bph ^ 1u);
      if (q + 1 < nq) wf = mbar_test(&w_full[ws1], wph1);
      uint32_t W[8][4];
      if constexpr (CARRY) {
#pragma unroll
        for (int i = 0; i < 8; i++) {
          const uint32_t L = (i & 1) ? cw[i >> 1].z : cw[i >> 1].x, Hh = (i & 1) ? cw[i >> 1].w : cw[i >> 1].y;
          if ((smask >> i) & 1u) cL = cH = 0u;
          planes_to_nibbles_interleaved(decode_block(L, Hh, cL, cH), W[i][0], W[i][1], W[i][2], W[i][3]);
          cL = L;
          cH = Hh;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; i++) {
          planes_to_nibbles_interleaved_i3(decode_block0_i3(cw[i].x, cw[i].y), W[2 * i][0], W[2 * i][1],
                                           W[2 * i][2], W[2 * i][3]);
          planes_to_nibbles_interleaved_i3(decode_block0_i3(cw[i].z, cw[i].w), W[2 * i + 1][0], W[2 * i + 1][1],
                                           W[2 * i + 1][2], W[2 * i + 1][3]);
        }
      }
      __syncwarp();  // every word of the stage has been read (and used): free the slot
      mbar_arrive_one(&w_empty[ws]);
      if (q >= kNA) {
        if (!__all_sync(0xffffffffu, ae != 0u) && !(ok = warp_wait(&a_empty[2 * b + hf], bph ^ 1u, tmo, abort_flag)))
          break;
        tc_fence_after();
      }
      // the codes: columns 4 kNBT h.. of the stage's A. Columns of blocks beyond the row's end hold
      // the decode of the zero fill; no MMA reads them.
      tmem_st_codes<8>(acol + C::kACols * b, W);
      if (!ok) break;
      wf_ready = __all_sync(0xffffffffu, wf != 0u);
      ws = ws1;
      wph = wph1;
      // the scale factors of this row: its own quarter, column 4g + quarter of group g
      if constexpr (!TILED) {
#pragma unroll
        for (int g = 0; g < kNG; g++) {
          const uint32_t gg = (uint32_t)(kNG * h + g), wg = pa[2 * g] | (pa[2 * g + 1] << 16);
          if constexpr (SETS == 1) {
            tmem_st_x1(tq + kSfaCol + kKB * b + 4u * gg + (uint32_t)sp, wg);
          } else {  // the four powers of two of each E5M3 scale, set i at column i KB of the stage
            uint32_t st4[4];
            e5m3_scale_sets(wg, st4);
#pragma unroll
            for (int i = 0; i < 4; i++)
              tmem_st_x1(tq + kSfaCol + SETS * kKB * b + (uint32_t)i * kKB + 4u * gg + (uint32_t)sp, st4[i]);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      mbar_arrive_one(&a_full[2 * b + hf]);
#pragma unroll
      for (int i = 0; i < kNBT / 2; i++) pa[i] = na[i];
      if (++b == (uint32_t)kNA) {
        b = 0;
        bph ^= 1u;
      }
      if constexpr (CARRY) {
        r_c += seg_inc;
        if (r_c >= segb) r_c -= segb;
        if (++s_c == S) {
          s_c = 0;
          jl_c++;
        }
      }
    }
    if (!ok) *abort_flag = 1;
  } else if (warp == C::kWLoadWarp) {
    // ---------------------------------------------------------------- word loader warp
    // TMA front: stage qi of job jl_i, up to kNW stages ahead of the decode warps.
    const uint32_t wbase = smem_u32(smem + geo.off_W);
    unsigned char *my_maps = MODE == kModeGemv ? nullptr : a.maps + (size_t)blockIdx.x * kMapSlots * 128;
    int qi = 0, jl_i = 0, s_i = 0;
    uint32_t wi = 0;
    const void *map_i = &wmap;
    JobRows ji{};
    bool ok = true;
    while (ok && qi < nq && !*abort_flag) {  // whole warp; lane 0 issues the two boxes of stage qi
      if (s_i == 0) {
        ji = job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl_i));
        if (MODE != kModeGemv) {
          unsigned char *gm = my_maps + (size_t)(jl_i % kMapSlots) * 128;
          if (lane == 0) tmap_set_address(smem_u32(smap), ji.st);
          __syncwarp();
          tmap_publish(gm, smem_u32(smap));
          if (lane == 0) tmap_acquire(gm);
          map_i = gm;
        }
      }
      if (lane == 0) {
        if constexpr (MX) {
          // two halves of KB/2 blocks, each its own barrier pair: column box c (128 bytes = 8 blocks)
          // of rows y0.. at (2c) x 8 KB and of rows y1.. at (2c + 1) x 8 KB, so each column's 128
          // rows form one SBO = 1 KB operand tile
          const uint32_t dst = wbase + wi * kWStage;
#pragma unroll
          for (int hh = 0; hh < 2; hh++) {
            if (qi >= kNW && ok)
              ok = mbar_wait_sleep(&w_empty[2 * wi + hh], (uint32_t)((qi - kNW) / kNW) & 1u, tmo, kLoaderSleepNs);
            if (ok) {
              mbar_arrive_expect_tx(&w_full[2 * wi + hh], kWStage / 2);
#pragma unroll
              for (int c = hh * kKB / 16; c < (hh + 1) * kKB / 16; c++) {
                tma_load_2d(dst + (uint32_t)(2 * c) * 8192u, map_i, kKB * 16 * s_i + 128 * c, ji.y0, &w_full[2 * wi + hh]);
                tma_load_2d(dst + (uint32_t)(2 * c + 1) * 8192u, map_i, kKB * 16 * s_i + 128 * c, ji.y1,
                            &w_full[2 * wi + hh]);
              }
            }
          }
        } else {
          if (qi >= kNW) ok = mbar_wait_sleep(&w_empty[wi], (uint32_t)((qi - kNW) / kNW) & 1u, tmo, kLoaderSleepNs);
          if (ok) {
            mbar_arrive_expect_tx(&w_full[wi], kWStage);
            const uint32_t dst = wbase + wi * kWStage;
#pragma unroll
            for (int c = 0; c < C::kBoxCols; c++) {
              tma_load_2d(dst + (uint32_t)c * 8192u, map_i, kKB * 8 * s_i + 128 * c, ji.y0, &w_full[wi]);
              tma_load_2d(dst + (uint32_t)(C::kBoxCols + c) * 8192u, map_i, kKB * 8 * s_i + 128 * c, ji.y1,
                          &w_full[wi]);
            }
          }
        }
      }
      // At the start the first stage is let land before the third is requested: with every CTA's
      // stages requested at once, the first lands only near the end of the whole burst, and the
      // decode warps wait for it.
      if (!MX && qi == 1 && lane == 0 && ok) ok = mbar_wait_sleep(&w_full[0], 0u, tmo, 32u);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      wi = wi + 1 == (uint32_t)kNW ? 0u : wi + 1;
      qi++;
      if (++s_i == S) {
        s_i = 0;
        jl_i++;
      }
    }
    if (!ok) *abort_flag = 1;
    // drain: the last min(kNW, qi) issued stages may still be in flight
    if (lane == 0)
      for (int d = qi - 1; d >= 0 && d >= qi - kNW; d--) {
        if (!mbar_wait(&w_full[MX ? 2 * (d % kNW) : d % kNW], (uint32_t)(d / kNW) & 1u, tmo)) break;
        if (MX && !mbar_wait(&w_full[2 * (d % kNW) + 1], (uint32_t)(d / kNW) & 1u, tmo)) break;
      }
    __syncwarp();
  } else if (warp == C::kBLoadWarp) {
    // ---------------------------------------------------------------- B loader warp
    int issued = 0;
    grid_dep_wait();     // the activation terms come from the preceding kernel (a split, or gate/up)
    grid_dep_release();  // a dependent launch may start its prologue now
    if (lane == 0) {
      int jl = 0, s = 0;
      const uint8_t *src = nullptr;
      bool ok = true;
      for (int q = 0; q < nq; q++) {
        if (*abort_flag) break;
        const int bb = q % C::kNB;
        int job_chunk = 0;
        if (s == 0) {
          const JobRows jq = job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl));
          src = a.terms + (size_t)jq.group * tbytes;
        }
        if (TILED) job_chunk = job_of(jl);  // plain GEMV: the job is the 128-row tile
        // up to kNB stages ahead of the MMAs: the slot is free once its last use was released
        if (q >= C::kNB && !(ok = mbar_wait_sleep(&b_empty[bb], (uint32_t)((q - C::kNB) / C::kNB) & 1u, tmo,
                                                  kLoaderSleepNs)))
          break;
        mbar_arrive_expect_tx(&b_full[bb], geo.bslot);
        bulk_g2s(smem + geo.off_B + (uint32_t)bb * geo.bslot, src + (size_t)s * C::kBSlot, C::kBSlot, &b_full[bb]);
        if (TILED)
          bulk_g2s(smem + geo.off_B + (uint32_t)bb * geo.bslot + C::kBSlot,
                   a.sf_tiles + ((size_t)job_chunk * a.sf_groups + (size_t)s * (kKB / 4)) * 512u, C::kSfaTile,
                   &b_full[bb]);
        issued++;
        if (++s == S) {
          s = 0;
          ++jl;
        }
      }
      if (!ok) *abort_flag = 1;
      for (int d = issued - 1; d >= 0 && d >= issued - C::kNB; d--)
        if (!mbar_wait(&b_full[d % C::kNB], (uint32_t)(d / C::kNB) & 1u, tmo)) break;
    }
    __syncwarp();
  } else if (warp >= C::kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue warps
    // Warp C::kEpiWarp0 + i reads TMEM lane quarter eq = warp % 4, i.e. tile rows 32 eq..32 eq + 31.
    const int eq = warp & 3;
    auto epilogue = [&](int jl_e) {
      const JobRows jr = job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl_e));
      const int buf = jl_e & 1;                   // the gate/up exchange buffer
      const int abuf = jl_e % C::kNAcc;           // the accumulator
      // one warp polls; the others wait at a named barrier (no issue slots taken meanwhile). The
      // poller is the epilogue warp on the sub-partition of the B loader (warp % 4 == 3): the word
      // loader's and the MMA issuers' sub-partitions carry more besides their four decode warps.
      if (warp == C::kEpiWarp0 + 3) {
        if (!mbar_wait_sleep(&acc_full[abuf], (uint32_t)(jl_e / C::kNAcc) & 1u, tmo, kEpiSleepNs)) *abort_flag = 1;
      }
      named_bar(1, 128);
      if (*abort_flag) return;
      tc_fence_after();
      float v[C::kTok];
#pragma unroll
      for (int t = 0; t < C::kTok; t++) v[t] = 0.f;
      // with two issuers the second accumulator holds the second halves of the stages; it was never
      // written when the rows fit in half a stage
      const int nacc = C::kNI == 2 && nbr > kKB / 2 ? 2 : 1;
      for (int ia = 0; ia < nacc; ia++) {
#pragma unroll
        for (int c0 = 0; c0 < C::kTok * kTerms; c0 += 16) {
          uint32_t r[16];
          tmem_ld_x16(tbase + ((uint32_t)(32 * eq) << 16) + (uint32_t)((abuf * C::kNI + ia) * NMAX + c0), r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; i++)
            if (c0 + i < C::kTok * kTerms) v[(c0 + i) / kTerms] += __uint_as_float(r[i]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[abuf]);
      const int mrow = 32 * eq + lane;
      if (MODE == kModeGemv) {
        const int row = tile_row(jr, mrow);
        if (row >= 0)
#pragma unroll
          for (int t = 0; t < C::kTok; t++)
            if (t < a.T) a.y[(size_t)t * a.rows + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v[t]));
      } else if (MODE == kModeGateUp) {
        float *U = reinterpret_cast<float *>(smem + geo.off_U) + (size_t)buf * 64 * C::kTok;
        const uint32_t use = (uint32_t)(jl_e >> 1);
        if (eq >= 2) {  // up rows: hand them to the gate rows' warps
          if (use >= 1 && !mbar_wait(&u_empty[buf], (use - 1u) & 1u, tmo)) {
            *abort_flag = 1;
            return;
          }
#pragma unroll
          for (int t = 0; t < C::kTok; t++) U[(mrow - 64) * C::kTok + t] = v[t];
          __syncwarp();
          if (lane == 0) mbar_arrive(&u_full[buf]);
        } else {
          if (!mbar_wait(&u_full[buf], use & 1u, tmo)) {
            *abort_flag = 1;
            return;
          }
          // h = bf16(silu(g) u) of this warp's 32 rows, which are one 32-block of the down product's
          // K, for every token of the group: written out, and split here into the down kernel's
          // activation terms. The B rows of empty slots are not written: an MMA column depends on
          // its own B row only, and the down epilogue reads the columns of the group's tokens.
          constexpr int NT = C::kSplitNT, kTokPad = (C::kTok + NT - 1) / NT * NT;
          float hv[kTokPad];
#pragma unroll
          for (int t = 0; t < kTokPad; t++) {
            hv[t] = 0.f;
            if (t < C::kTok && t < jr.cnt && mrow < jr.na) {
              const float g = v[t], u = U[mrow * C::kTok + t];
              const int p = pl->list[jr.first + t];
              const __nv_bfloat16 hb = __float2bfloat16_rn(g / (1.0f + expf(-g)) * u);
              a.hidden[(size_t)p * a.I + jr.row0 + mrow] = __bfloat16_as_ushort(hb);
              hv[t] = __bfloat162float(hb);
            }
          }
          if (jr.row0 + 32 * eq < a.I) {  // warp-uniform
            const int S_dn = (a.I / 32 + kKB - 1) / kKB, kb_dn = jr.row0 / 32 + eq;
            uint8_t *tg = a.terms_dn + (size_t)jr.group * terms_bytes<NMAX>(S_dn);
            if (jr.cnt == 1) {  // one token in the group (batch 1 and most small batches): split it alone
              split_terms_n<NMAX, MX, 1>(hv, 0, 1, kb_dn, S_dn, tg);
            } else {
#pragma unroll
              for (int t0 = 0; t0 < kTokPad; t0 += NT)
                if (t0 < jr.cnt) split_terms_n<NMAX, MX, NT>(hv + t0, t0, jr.cnt, kb_dn, S_dn, tg);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&u_empty[buf]);
        }
      } else {
        const int row = tile_row(jr, mrow);
        if (row >= 0)
#pragma unroll
          for (int t = 0; t < C::kTok; t++)
            if (t < jr.cnt) a.yws[(size_t)pl->list[jr.first + t] * a.H + row] = v[t];
        __threadfence();
        __syncwarp();
        // the last group to finish this warp's 32 rows of the chunk combines them:
        // out = sum_j w_j y_j over the token's routed pairs, in fixed j order
        int last = 0;
        if (lane == 0) last = atomicAdd(&a.counters[jr.chunk * 4 + eq], 1) == pl->n_groups - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          const int n = jr.row0 + mrow;
          if (n < a.H)
            for (int t = 0; t < a.Tm; t++) {
              // every load of the token's pairs first (their latencies overlap), then the sum in j order
              float yv[kMaxTopK], wv[kMaxTopK];
              bool use[kMaxTopK];
#pragma unroll
              for (int jj = 0; jj < kMaxTopK; jj++) {
                const int p = t * a.k + jj;
                const int ee = jj < a.k ? pl->ids[p] : -1;
                use[jj] = ee >= 0 && ee < a.E;
                yv[jj] = use[jj] ? __ldcg(a.yws + (size_t)p * a.H + n) : 0.f;
                wv[jj] = use[jj] ? __ldg(a.wts + p) : 0.f;
              }
              float acc = 0.f;
#pragma unroll
              for (int jj = 0; jj < kMaxTopK; jj++)
                if (use[jj]) acc = fmaf(wv[jj], yv[jj], acc);
              a.out[(size_t)t * a.H + n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
            }
        }
      }
    };
    for (int jl = 0; jl < my_jobs && !*abort_flag; jl++) epilogue(jl);
  } else if (warp - C::kMmaWarp < C::kNI) {
    // ---------------------------------------------------------------- MMA warp(s)
    // The whole warp runs the loop (its values are warp-uniform); one elected lane issues the
    // tcgen05 operations. With two issuers, warp C::kMmaWarp + i issues the MMAs of half i of every
    // stage into accumulator i of the job's pair; with one, warp C::kMmaWarp issues both halves.
    const bool leader = elect_one();
    const int h_lo = C::kNI == 2 ? warp - C::kMmaWarp : 0, h_hi = C::kNI == 2 ? h_lo + 1 : 2;
    int jl = 0, s = 0;
    uint32_t ncols = (uint32_t)(my_jobs ? job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(0)).ncols : 16);
    uint32_t idesc0 = idesc_mxf4(ncols, 0u), idesc2 = idesc_mxf4(ncols, 2u);
    const uint32_t b0 = smem_u32(smem + geo.off_B);
    bool ok = true;
    for (int q = 0; q < nq; q++) {
      if (*abort_flag) break;
      const int b = q % kNA;
      const uint32_t ph = (uint32_t)(q / kNA) & 1u;
      const int bb = q % C::kNB;
      ok = mbar_wait_sleep(&b_full[bb], (uint32_t)(q / C::kNB) & 1u, tmo, kMmaSleepNs);
      if (ok && s == 0 && jl >= C::kNAcc)  // the job's accumulator was read out by its last user
        ok = mbar_wait_sleep(&acc_empty[jl % C::kNAcc], (uint32_t)(jl / C::kNAcc - 1) & 1u, tmo, kMmaSleepNs);
      const int nmma = (nbr - kKB * s < kKB ? nbr - kKB * s : kKB) >> 1;
      const uint32_t at = tbase + C::kACol + C::kACols * (uint32_t)b;
      // Descriptors of this stage's B slot: the low words of a start address advance by immediates
      // (16-byte units, inside the 14-bit field), the high words stay.
      const uint64_t bd = smem_desc(b0 + (uint32_t)bb * geo.bslot, 128u, C::kSbo);
      const uint32_t bd_lo = (uint32_t)bd, bd_hi = (uint32_t)(bd >> 32);
      // the stage's B scale tiles, then (TILED) the weights' scale tiles: 512 bytes = 32 units each
      const uint64_t sd = smem_desc(b0 + (uint32_t)bb * geo.bslot + C::kBStage, 128u, 128u);
      const uint32_t sd_lo = (uint32_t)sd, sd_hi = (uint32_t)(sd >> 32);
      const uint32_t sfa = tbase + kSfaCol + SETS * kKB * (uint32_t)b, sfb = tbase + kSfbCol + C::kSfbCols * (uint32_t)b;
      const int wsx = q % kNW;  // MX: the stage's word slot
      const uint64_t ad0 = MX ? desc_sw128(smem_u32(smem + geo.off_W) + (uint32_t)wsx * kWStage) : 0ull;
      // This issuer's halves of the stage, in order: half h_lo only with two issuers, both with one.
      // Inside a half every operand is a per-half base plus a compile-time offset (kKB / 4 MMAs of
      // K = 64, kKB / 8 groups of four blocks; kKB / 4 is even, so MMA j0 + jj takes scale id
      // 2 (jj & 1) of group g0 + jj / 2).
#pragma unroll
      for (int hi = 0; hi < 3 - C::kNI; hi++) {
        const int hh = C::kNI == 2 ? h_lo : hi;
        ok = __all_sync(0xffffffffu, ok && mbar_wait_sleep(&a_full[2 * b + hh], ph, tmo, kMmaSleepNs));
        if (MX && ok)
          ok = __all_sync(0xffffffffu,
                          mbar_wait_sleep(&w_full[2 * wsx + hh], (uint32_t)(q / kNW) & 1u, tmo, kMmaSleepNs));
        if (!ok) break;
        tc_fence_after();
        const int j0 = hh * (kKB / 4), g0 = hh * (kKB / 8);
        const int lim = nmma - j0;  // MMAs of this half inside the row (fewer in a row's last stage)
        // the first MMA of a job into this issuer's accumulator starts it (each issuer has its own)
        const bool first = s == 0 && (C::kNI == 2 || hh == 0);
        const uint32_t d_t = tbase + (uint32_t)(((jl % C::kNAcc) * C::kNI + (C::kNI == 2 ? hh : 0)) * NMAX);
        if (leader) {
          // the B scale factors of this half's groups, ahead of the MMAs that read them (tcgen05
          // operations of one thread run in issue order)
          const uint32_t sdb = sd_lo + 32u * (uint32_t)(C::kNTile * g0), sfb_h = sfb + C::kSfbGCols * (uint32_t)g0;
#pragma unroll
          for (int gg = 0; gg < kKB / 8; gg++)
            if (2 * gg < lim)
#pragma unroll
              for (int ti = 0; ti < C::kNTile; ti++)
                tmem_cp_sf(sfb_h + C::kSfbGCols * (uint32_t)gg + 4u * ti,
                           desc_of(sdb + 32u * (uint32_t)(C::kNTile * gg + ti), sd_hi));
          const uint32_t sfa_h = sfa + 4u * (uint32_t)g0;
          if constexpr (TILED) {  // the weights' scale factors: tile row r to lanes r, 32 + r, 64 + r, 96 + r
            const uint32_t sda = sd_lo + (C::kSfbStage >> 4) + 32u * (uint32_t)g0;
#pragma unroll
            for (int gg = 0; gg < kKB / 8; gg++)
              if (2 * gg < lim) tmem_cp_sf(sfa_h + 4u * (uint32_t)gg, desc_of(sda + 32u * (uint32_t)gg, sd_hi));
          }
          const uint32_t at_h = at + 8u * (uint32_t)j0, bd_h = bd_lo + 16u * (uint32_t)j0;
#pragma unroll
          for (int jj = 0; jj < kKB / 4; jj++) {
            if (jj < lim) {
              // +256 bytes of B per MMA: the descriptor's start address counts 16-byte units; the
              // scale id sits in bits 30-31 of the scale-factor address (zero lane bits here)
              const uint32_t sfo = 4u * (uint32_t)(jj >> 1) + ((uint32_t)(jj & 1) << 31);
              const uint32_t id = (jj & 1) ? idesc2 : idesc0;
              if constexpr (MX)  // A: column box j / 4 (16 KB apart), 32 bytes per MMA inside it
                mma_mxf4_ss(d_t, ad0 + (uint64_t)(((j0 + jj) >> 2) * 1024 + 2 * (jj & 3)),
                            desc_of(bd_h + 16u * (uint32_t)jj, bd_hi), id, sfa_h + sfo,
                            sfb_h + C::kSfbGCols * (uint32_t)(jj >> 1) + ((uint32_t)(jj & 1) << 31),
                            !(first && jj == 0));
              else
#pragma unroll
                for (int st = 0; st < SETS; st++)  // one MMA per scale set (SETS = 4: E5M3)
                  mma_mxf4_ts(d_t, at_h + 8u * (uint32_t)jj, desc_of(bd_h + 16u * (uint32_t)jj, bd_hi), id,
                              sfa_h + (uint32_t)st * kKB + sfo,
                              sfb_h + C::kSfbGCols * (uint32_t)(jj >> 1) + ((uint32_t)(jj & 1) << 31),
                              !(first && jj == 0 && st == 0));
            }
          }
          tc_commit(&a_empty[2 * b + hh]);
          if (MX) tc_commit(&w_empty[2 * wsx + hh]);
          if (hh == h_hi - 1) {
            tc_commit(&b_empty[bb]);
            if (s == S - 1) tc_commit(&acc_full[jl % C::kNAcc]);
          }
        }
      }
      if (!ok) break;
      __syncwarp();
      if (++s == S) {
        s = 0;
        if (++jl < my_jobs) {
          const uint32_t nc = (uint32_t)job_rows<MAXE, MODE, NMAX>(a, tab, pl, job_of(jl)).ncols;
          if (nc != ncols) {
            ncols = nc;
            idesc0 = idesc_mxf4(ncols, 0u);
            idesc2 = idesc_mxf4(ncols, 2u);
          }
        }
      }
    }
    if (!ok && lane == 0) *abort_flag = 1;
    // drain: every tcgen05 operation this issuer started (the barrier completes once every issuer
    // has committed)
    if (leader) {
      tc_commit(drain);
      mbar_wait(drain, 0u, tmo);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == C::kMmaWarp) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------------------- host side

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Tensor map of a trellis stream seen as a [rows][nbr*8] byte matrix (bpb = 8 bytes per block), or
// of a resident MXFP4 nibble matrix [rows][nbr*16] (bpb = 16): boxes of 64 rows x 128 bytes with
// the 128-byte swizzle (the decode threads' 16-byte reads of consecutive rows then fall in distinct
// banks; for MXFP4 it is the MMA's K-major A layout); rows and columns beyond the matrix read as
// zero.
static bool make_word_map(CUtensorMap *map, const void *stream, int rows, int nbr, int bpb = 8) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)nbr * (cuuint64_t)bpb, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)nbr * (cuuint64_t)bpb};
  cuuint32_t box[2] = {128u, 64u};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(stream), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// GEMV tokens per pass; B width (template NMAX) for a pass or group of T tokens: up to 5 tokens on
// the 32-row B operand, up to 16 on the 96-row one, up to 32 on the 192-row one.
constexpr int kGemvTok = Cfg<192>::kTok;
// (6 to 10 tokens on the 64-row one, which keeps the 32-block stages and their 16 decode warps).
static int nmax_for(int tokens_per_group) {
  return tokens_per_group <= Cfg<32>::kTok   ? 32
         : tokens_per_group <= Cfg<64>::kTok ? 64
         : tokens_per_group <= Cfg<96>::kTok ? 96
                                             : 192;
}
// The resident-MXFP4 source has no 64-row configuration (its 32-block A tiles leave no room).
static int mx_nmax_for(int tokens_per_group) {
  const int n = nmax_for(tokens_per_group);
  return n == 64 ? 96 : n;
}
// The grouped MoE keeps groups of at most 16 tokens: with routed tokens spread over the experts a
// wider B operand would mostly multiply empty slots.
static int moe_nmax_for(int T) { return nmax_for(T) == 32 ? 32 : 96; }
static uint32_t geom_smem_for(int NMAX, int mode, bool mx, bool tiled);
// E5M3 scales (four scale sets) have no 64-row configuration either.
static int e5_nmax_for(int tokens_per_group) { return mx_nmax_for(tokens_per_group); }
template <int NMAX, int SETS = 1>
static uint32_t geom_smem(int mode, bool mx, bool tiled) { return mma_geom<NMAX, SETS>(mode, mx, tiled).smem; }
static uint32_t geom_smem_for(int NMAX, int mode, bool mx, bool tiled, int sets = 1) {
  if (sets == 4)
    return NMAX == 32 ? geom_smem<32, 4>(mode, mx, tiled)
                      : (NMAX == 96 ? geom_smem<96, 4>(mode, mx, tiled) : geom_smem<192, 4>(mode, mx, tiled));
  return NMAX == 32   ? geom_smem<32>(mode, mx, tiled)
         : NMAX == 64 ? geom_smem<64>(mode, mx, tiled)
         : NMAX == 96 ? geom_smem<96>(mode, mx, tiled)
                      : geom_smem<192>(mode, mx, tiled);
}

static bool mma_fits(int NMAX, int mode, bool mx = false, bool tiled = false, int sets = 1) {
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
  const uint32_t need = geom_smem_for(NMAX, mode, mx, tiled, sets);
  return need <= (uint32_t)optin;
}

// The tensor-core path needs an even number of 32-blocks per row (whole K = 64 MMAs, and a row
// pitch that is a multiple of 16 bytes for the tensor map) and a 16-byte aligned stream.
static bool k_ok(int nbr) { return nbr >= 2 && nbr % 2 == 0; }

static size_t terms_for(int nbr, int NMAX, int sets = 1) {
  if (sets == 4)
    return NMAX == 32   ? terms_bytes<32, 4>((nbr + Cfg<32, 4>::kKB - 1) / Cfg<32, 4>::kKB)
           : NMAX == 96 ? terms_bytes<96, 4>((nbr + Cfg<96, 4>::kKB - 1) / Cfg<96, 4>::kKB)
                        : terms_bytes<192, 4>((nbr + Cfg<192, 4>::kKB - 1) / Cfg<192, 4>::kKB);
  return NMAX == 32   ? terms_bytes<32>((nbr + Cfg<32>::kKB - 1) / Cfg<32>::kKB)
         : NMAX == 64 ? terms_bytes<64>((nbr + Cfg<64>::kKB - 1) / Cfg<64>::kKB)
         : NMAX == 96 ? terms_bytes<96>((nbr + Cfg<96>::kKB - 1) / Cfg<96>::kKB)
                      : terms_bytes<192>((nbr + Cfg<192>::kKB - 1) / Cfg<192>::kKB);
}

// The scale-factor threads read a row's scale bytes in pairs (16-bit loads): the scales must be
// 2-byte aligned (rows are, with an even block count).
bool gemv_mma_supported(const MatView &w, int T) {
  return k_ok(w.nbr) && (reinterpret_cast<uintptr_t>(w.stream) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(w.scales) & 1u) == 0 && tensor_map_encoder() != nullptr &&
         mma_fits(nmax_for(T < kGemvTok ? T : kGemvTok), kModeGemv);
}
bool mx_gemv_supported(const MatView &w, int T) {
  return k_ok(w.nbr) && (reinterpret_cast<uintptr_t>(w.stream) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(w.scales) & 1u) == 0 && tensor_map_encoder() != nullptr &&
         mma_fits(mx_nmax_for(T < kGemvTok ? T : kGemvTok), kModeGemv, true);
}

// The tiled GEMV: the tensor-core path with the scale-tile ring (the tiles' pointer 16-byte aligned).
bool gemv_tiled_supported(const MatView &w, const uint8_t *tiles, int T) {
  return k_ok(w.nbr) && (reinterpret_cast<uintptr_t>(w.stream) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(tiles) & 15u) == 0 && tensor_map_encoder() != nullptr &&
         mma_fits(nmax_for(T < kGemvTok ? T : kGemvTok), kModeGemv, false, true);
}

static int sm_count_impl();
static int sm_count() { return sm_count_impl(); }

// Scale tiles of a [rows][nbr] matrix: 128-row tiles, each with sf_groups = 8 * ceil(nbr / 32)
// tiles of 512 bytes (a whole number of 32-block stages); byte 16 r + 4 q + i of group g of tile t
// is the scale of row 128 t + 32 q + r, block 4 g + i (0 past the matrix).
static int scale_tile_groups(int nbr) { return 8 * ((nbr + 31) / 32); }
size_t scale_tiles_bytes(const MatView &w) { return (size_t)((w.rows + 127) / 128) * scale_tile_groups(w.nbr) * 512u; }

__global__ void __launch_bounds__(256) k_scale_tiles(const uint8_t *__restrict__ sc, int rows, int nbr, int groups,
                                                     uint32_t *__restrict__ tiles, size_t nwords) {
  grid_dep_wait();
  // No early release: this kernel writes weights, which a following product kernel may read before
  // its own grid-dependency wait; its dependents start once it has exited.
  for (size_t w = (size_t)blockIdx.x * blockDim.x + threadIdx.x; w < nwords; w += (size_t)gridDim.x * blockDim.x) {
    const size_t t = w / ((size_t)groups * 128u);
    const uint32_t rem = (uint32_t)(w - t * groups * 128u), g = rem >> 7, r = (rem >> 2) & 31u, q = rem & 3u;
    const int row = (int)(128u * t + 32u * q + r);
    uint32_t v = 0;
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const int blk = (int)(4u * g) + i;
      if (row < rows && blk < nbr) v |= (uint32_t)sc[(size_t)row * nbr + blk] << (8 * i);
    }
    tiles[w] = v;
  }
}

cudaError_t launch_scale_tiles(const MatView &w, uint8_t *tiles, cudaStream_t s) {
  const size_t nwords = scale_tiles_bytes(w) / 4;
  const int grid = (int)((nwords + 255) / 256 < (size_t)(8 * sm_count()) ? (nwords + 255) / 256 : 8 * sm_count());
  return launch_dependent(k_scale_tiles, dim3(grid), dim3(256), 0, s, w.scales, w.rows, w.nbr,
                          scale_tile_groups(w.nbr), reinterpret_cast<uint32_t *>(tiles), nwords);
}

// Tokens beyond kGemvTok run as further passes, each with its own split of x.
size_t gemv_mma_workspace(const MatView &w, int T) { return terms_for(w.nbr, nmax_for(T < kGemvTok ? T : kGemvTok)); }
size_t mx_gemv_workspace(const MatView &w, int T) { return terms_for(w.nbr, mx_nmax_for(T < kGemvTok ? T : kGemvTok)); }
// E5M3 scales on the tensor cores: the trellis conditions, with the four-set configurations.
bool gemv_e5m3_mma_supported(const MatView &w, int T) {
  return k_ok(w.nbr) && (reinterpret_cast<uintptr_t>(w.stream) & 15u) == 0 &&
         (reinterpret_cast<uintptr_t>(w.scales) & 1u) == 0 && tensor_map_encoder() != nullptr &&
         mma_fits(e5_nmax_for(T < kGemvTok ? T : kGemvTok), kModeGemv, false, false, 4);
}
size_t gemv_e5m3_mma_workspace(const MatView &w, int T) {
  return terms_for(w.nbr, e5_nmax_for(T < kGemvTok ? T : kGemvTok), 4);
}

static int sm_count_impl() {
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  return nsm;
}

// One launch of a product kernel instance (dynamic shared memory attribute set once per instance).
template <int MAXE, int MODE, int NMAX, bool MX, bool CARRY, bool RS, bool TILED = false, int SETS = 1>
static cudaError_t launch_product_rs(int grid, const MmaArgs &args, const MoeTable<MAXE> &tab, const CUtensorMap &map,
                                     cudaStream_t s) {
  static unsigned long long attr = 0;
  cudaError_t e = ensure_max_dynamic_smem(k_mma<MAXE, MODE, NMAX, MX, CARRY, RS, TILED, SETS>, attr);
  if (e != cudaSuccess) return e;
  return launch_dependent(k_mma<MAXE, MODE, NMAX, MX, CARRY, RS, TILED, SETS>, dim3(grid),
                          dim3(Cfg<NMAX, SETS>::kThreads), mma_geom<NMAX, SETS>(MODE, MX, TILED).smem, s, args, tab,
                          map);
}

// True when the register-split instance was compiled with at least kRsLaunchRegs registers per
// thread, so that its split can be granted (checked once per instance).
template <int MAXE, int MODE, int NMAX, bool MX, bool CARRY, bool TILED>
static bool register_split_ok() {
  static int ok = -1;
  if (ok < 0) {
    cudaFuncAttributes fa;
    ok = cudaFuncGetAttributes(&fa, k_mma<MAXE, MODE, NMAX, MX, CARRY, true, TILED>) == cudaSuccess &&
         fa.numRegs >= kRsLaunchRegs;
  }
  return ok == 1;
}

// The decode GEMV at NMAX = 32 takes the register split when its compiled registers allow it.
template <int MAXE, int MODE, int NMAX, bool MX, bool CARRY, bool TILED = false, int SETS = 1>
static cudaError_t launch_product(int grid, const MmaArgs &args, const MoeTable<MAXE> &tab, const CUtensorMap &map,
                                  cudaStream_t s) {
  if constexpr (MODE == kModeGemv && NMAX == 32 && !MX && SETS == 1) {
    if (register_split_ok<MAXE, MODE, NMAX, MX, CARRY, TILED>())
      return launch_product_rs<MAXE, MODE, NMAX, MX, CARRY, true, TILED>(grid, args, tab, map, s);
  }
  return launch_product_rs<MAXE, MODE, NMAX, MX, CARRY, false, TILED, SETS>(grid, args, tab, map, s);
}
template <int MAXE, int MODE, int NMAX, bool MX, int SETS = 1>
static cudaError_t launch_product_seg(int grid, const MmaArgs &args, const MoeTable<MAXE> &tab, const CUtensorMap &map,
                                      cudaStream_t s) {
  if constexpr (SETS > 1) {
    return args.seg_blocks > 1 ? launch_product<MAXE, MODE, NMAX, false, true, false, SETS>(grid, args, tab, map, s)
                               : launch_product<MAXE, MODE, NMAX, false, false, false, SETS>(grid, args, tab, map, s);
  } else if constexpr (MX) {
    return launch_product<MAXE, MODE, NMAX, true, false>(grid, args, tab, map, s);
  } else if constexpr (MODE == kModeGemv) {
    if (args.sf_tiles != nullptr)
      return args.seg_blocks > 1 ? launch_product<MAXE, MODE, NMAX, false, true, true>(grid, args, tab, map, s)
                                 : launch_product<MAXE, MODE, NMAX, false, false, true>(grid, args, tab, map, s);
    return args.seg_blocks > 1 ? launch_product<MAXE, MODE, NMAX, false, true>(grid, args, tab, map, s)
                               : launch_product<MAXE, MODE, NMAX, false, false>(grid, args, tab, map, s);
  } else {
    return args.seg_blocks > 1 ? launch_product<MAXE, MODE, NMAX, false, true>(grid, args, tab, map, s)
                               : launch_product<MAXE, MODE, NMAX, false, false>(grid, args, tab, map, s);
  }
}

template <int NMAX, bool MX, int SETS = 1>
static cudaError_t launch_gemv_pass(const MatView &w, const CUtensorMap &map, const uint16_t *x, int T, uint16_t *y,
                                    void *ws, cudaStream_t s, const uint8_t *tiles) {
  uint8_t *terms = static_cast<uint8_t *>(ws);
  const int warps = T * w.nbr, wpc = kSplitThreads / 32;
  cudaError_t e = launch_dependent(k_bsplit_gemv<NMAX, MX, SETS>, dim3((warps + wpc - 1) / wpc), dim3(kSplitThreads),
                                   0, s, x, T, w.nbr * 32, terms);
  if (e != cudaSuccess) return e;
  const int ntiles = (w.rows + 127) / 128, nsm = sm_count();
  MmaArgs args{};
  args.stream = w.stream;
  args.seg_blocks = MX ? 1 : w.seg_blocks;
  args.scales = w.scales;
  args.rows = w.rows;
  args.nbr = w.nbr;
  args.terms = terms;
  args.T = T;
  args.y = y;
  args.sf_tiles = tiles;
  args.sf_groups = scale_tile_groups(w.nbr);
  MoeTable<32> none{};
  return launch_product_seg<32, kModeGemv, NMAX, MX, SETS>(ntiles < nsm ? ntiles : nsm, args, none, map, s);
}

template <bool MX>
static cudaError_t launch_gemv_t(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s,
                                 const uint8_t *tiles = nullptr) {
  CUtensorMap map;
  if (!make_word_map(&map, w.stream, w.rows, w.nbr, MX ? 16 : 8)) return cudaErrorInvalidValue;
  const int nm = MX ? mx_nmax_for(T < kGemvTok ? T : kGemvTok) : nmax_for(T < kGemvTok ? T : kGemvTok);
  for (int t0 = 0; t0 < T; t0 += kGemvTok) {
    const int n = T - t0 < kGemvTok ? T - t0 : kGemvTok;
    const uint16_t *xp = x + (size_t)t0 * w.nbr * 32;
    uint16_t *yp = y + (size_t)t0 * w.rows;
    cudaError_t e;
    if (nm == 32)
      e = launch_gemv_pass<32, MX>(w, map, xp, n, yp, ws, s, tiles);
    else if (nm == 96)
      e = launch_gemv_pass<96, MX>(w, map, xp, n, yp, ws, s, tiles);
    else if (nm == 192)
      e = launch_gemv_pass<192, MX>(w, map, xp, n, yp, ws, s, tiles);
    else if constexpr (!MX)
      e = launch_gemv_pass<64, false>(w, map, xp, n, yp, ws, s, tiles);
    else
      e = cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_gemv_mma(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s) {
  return launch_gemv_t<false>(w, x, T, y, ws, s);
}
cudaError_t launch_mx_gemv(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s) {
  return launch_gemv_t<true>(w, x, T, y, ws, s);
}
cudaError_t launch_gemv_tiled(const MatView &w, const uint8_t *tiles, const uint16_t *x, int T, uint16_t *y, void *ws,
                              cudaStream_t s) {
  return launch_gemv_t<false>(w, x, T, y, ws, s, tiles);
}
cudaError_t launch_gemv_e5m3_mma(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s) {
  CUtensorMap map;
  if (!make_word_map(&map, w.stream, w.rows, w.nbr, 8)) return cudaErrorInvalidValue;
  const int nm = e5_nmax_for(T < kGemvTok ? T : kGemvTok);
  for (int t0 = 0; t0 < T; t0 += kGemvTok) {
    const int n = T - t0 < kGemvTok ? T - t0 : kGemvTok;
    const uint16_t *xp = x + (size_t)t0 * w.nbr * 32;
    uint16_t *yp = y + (size_t)t0 * w.rows;
    const cudaError_t e = nm == 32   ? launch_gemv_pass<32, false, 4>(w, map, xp, n, yp, ws, s, nullptr)
                          : nm == 96 ? launch_gemv_pass<96, false, 4>(w, map, xp, n, yp, ws, s, nullptr)
                                     : launch_gemv_pass<192, false, 4>(w, map, xp, n, yp, ws, s, nullptr);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ----------------------------------------------------------------------------- MoE on the tensor cores

static int moe_groups_max(int E, int P, int gmax) { return (E < P ? E : P) + P / gmax + 1; }

bool moe_mma_supported(const tcf4_moe &m, int gu_seg, int dn_seg, int T) {
  (void)gu_seg;  // any segment length: blocks after a segment's first carry the state (CARRY)
  (void)dn_seg;
  if (!k_ok(m.H / 32) || !k_ok(m.I / 32) || tensor_map_encoder() == nullptr) return false;
  for (int e = 0; e < m.E; e++)
    if (((reinterpret_cast<uintptr_t>(m.gate_up[e].stream) | reinterpret_cast<uintptr_t>(m.down[e].stream)) & 15u) ||
        ((reinterpret_cast<uintptr_t>(m.gate_up[e].scales) | reinterpret_cast<uintptr_t>(m.down[e].scales)) & 1u))
      return false;
  const int NMAX = moe_nmax_for(T);
  return mma_fits(NMAX, kModeGateUp) && mma_fits(NMAX, kModeDown);
}
// The same layer as resident MXFP4 (stream fields point at the nibble matrices).
bool moe_mx_supported(const tcf4_moe &m, int T) {
  if (!k_ok(m.H / 32) || !k_ok(m.I / 32) || tensor_map_encoder() == nullptr) return false;
  for (int e = 0; e < m.E; e++)
    if (((reinterpret_cast<uintptr_t>(m.gate_up[e].stream) | reinterpret_cast<uintptr_t>(m.down[e].stream)) & 15u) ||
        ((reinterpret_cast<uintptr_t>(m.gate_up[e].scales) | reinterpret_cast<uintptr_t>(m.down[e].scales)) & 1u))
      return false;
  const int NMAX = moe_nmax_for(T);
  return mma_fits(NMAX, kModeGateUp, true) && mma_fits(NMAX, kModeDown, true);
}

MoeMmaWorkspace moe_mma_workspace_layout(const tcf4_moe &m, int T, int k) {
  auto a256 = [](size_t v) { return (v + 255) & ~(size_t)255; };
  const int P = T * k, NMAX = moe_nmax_for(T);
  const int G = moe_groups_max(m.E, P, NMAX == 32 ? Cfg<32>::kTok : (NMAX == 96 ? Cfg<96>::kTok : Cfg<192>::kTok));
  MoeMmaWorkspace L;
  size_t off = 0;
  L.counters = off; off = a256(off + sizeof(int) * 4 * ((m.H + 127) / 128));
  L.hidden = off;   off = a256(off + sizeof(uint16_t) * (size_t)P * m.I);
  L.y = off;        off = a256(off + sizeof(float) * (size_t)P * m.H);
  L.bg_gu = off;    off = a256(off + (size_t)G * terms_for(m.H / 32, NMAX));
  L.bg_dn = off;    off = a256(off + (size_t)G * terms_for(m.I / 32, NMAX));
  // tensor-map slots: one region for the gate/up kernel and one for the down kernel (the down kernel
  // may start while gate/up CTAs still run)
  L.maps = off;     off = a256(off + 2 * (size_t)sm_count() * kMapSlots * 128);
  L.total = off;
  return L;
}

template <int MAXE, int NMAX, bool MX>
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
  CUtensorMap map_gu, map_dn;  // templates from expert 0 (every expert's matrices have the same shape)
  if (!make_word_map(&map_gu, m.gate_up[0].stream, 2 * m.I, m.H / 32, MX ? 16 : 8) ||
      !make_word_map(&map_dn, m.down[0].stream, m.H, m.I / 32, MX ? 16 : 8))
    return cudaErrorInvalidValue;
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
  args.maps = reinterpret_cast<unsigned char *>(base + L.maps);
  const int nsm = sm_count();
  const int P = T * k, G = moe_groups_max(m.E, P, Cfg<NMAX>::kTok);

  // gate_up: split x per group (and clear the down counters), then decode + MMA + SwiGLU
  {
    uint8_t *terms = reinterpret_cast<uint8_t *>(base + L.bg_gu);
    const int nbr = m.H / 32;
    const int warps = P * nbr, wpc = kSplitThreads / 32;  // one warp per routed pair and 32-block
    const int sgrid = (warps + wpc - 1) / wpc < 8 * nsm ? (warps + wpc - 1) / wpc : 8 * nsm;
    cudaError_t e = launch_dependent(k_bsplit_moe<NMAX, MX>, dim3(sgrid), dim3(kSplitThreads), 0, s, ids, P, m.E, k, x,
                                     m.H, terms, args.counters, 4 * ((m.H + 127) / 128));
    if (e != cudaSuccess) return e;
    args.nbr = nbr;
    args.terms = terms;
    args.terms_dn = reinterpret_cast<uint8_t *>(base + L.bg_dn);
    args.seg_blocks = MX ? 1 : (int)(m.gate_up[0].seg_len / 32);
    const int jobs = G * ((m.I + 63) / 64);
    e = launch_product_seg<MAXE, kModeGateUp, NMAX, MX>(jobs < nsm ? jobs : nsm, args, tab, map_gu, s);
    if (e != cudaSuccess) return e;
  }
  // down: decode + MMA of the terms the gate/up epilogue wrote, y to the workspace, last arriver per
  // chunk combines
  {
    uint8_t *terms = reinterpret_cast<uint8_t *>(base + L.bg_dn);
    const int nbr = m.I / 32;
    args.nbr = nbr;
    args.terms = terms;
    args.seg_blocks = MX ? 1 : (int)(m.down[0].seg_len / 32);
    args.maps += (size_t)nsm * kMapSlots * 128;  // the down kernel's own tensor-map slots
    const int jobs = G * ((m.H + 127) / 128);
    const cudaError_t e = launch_product_seg<MAXE, kModeDown, NMAX, MX>(jobs < nsm ? jobs : nsm, args, tab, map_dn, s);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

template <bool MX>
static cudaError_t launch_moe_t(const tcf4_moe &m, const uint16_t *x, int T, const int32_t *ids, const float *wts,
                                int k, uint16_t *out, void *ws, cudaStream_t s) {
  const bool n32 = moe_nmax_for(T) == 32;
  if (m.E <= 32)
    return n32 ? launch_moe_mma_t<32, 32, MX>(m, x, T, ids, wts, k, out, ws, s)
               : launch_moe_mma_t<32, 96, MX>(m, x, T, ids, wts, k, out, ws, s);
  return n32 ? launch_moe_mma_t<256, 32, MX>(m, x, T, ids, wts, k, out, ws, s)
             : launch_moe_mma_t<256, 96, MX>(m, x, T, ids, wts, k, out, ws, s);
}
cudaError_t launch_moe_mma(const tcf4_moe &m, const uint16_t *x, int T, const int32_t *ids, const float *wts, int k,
                           uint16_t *out, void *ws, cudaStream_t s) {
  return launch_moe_t<false>(m, x, T, ids, wts, k, out, ws, s);
}
cudaError_t launch_moe_mx(const tcf4_moe &m, const uint16_t *x, int T, const int32_t *ids, const float *wts, int k,
                          uint16_t *out, void *ws, cudaStream_t s) {
  return launch_moe_t<true>(m, x, T, ids, wts, k, out, ws, s);
}

unsigned int take_timeouts_mma() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_tcf4_timeouts_mma, sizeof v) != cudaSuccess) return 0;
  cudaMemcpyToSymbol(g_tcf4_timeouts_mma, &zero, sizeof zero);
  return v;
}

}  // namespace tcf4
