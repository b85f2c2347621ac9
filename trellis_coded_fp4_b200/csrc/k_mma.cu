// k_mma.cu -- fused trellis decode + block-scaled tensor-core product (tcgen05, sm_100a).
//
// HEPH abstract, first serving mode: the compressed stream stays resident and is decoded inside the
// product. Here the product runs on the 5th-generation tensor cores instead of CUDA-core FMAs: the
// decoded weights are already MXFP4 elements (E2M1 codes with a UE8M0 scale per 32 weights), so they
// feed a block-scaled kind::mxf8f6f4 MMA directly as the A operand (E2M1, scale factors = the
// weights' own UE8M0 bytes). The bf16 activations become the B operand, split exactly into two E4M3
// terms per element (hi + lo, each 32-block with its own UE8M0 scale); B column 2t holds token t's
// hi term and column 2t+1 its lo term, so y[t] = D[:, 2t] + D[:, 2t+1] in fp32.
//
// CTA = 8 decode warps + 1 control warp, one CTA per SM, persistent over 128-row tiles:
//  * decode thread (warp w, lane l) owns row 32(w%4)+l of the tile and K-blocks 2(w/4), 2(w/4)+1 of
//    each 128-wide K stage. It prefetches its 16 bytes of trellis words kPref stages ahead with
//    cp.async, decodes them in registers (bit-sliced) and writes the E2M1 codes into the shared A
//    stage. Warps 0-3 write the stage's A and B scale factors into TMEM (tcgen05.st).
//  * the control thread streams the pre-split activation stage (B) with bulk copies kNB stages ahead
//    and issues the stage's 4 MMAs (K = 32 each) into a double-buffered TMEM accumulator; the
//    epilogue of tile i (tcgen05.ld, y = hi + lo, bf16 stores) runs in warps 0-3 during tile i+1.
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

constexpr int kNA = 4;                // A stages (E2M1 tile + scale-factor TMEM slot)
constexpr int kNB = 8;                // B stages (activation split)
constexpr int kPref = 8;              // trellis-word stages in flight per decode thread
constexpr int kDec = 256;             // decode threads
constexpr int kMmaThreads = kDec + 32;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kSfaCol = 128, kSfbCol = 144;  // TMEM columns of the scale-factor slots

// K position (0..31) inside a 32-block of the MMA that holds weight i of the block: the decoder's
// interleaved nibble words put weight 4v+j in nibble v of word j, and word j fills bytes 4j..4j+3
// of the block's 16 data bytes (16-element chunk j/2, elements 8(j%2)..8(j%2)+7).
__host__ __device__ constexpr int kpos_of_weight(int i) { return 16 * ((i & 3) >> 1) + 8 * (i & 1) + (i >> 2); }

// Byte offset of element (n, k) (k < 128) in a K-major no-swizzle stage of 8-bit containers:
// core matrices of 8 rows x 16 bytes, LBO = 128 (K chunks), SBO = 1024 (8-row groups).
__host__ __device__ constexpr uint32_t kmajor_off(uint32_t n, uint32_t k) {
  return (n >> 3) * 1024u + (k >> 4) * 128u + (n & 7u) * 16u + (k & 15u);
}

// ------------------------------------------------------------------------------- activation split
// x [T][K] bf16 -> Bg [S][NMAX*128] E4M3 (column 2t = hi(x_t), 2t+1 = lo(x_t), columns >= 2T zero)
// and Bsf [S][32][2] UE8M0 words (byte kb%4 of word n/32 at lane n%32: scale of column n, block kb).
// hi = E4M3(x / 2^Eh) with 2^Eh = 2^(floor(log2 max|x|) - 7) over the 32-block; lo the same for the
// residual x - hi*2^Eh, which is exact in fp32. hi*2^Eh + lo*2^El reproduces every bf16 x of the
// block except elements more than ~17 binades below the block maximum.
__device__ __forceinline__ void split_e4m3(float v, float mx, uint8_t &q, uint32_t &sf, float &back) {
  if (!(mx > 0.f)) {
    q = 0;
    sf = 127u;
    back = 0.f;
    return;
  }
  int e = ilogbf(mx) - 7;
  e = e < -126 ? -126 : (e > 127 ? 127 : e);
  const float scaled = scalbnf(v, -e);
  q = (uint8_t)__nv_cvt_float_to_fp8(scaled, __NV_SATFINITE, __NV_E4M3);
  const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)q, __NV_E4M3);
  back = scalbnf(__half2float(__half(hr)), e);
  sf = (uint32_t)(e + 127);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One warp per (token slot p, 32-block kb); rows of x come from src[rows[p]] (p < ntok).
template <int NMAX>
__global__ void __launch_bounds__(256) k_bsplit(const uint16_t *__restrict__ src, const int *__restrict__ rows,
                                                int ntok, int K, uint8_t *__restrict__ Bg,
                                                uint32_t *__restrict__ Bsf) {
  const int lane = threadIdx.x & 31;
  const int nb = K >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  for (int wi = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; wi < (NMAX / 2) * nb; wi += nwarps) {
    const int p = wi / nb, kb = wi - p * nb;
    float v = 0.f;
    if (p < ntok) {
      const int r = rows ? rows[p] : p;
      v = __uint_as_float((uint32_t)src[(size_t)r * K + kb * 32 + lane] << 16);
    }
    uint8_t qh, ql;
    uint32_t sfh, sfl;
    float bh, bl;
    split_e4m3(v, warp_max(fabsf(v)), qh, sfh, bh);
    const float res = v - bh;
    split_e4m3(res, warp_max(fabsf(res)), ql, sfl, bl);
    const int s = kb >> 2, kin = (kb & 3) * 32 + kpos_of_weight(lane);
    uint8_t *stage = Bg + (size_t)s * NMAX * 128;
    stage[kmajor_off(2 * p, kin)] = qh;
    stage[kmajor_off(2 * p + 1, kin)] = ql;
    if (lane < 2) {
      const int n = 2 * p + lane;
      uint8_t *sfbytes = reinterpret_cast<uint8_t *>(Bsf + ((size_t)s * 32 + (n & 31)) * 2 + (n >> 5));
      sfbytes[kb & 3] = (uint8_t)(lane == 0 ? sfh : sfl);
    }
  }
}

// ------------------------------------------------------------------------------- geometry

// Shared memory: barriers | A ring (kNA x 16 KB) | B ring (kNB x NMAX*128) | trellis-word ring
// (kPref x 256 threads x 16 B) | B-scale ring (kPref x 128 threads x 8 B) | 2 scale slabs.
struct MmaGeom {
  uint32_t off_A, off_B, off_C, off_F, off_S, slab, smem;
};

__host__ __device__ inline MmaGeom mma_geom(int nbr, int NMAX) {
  MmaGeom g;
  g.off_A = 1024u;
  g.off_B = g.off_A + kNA * 16384u;
  g.off_C = g.off_B + kNB * (uint32_t)NMAX * 128u;
  g.off_F = g.off_C + kPref * kDec * 16u;
  g.off_S = g.off_F + kPref * 128u * 8u;
  g.slab = round_up(128u * (uint32_t)nbr, 16u);
  g.smem = g.off_S + 2u * g.slab;
  return g;
}

__device__ __forceinline__ void cp_async8(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts_u2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

// ------------------------------------------------------------------------------- fused GEMV

template <int NMAX>
__global__ void __launch_bounds__(kMmaThreads, 1) k_mma_gemv(MatView w, const uint8_t *__restrict__ Bg,
                                                             const uint32_t *__restrict__ Bsf, int T,
                                                             uint16_t *__restrict__ y) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbr = w.nbr, S = (nbr + 3) >> 2;
  const MmaGeom geo = mma_geom(nbr, NMAX);
  uint64_t *a_full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *a_empty = a_full + 4, *b_full = a_full + 8, *b_empty = a_full + 16, *acc_full = a_full + 24,
           *acc_empty = a_full + 26;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 256);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + 260);
  unsigned int *tmo = &g_tcf4_timeouts_mma;

  const int ntiles = (w.rows + 127) >> 7;
  const int my_tiles = (int)blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int nq = my_tiles * S;

  if (tid == 0) {
    for (int b = 0; b < kNA; b++) {
      mbar_init(&a_full[b], 8);
      mbar_init(&a_empty[b], 1);
    }
    for (int b = 0; b < kNB; b++) {
      mbar_init(&b_full[b], 1);
      mbar_init(&b_empty[b], 1);
    }
    for (int a = 0; a < 2; a++) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp < 8) {
    // ---------------------------------------------------------------- decode warps
    const int sp = warp & 3, h = warp >> 2, m = 32 * sp + lane;
    const uint32_t cbase = smem_u32(smem + geo.off_C), fbase = smem_u32(smem + geo.off_F);
    auto issue = [&](int q) {
      if (q < nq) {
        const int tl = q / S, s = q - tl * S, tile = (int)blockIdx.x + tl * (int)gridDim.x;
        const int row = tile * 128 + m, kb0 = 4 * s + 2 * h;
        int nbv = nbr - kb0;
        nbv = nbv < 0 ? 0 : (nbv > 2 ? 2 : nbv);
        const uint32_t bytes = row < w.rows ? (uint32_t)nbv * 8u : 0u;
        const void *src = bytes ? static_cast<const void *>(w.stream + (size_t)row * nbr + kb0)
                                : static_cast<const void *>(w.stream);
        cp_async16(cbase + (uint32_t)((q % kPref) * kDec + tid) * 16u, src, bytes);
        if (warp < 4) cp_async8(fbase + (uint32_t)((q % kPref) * 128 + tid) * 8u, Bsf + ((size_t)s * 32 + lane) * 2);
        if (s == 0) {  // this tile's scale bytes, into slab buffer tl % 2
          const int r0 = tile * 128;
          const int nr = w.rows - r0 < 128 ? w.rows - r0 : 128;
          const uint32_t total = (uint32_t)nr * (uint32_t)nbr;
          const uint8_t *ssrc = w.scales + (size_t)r0 * nbr;
          const uint32_t sdst = smem_u32(smem + geo.off_S + (uint32_t)(tl & 1) * geo.slab);
          for (uint32_t c = tid; c * 16u < total; c += kDec)
            cp_async16(sdst + c * 16u, ssrc + c * 16u, total - c * 16u < 16u ? total - c * 16u : 16u);
        }
      }
      cp_async_commit();
    };
    auto epilogue = [&](int tl) {
      const int a = tl & 1;
      if (!mbar_wait(&acc_full[a], (uint32_t)(tl >> 1) & 1u, tmo)) *abort_flag = 1;
      tc_fence_after();
      const int row = ((int)blockIdx.x + tl * (int)gridDim.x) * 128 + 32 * warp + lane;
#pragma unroll
      for (int c0 = 0; c0 < NMAX; c0 += 16) {
        uint32_t r[16];
        tmem_ld_x16(tbase + ((uint32_t)(32 * warp) << 16) + (uint32_t)(a * NMAX + c0), r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; j++) {
          const int t = c0 / 2 + j;
          if (t < T && row < w.rows)
            y[(size_t)t * w.rows + row] =
                __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[2 * j]) + __uint_as_float(r[2 * j + 1])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
    };

    for (int q = 0; q < kPref; q++) issue(q);
    int q = 0;
    for (; q < nq; q++) {
      const int tl = q / S, s = q - tl * S;
      const int b = q % kNA;
      const uint32_t u = (uint32_t)(q / kNA);
      cp_async_wait<kPref - 1>();
      named_bar(1, kDec);
      if (*abort_flag) break;
      const uint4 cw = lds_u4(cbase + (uint32_t)((q % kPref) * kDec + tid) * 16u);
      uint2 sfb = make_uint2(0u, 0u);
      if (warp < 4) sfb = lds_u2(fbase + (uint32_t)((q % kPref) * 128 + tid) * 8u);
      issue(q + kPref);
      // decode the thread's two blocks into interleaved nibble words
      uint32_t A0[4], A1[4];
      planes_to_nibbles_interleaved(decode_block0(cw.x, cw.y), A0[0], A0[1], A0[2], A0[3]);
      planes_to_nibbles_interleaved(decode_block0(cw.z, cw.w), A1[0], A1[1], A1[2], A1[3]);
      uint32_t sfa[4] = {0u, 0u, 0u, 0u};
      if (warp < 4) {  // A scale factors: rows 32c + lane, K-blocks 4s..4s+3
        const uint32_t sb = smem_u32(smem + geo.off_S + (uint32_t)(tl & 1) * geo.slab);
        const int r0 = ((int)blockIdx.x + tl * (int)gridDim.x) * 128;
#pragma unroll
        for (int c = 0; c < 4; c++) {
          const int rl = 32 * c + lane;
          uint32_t word = 0u;
#pragma unroll
          for (int kb = 0; kb < 4; kb++) {
            const int j = 4 * s + kb;
            const uint32_t byte = (r0 + rl < w.rows && j < nbr) ? lds_u8(sb + (uint32_t)(rl * nbr + j)) : 127u;
            word |= byte << (8 * kb);
          }
          sfa[c] = word;
        }
      }
      if (u >= 1 && !mbar_wait(&a_empty[b], (u - 1u) & 1u, tmo)) *abort_flag = 1;
      const uint32_t abase = smem_u32(smem + geo.off_A + (uint32_t)b * 16384u) + (uint32_t)(m >> 3) * 1024u +
                             (uint32_t)(m & 7) * 16u;
      const uint32_t kb0 = 2u * (uint32_t)h;
      sts_u2(abase + (2u * kb0) * 128u, A0[0], A0[1]);
      sts_u2(abase + (2u * kb0 + 1u) * 128u, A0[2], A0[3]);
      sts_u2(abase + (2u * kb0 + 2u) * 128u, A1[0], A1[1]);
      sts_u2(abase + (2u * kb0 + 3u) * 128u, A1[2], A1[3]);
      if (warp < 4) {
        const uint32_t lane_addr = tbase + ((uint32_t)(32 * warp) << 16);
        tmem_st_x4(lane_addr + kSfaCol + 4u * b, sfa[0], sfa[1], sfa[2], sfa[3]);
        tmem_st_x2(lane_addr + kSfbCol + 4u * b, sfb.x, sfb.y);
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[b]);
      if (warp < 4 && tl >= 1 && s == 2) epilogue(tl - 1);
    }
    if (q == nq && warp < 4 && my_tiles >= 1) epilogue(my_tiles - 1);
    cp_async_wait_all();
  } else {
    // ---------------------------------------------------------------- control warp
    if (lane == 0) {
      const uint32_t bstage = (uint32_t)NMAX * 128u;
      auto issue_b = [&](int q) {
        if (q < nq) {
          const int s = q % S, bb = q % kNB;
          mbar_arrive_expect_tx(&b_full[bb], bstage);
          bulk_g2s(smem + geo.off_B + (uint32_t)bb * bstage, Bg + (size_t)s * bstage, bstage, &b_full[bb]);
        }
      };
      for (int q = 0; q < kNB; q++) issue_b(q);
      for (int q = 0; q < nq; q++) {
        const int tl = q / S, s = q - tl * S;
        const int b = q % kNA, bb = q % kNB;
        bool ok = mbar_wait(&a_full[b], (uint32_t)(q / kNA) & 1u, tmo);
        ok = ok && mbar_wait(&b_full[bb], (uint32_t)(q / kNB) & 1u, tmo);
        if (ok && s == 0 && tl >= 2) ok = mbar_wait(&acc_empty[tl & 1], (uint32_t)((tl >> 1) - 1) & 1u, tmo);
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const int nkb = nbr - 4 * s < 4 ? nbr - 4 * s : 4;
        const uint32_t a_s = smem_u32(smem + geo.off_A + (uint32_t)b * 16384u);
        const uint32_t b_s = smem_u32(smem + geo.off_B + (uint32_t)bb * bstage);
        const uint32_t d_t = tbase + (uint32_t)((tl & 1) * NMAX);
        for (int kb = 0; kb < nkb; kb++) {
          const uint64_t ad = smem_desc(a_s + 256u * kb, 128u, 1024u);
          const uint64_t bd = smem_desc(b_s + 256u * kb, 128u, 1024u);
          const uint32_t id = idesc_mxf8f6f4_e2m1_e4m3((uint32_t)NMAX, (uint32_t)kb, (uint32_t)kb);
          const uint32_t sfa_t = (tbase + kSfaCol + 4u * b) | ((uint32_t)kb << 30);
          const uint32_t sfb_t = (tbase + kSfbCol + 4u * b) | ((uint32_t)kb << 30);
          mma_mxf8f6f4(d_t, ad, bd, id, sfa_t, sfb_t, !(s == 0 && kb == 0));
        }
        tc_commit(&a_empty[b]);
        tc_commit(&b_empty[bb]);
        if (s == S - 1) tc_commit(&acc_full[tl & 1]);
        if (q >= 1 && q - 1 + kNB < nq) {
          if (!mbar_wait(&b_empty[(q - 1) % kNB], (uint32_t)((q - 1) / kNB) & 1u, tmo)) {
            *abort_flag = 1;
            break;
          }
          issue_b(q - 1 + kNB);
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

static int nmax_for(int T) { return 2 * T <= 16 ? 16 : (2 * T <= 32 ? 32 : 64); }

// The tensor-core path needs at least kPref K stages (K >= 1024), an even number of 32-blocks per
// row (16-byte aligned row starts), 16-byte aligned scales, and its buffers within shared memory.
bool gemv_mma_supported(const MatView &w, int T) {
  const int nbr = w.nbr;
  if (nbr < 4 * kPref || nbr % 2 != 0 || (reinterpret_cast<uintptr_t>(w.scales) & 15u) != 0) return false;
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
  return mma_geom(nbr, nmax_for(T)).smem <= (uint32_t)optin;
}

size_t gemv_mma_workspace(const MatView &w, int T) {
  const int S = (w.nbr + 3) / 4, NMAX = nmax_for(T);
  return (size_t)S * NMAX * 128 + (size_t)S * 32 * 8;
}

template <int NMAX>
static cudaError_t launch_mma_t(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s) {
  const int S = (w.nbr + 3) / 4;
  uint8_t *Bg = static_cast<uint8_t *>(ws);
  uint32_t *Bsf = reinterpret_cast<uint32_t *>(Bg + (size_t)S * NMAX * 128);
  const int warps = (NMAX / 2) * w.nbr;
  k_bsplit<NMAX><<<(warps + 7) / 8, 256, 0, s>>>(x, nullptr, T, w.nbr * 32, Bg, Bsf);
  static unsigned long long attr = 0;
  cudaError_t e = ensure_max_dynamic_smem(k_mma_gemv<NMAX>, attr);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = (w.rows + 127) / 128;
  const int grid = ntiles < nsm ? ntiles : nsm;
  const MmaGeom g = mma_geom(w.nbr, NMAX);
  k_mma_gemv<NMAX><<<grid, kMmaThreads, g.smem, s>>>(w, Bg, Bsf, T, y);
  return cudaGetLastError();
}

cudaError_t launch_gemv_mma(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s) {
  switch (nmax_for(T)) {
    case 16: return launch_mma_t<16>(w, x, T, y, ws, s);
    case 32: return launch_mma_t<32>(w, x, T, y, ws, s);
    default: return launch_mma_t<64>(w, x, T, y, ws, s);
  }
}

unsigned int take_timeouts_mma() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_tcf4_timeouts_mma, sizeof v) != cudaSuccess) return 0;
  cudaMemcpyToSymbol(g_tcf4_timeouts_mma, &zero, sizeof zero);
  return v;
}

}  // namespace tcf4
