// tcf4_internal.h -- launchers shared between the C-ABI layer and the kernel files.
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <utility>

#include "tcf4.h"

namespace tcf4 {

// Programmatic dependent launch. Every kernel of the library is launched with programmatic stream
// serialization. Each kernel calls grid_dep_wait before it touches anything a preceding kernel
// writes or still reads, and releases its successor (grid_dep_release) only after that wait: so a
// kernel overlaps at most its immediate predecessor, and only with work that depends on nothing in
// flight (launch latency, setup, loads of resident weights).
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... P, typename... A>
inline cudaError_t launch_dependent(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                    A &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

constexpr int kMaxExperts = 256;
constexpr int kMaxTokens = 32;
constexpr int kMaxTopK = 8;
constexpr int kMaxCols = 16384;

// Device-side view of one trellis-coded matrix.
struct MatView {
  const uint2 *stream;    // [rows][nbr] block words (lo plane, hi plane)
  const uint8_t *scales;  // [rows][nbr]
  int32_t rows;
  int32_t nbr;            // blocks per row = cols / 32
  int32_t seg_blocks;     // seg_len / 32
};

// Per-expert pointer table passed by value to the MoE kernels.
template <int MAXE>
struct MoeTable {
  const uint2 *gu[MAXE];
  const uint8_t *gus[MAXE];
  const uint2 *dn[MAXE];
  const uint8_t *dns[MAXE];
};

// Offsets of the MoE workspace regions (bytes, 256-aligned): per-row-chunk counters of the down
// kernel, h (bf16 [T*k][I]) and y (fp32 [T*k][H]).
struct MoeWorkspace {
  size_t counters, hidden, y, total;
};
MoeWorkspace moe_workspace_layout(int E, int T, int k, int H, int I);

// Allow a kernel the largest dynamic shared memory the device offers beyond its static shared
// memory, once per device (a bit per device ordinal in `done`).
template <class F>
cudaError_t ensure_max_dynamic_smem(F *func, unsigned long long &done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done & bit) return cudaSuccess;
  cudaFuncAttributes a;
  e = cudaFuncGetAttributes(&a, func);
  if (e != cudaSuccess) return e;
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)a.sharedSizeBytes);
  if (e == cudaSuccess) done |= bit;
  return e;
}

cudaError_t launch_expand(const MatView &w, uint8_t *out_nibbles, uint8_t *out_scales, cudaStream_t s);
// Interleaved -> planar stream words of nblocks 32-weight blocks (in == out allowed).
cudaError_t launch_repack(const uint32_t *in, uint32_t *out, uint32_t nblocks, cudaStream_t s);
// CUDA-core fused decode GEMV; e5m3: the scale bytes are E5M3 block scales instead of UE8M0.
cudaError_t launch_gemv(const MatView &w, const uint16_t *x, int T, uint16_t *y, cudaStream_t s, bool e5m3 = false);
cudaError_t launch_route(const float *logits, int T, int E, int k, int32_t *ids, float *wts, cudaStream_t s);
cudaError_t launch_moe(const tcf4_moe &m, int gu_seg, int dn_seg, const uint16_t *x, int T, const int32_t *ids,
                       const float *wts, int k, uint16_t *out, void *ws, cudaStream_t s);

// Tensor-core fused decode GEMV (k_mma.cu): whether it applies, its workspace, its launch.
bool gemv_mma_supported(const MatView &w, int T);
size_t gemv_mma_workspace(const MatView &w, int T);
cudaError_t launch_gemv_mma(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s);
// The same with the weights' scales as scale tiles (k_mma.cu): their size, the rearranging kernel,
// whether the tiled path applies, its launch (workspace as for launch_gemv_mma).
size_t scale_tiles_bytes(const MatView &w);
cudaError_t launch_scale_tiles(const MatView &w, uint8_t *tiles, cudaStream_t s);
bool gemv_tiled_supported(const MatView &w, const uint8_t *tiles, int T);
cudaError_t launch_gemv_tiled(const MatView &w, const uint8_t *tiles, const uint16_t *x, int T, uint16_t *y, void *ws,
                              cudaStream_t s);

// Tensor-core grouped MoE (k_mma.cu): workspace regions (bytes, 256-aligned): the down kernel's
// counters (4 per 128-row chunk of H), h (bf16 [T*k][I]), y (fp32 [T*k][H]), the activation terms
// of the gate_up and down passes, and per-CTA tensor-map slots.
struct MoeMmaWorkspace {
  size_t counters, hidden, y, bg_gu, bg_dn, maps, total;
};
bool moe_mma_supported(const tcf4_moe &m, int gu_seg, int dn_seg, int T);
// D-weighted Viterbi encoder (k_encode.cu): back-pointer bytes of one CTA, the workspace for one
// segment per SM, and the launch (as many concurrent segments as ws_bytes holds, at most one per SM).
size_t encode_cta_bytes(int seg);
size_t encode_workspace(int rows, int cols, int seg);
cudaError_t launch_encode(const double *target, const double *D, const uint8_t *scales, int rows, int cols, int seg,
                          uint32_t *out_stream, double *out_cost, void *ws, size_t ws_bytes, cudaStream_t s);
// Resident MXFP4 consumers (the tensor-core kernel reading nibble tiles): the views' stream fields
// point at the nibble matrices [rows][cols/2]. Workspaces are the same as the trellis paths'.
bool mx_gemv_supported(const MatView &w, int T);
size_t mx_gemv_workspace(const MatView &w, int T);
// E5M3 block scales on the tensor cores (k_mma.cu, four UE8M0 scale sets per block).
bool gemv_e5m3_mma_supported(const MatView &w, int T);
size_t gemv_e5m3_mma_workspace(const MatView &w, int T);
cudaError_t launch_gemv_e5m3_mma(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s);
cudaError_t launch_mx_gemv(const MatView &w, const uint16_t *x, int T, uint16_t *y, void *ws, cudaStream_t s);
bool moe_mx_supported(const tcf4_moe &m, int T);
cudaError_t launch_moe_mx(const tcf4_moe &m, const uint16_t *x, int T, const int32_t *ids, const float *wts, int k,
                          uint16_t *out, void *ws, cudaStream_t s);
MoeMmaWorkspace moe_mma_workspace_layout(const tcf4_moe &m, int T, int k);
cudaError_t launch_moe_mma(const tcf4_moe &m, const uint16_t *x, int T, const int32_t *ids, const float *wts, int k,
                           uint16_t *out, void *ws, cudaStream_t s);

// Read and clear the bounded-wait timeout counters of the kernel files.
unsigned int take_timeouts_gemv();
unsigned int take_timeouts_moe();
unsigned int take_timeouts_mma();

}  // namespace tcf4
