// tcf4_api.cu -- the extern "C" entry points declared in include/tcf4.h.
//
// Validates every argument on the host before any launch, converts the public descriptors into
// device views, and dispatches to the kernels. No allocation, no synchronisation.
#include <cuda_runtime.h>

#include <cstdint>

#include "tcf4.h"
#include "tcf4_internal.h"

using namespace tcf4;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

tcf4_status check_matrix(const tcf4_matrix &w) {
  if (w.rows < 0 || w.cols < 0) return TCF4_ERR_INVALID_ARG;
  if (w.cols % 32 != 0) return TCF4_ERR_INVALID_ARG;
  if (w.rows == 0 || w.cols == 0) return TCF4_OK;
  if (w.stream == nullptr || w.scales == nullptr) return TCF4_ERR_INVALID_ARG;
  if (w.seg_len <= 0 || w.seg_len % 32 != 0 || w.cols % w.seg_len != 0) return TCF4_ERR_INVALID_ARG;
  if (!aligned16(w.stream)) return TCF4_ERR_MISALIGNED;
  if (w.rows > INT32_MAX || w.cols / 32 > INT32_MAX) return TCF4_ERR_UNSUPPORTED;
  return TCF4_OK;
}

MatView view(const tcf4_matrix &w) {
  MatView v;
  v.stream = reinterpret_cast<const uint2 *>(w.stream);
  v.scales = w.scales;
  v.rows = (int32_t)w.rows;
  v.nbr = (int32_t)(w.cols / 32);
  v.seg_blocks = w.seg_len / 32;
  return v;
}

tcf4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TCF4_OK : TCF4_ERR_CUDA; }

tcf4_status check_mx(const tcf4_mxfp4 &w) {
  if (w.rows < 0 || w.cols < 0 || w.cols % 32 != 0) return TCF4_ERR_INVALID_ARG;
  if (w.rows == 0 || w.cols == 0) return TCF4_OK;
  if (w.nibbles == nullptr || w.scales == nullptr) return TCF4_ERR_INVALID_ARG;
  if (!aligned16(w.nibbles) || (reinterpret_cast<uintptr_t>(w.scales) & 1u) != 0) return TCF4_ERR_MISALIGNED;
  if (w.cols % 64 != 0 || w.cols > kMaxCols || w.rows > INT32_MAX) return TCF4_ERR_UNSUPPORTED;
  return TCF4_OK;
}

// The MXFP4 consumers reuse the trellis views: stream points at the nibble matrix.
MatView mx_view(const tcf4_mxfp4 &w) {
  MatView v;
  v.stream = reinterpret_cast<const uint2 *>(w.nibbles);
  v.scales = w.scales;
  v.rows = (int32_t)w.rows;
  v.nbr = (int32_t)(w.cols / 32);
  v.seg_blocks = 1;
  return v;
}

tcf4_matrix mx_as_matrix(const tcf4_mxfp4 &w) {
  tcf4_matrix m;
  m.stream = reinterpret_cast<const uint32_t *>(w.nibbles);
  m.scales = w.scales;
  m.rows = w.rows;
  m.cols = w.cols;
  m.seg_len = 32;
  return m;
}

// A non-sticky error left pending by earlier, unrelated CUDA calls would otherwise be reported
// as this call's launch failure; clear it before launching (documented in tcf4.h).
void clear_pending_error() { (void)cudaGetLastError(); }

}  // namespace

extern "C" {

const char *tcf4_status_string(tcf4_status s) {
  switch (s) {
    case TCF4_OK: return "ok";
    case TCF4_ERR_INVALID_ARG: return "invalid argument";
    case TCF4_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case TCF4_ERR_UNSUPPORTED: return "size beyond the supported limits";
    case TCF4_ERR_WORKSPACE: return "workspace missing or too small";
    case TCF4_ERR_CUDA: return "CUDA launch failed";
  }
  return "unknown status";
}

tcf4_status trellis_decode_to_mxfp4(tcf4_matrix w, uint8_t *out_nibbles, uint8_t *out_scales, void *stream) {
  tcf4_status st = check_matrix(w);
  if (st != TCF4_OK) return st;
  if (w.rows == 0 || w.cols == 0) return TCF4_OK;
  if (out_nibbles == nullptr || out_scales == nullptr) return TCF4_ERR_INVALID_ARG;
  if (!aligned16(out_nibbles)) return TCF4_ERR_MISALIGNED;
  if (w.rows * (w.cols / 32) >= ((int64_t)1 << 31)) return TCF4_ERR_UNSUPPORTED;
  clear_pending_error();
  return from_cuda(launch_expand(view(w), out_nibbles, out_scales, static_cast<cudaStream_t>(stream)));
}

tcf4_status trellis_repack_interleaved(const uint32_t *in, int64_t rows, int64_t cols, uint32_t *out, void *stream) {
  if (rows < 0 || cols < 0 || cols % 32 != 0) return TCF4_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return TCF4_OK;
  if (in == nullptr || out == nullptr) return TCF4_ERR_INVALID_ARG;
  const uintptr_t ib = reinterpret_cast<uintptr_t>(in), ob = reinterpret_cast<uintptr_t>(out);
  if (((ib | ob) & 7u) != 0) return TCF4_ERR_MISALIGNED;
  if (rows > INT32_MAX || cols / 32 > INT32_MAX || rows * (cols / 32) >= ((int64_t)1 << 31))
    return TCF4_ERR_UNSUPPORTED;
  const int64_t nblocks = rows * (cols / 32);
  const uintptr_t nbytes = (uintptr_t)nblocks * 8u;
  if (ib != ob && ib < ob + nbytes && ob < ib + nbytes) return TCF4_ERR_INVALID_ARG;
  clear_pending_error();
  return from_cuda(launch_repack(in, out, (uint32_t)nblocks, static_cast<cudaStream_t>(stream)));
}

static tcf4_status check_gemv(const tcf4_matrix &w, int32_t T) {
  tcf4_status st = check_matrix(w);
  if (st != TCF4_OK) return st;
  if (T < 0) return TCF4_ERR_INVALID_ARG;
  if (T == 0 || w.rows == 0) return TCF4_OK;
  if (T > kMaxTokens) return TCF4_ERR_UNSUPPORTED;
  if (w.cols == 0) return TCF4_ERR_INVALID_ARG;
  if (w.cols > kMaxCols) return TCF4_ERR_UNSUPPORTED;
  return TCF4_OK;
}

// The tensor-core path runs whenever it applies (any seg_len; see gemv_mma_supported); it needs
// the workspace for the activation split. Other shapes run the CUDA-core kernel without one.
static bool gemv_uses_mma(const tcf4_matrix &w, int32_t T) {
  return w.rows > 0 && T > 0 && gemv_mma_supported(view(w), T);
}

size_t trellis_gemv_workspace(tcf4_matrix w, int32_t T) {
  if (check_gemv(w, T) != TCF4_OK || T == 0 || w.rows == 0) return 0;
  return gemv_uses_mma(w, T) ? gemv_mma_workspace(view(w), T) : 0;
}

tcf4_status trellis_gemv(tcf4_matrix w, const uint16_t *x, int32_t T, uint16_t *y, void *workspace,
                         size_t ws_bytes, void *stream) {
  tcf4_status st = check_gemv(w, T);
  if (st != TCF4_OK) return st;
  if (T == 0 || w.rows == 0) return TCF4_OK;
  if (x == nullptr || y == nullptr) return TCF4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return TCF4_ERR_MISALIGNED;
  const MatView v = view(w);
  if (gemv_uses_mma(w, T)) {
    if (workspace == nullptr || ws_bytes < gemv_mma_workspace(v, T)) return TCF4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TCF4_ERR_MISALIGNED;
    clear_pending_error();
    return from_cuda(launch_gemv_mma(v, x, T, y, workspace, static_cast<cudaStream_t>(stream)));
  }
  clear_pending_error();
  return from_cuda(launch_gemv(v, x, T, y, static_cast<cudaStream_t>(stream)));
}

size_t trellis_scale_tiles_bytes(tcf4_matrix w) {
  if (check_matrix(w) != TCF4_OK || w.rows == 0 || w.cols == 0) return 0;
  return scale_tiles_bytes(view(w));
}

tcf4_status trellis_make_scale_tiles(tcf4_matrix w, uint8_t *tiles, void *stream) {
  tcf4_status st = check_matrix(w);
  if (st != TCF4_OK) return st;
  if (w.rows == 0 || w.cols == 0) return TCF4_OK;
  if (tiles == nullptr) return TCF4_ERR_INVALID_ARG;
  if (!aligned16(tiles)) return TCF4_ERR_MISALIGNED;
  if (scale_tiles_bytes(view(w)) / 4 >= ((size_t)1 << 31)) return TCF4_ERR_UNSUPPORTED;
  clear_pending_error();
  return from_cuda(launch_scale_tiles(view(w), tiles, static_cast<cudaStream_t>(stream)));
}

tcf4_status trellis_gemv_tiled(tcf4_matrix w, const uint8_t *tiles, const uint16_t *x, int32_t T, uint16_t *y,
                               void *workspace, size_t ws_bytes, void *stream) {
  tcf4_matrix wc = w;
  if (wc.scales == nullptr) wc.scales = tiles;  // the raw scales are not read here
  tcf4_status st = check_gemv(wc, T);
  if (st != TCF4_OK) return st;
  if (T == 0 || w.rows == 0) return TCF4_OK;
  if (x == nullptr || y == nullptr || tiles == nullptr) return TCF4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y) || !aligned16(tiles)) return TCF4_ERR_MISALIGNED;
  const MatView v = view(wc);
  if (!gemv_tiled_supported(v, tiles, T)) return TCF4_ERR_UNSUPPORTED;
  if (workspace == nullptr || ws_bytes < gemv_mma_workspace(v, T)) return TCF4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TCF4_ERR_MISALIGNED;
  clear_pending_error();
  return from_cuda(launch_gemv_tiled(v, tiles, x, T, y, workspace, static_cast<cudaStream_t>(stream)));
}

static bool gemv_e5m3_uses_mma(const tcf4_matrix &w, int32_t T) {
  return w.rows > 0 && T > 0 && gemv_e5m3_mma_supported(view(w), T);
}

size_t trellis_gemv_e5m3_workspace(tcf4_matrix w, int32_t T) {
  if (check_gemv(w, T) != TCF4_OK || T == 0 || w.rows == 0) return 0;
  return gemv_e5m3_uses_mma(w, T) ? gemv_e5m3_mma_workspace(view(w), T) : 0;
}

tcf4_status trellis_gemv_e5m3(tcf4_matrix w, const uint16_t *x, int32_t T, uint16_t *y, void *workspace,
                              size_t ws_bytes, void *stream) {
  tcf4_status st = check_gemv(w, T);
  if (st != TCF4_OK) return st;
  if (T == 0 || w.rows == 0) return TCF4_OK;
  if (x == nullptr || y == nullptr) return TCF4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return TCF4_ERR_MISALIGNED;
  const MatView v = view(w);
  if (gemv_e5m3_uses_mma(w, T)) {
    if (workspace == nullptr || ws_bytes < gemv_e5m3_mma_workspace(v, T)) return TCF4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TCF4_ERR_MISALIGNED;
    clear_pending_error();
    return from_cuda(launch_gemv_e5m3_mma(v, x, T, y, workspace, static_cast<cudaStream_t>(stream)));
  }
  clear_pending_error();
  return from_cuda(launch_gemv(v, x, T, y, static_cast<cudaStream_t>(stream), true));
}

tcf4_status trellis_moe_route(const float *logits, int32_t T, int32_t E, int32_t k, int32_t *topk_ids,
                              float *topk_w, void *stream) {
  if (T < 0 || k < 1 || E < k) return TCF4_ERR_INVALID_ARG;
  if (T == 0) return TCF4_OK;
  if (k > kMaxTopK || E > kMaxExperts || T > kMaxTokens) return TCF4_ERR_UNSUPPORTED;
  if (logits == nullptr || topk_ids == nullptr || topk_w == nullptr) return TCF4_ERR_INVALID_ARG;
  clear_pending_error();
  return from_cuda(launch_route(logits, T, E, k, topk_ids, topk_w, static_cast<cudaStream_t>(stream)));
}

static tcf4_status check_moe(const tcf4_moe *m, int32_t T, int32_t k, int *gu_seg, int *dn_seg) {
  if (m == nullptr || m->gate_up == nullptr || m->down == nullptr) return TCF4_ERR_INVALID_ARG;
  if (m->E < 1 || m->H < 32 || m->I < 32 || m->H % 32 != 0 || m->I % 32 != 0) return TCF4_ERR_INVALID_ARG;
  if (T < 0 || k < 1 || k > m->E) return TCF4_ERR_INVALID_ARG;
  if (m->E > kMaxExperts || k > kMaxTopK || T > kMaxTokens || m->H > kMaxCols || m->I > kMaxCols)
    return TCF4_ERR_UNSUPPORTED;
  *gu_seg = m->gate_up[0].seg_len / 32;
  *dn_seg = m->down[0].seg_len / 32;
  for (int e = 0; e < m->E; e++) {
    const tcf4_matrix &g = m->gate_up[e], &d = m->down[e];
    if (g.rows != 2 * (int64_t)m->I || g.cols != m->H) return TCF4_ERR_INVALID_ARG;
    if (d.rows != m->H || d.cols != m->I) return TCF4_ERR_INVALID_ARG;
    tcf4_status s1 = check_matrix(g), s2 = check_matrix(d);
    if (s1 != TCF4_OK) return s1;
    if (s2 != TCF4_OK) return s2;
    if (g.seg_len / 32 != *gu_seg || d.seg_len / 32 != *dn_seg) return TCF4_ERR_UNSUPPORTED;
  }
  return TCF4_OK;
}

// The tensor-core MoE runs whenever it applies (see moe_mma_supported); otherwise the CUDA-core
// kernels do. The workspace layout follows the path.
static bool moe_uses_mma(const tcf4_moe *m, int gu_seg, int dn_seg, int32_t T) {
  return T > 0 && moe_mma_supported(*m, gu_seg, dn_seg, T);
}

size_t trellis_grouped_moe_workspace(const tcf4_moe *m, int32_t T, int32_t k) {
  int a, b;
  if (check_moe(m, T, k, &a, &b) != TCF4_OK) return 0;
  if (moe_uses_mma(m, a, b, T)) return moe_mma_workspace_layout(*m, T, k).total;
  return moe_workspace_layout(m->E, T, k, m->H, m->I).total;
}

size_t trellis_grouped_moe_hidden_offset(const tcf4_moe *m, int32_t T, int32_t k) {
  int a, b;
  if (check_moe(m, T, k, &a, &b) != TCF4_OK) return 0;
  if (moe_uses_mma(m, a, b, T)) return moe_mma_workspace_layout(*m, T, k).hidden;
  return moe_workspace_layout(m->E, T, k, m->H, m->I).hidden;
}

tcf4_status trellis_grouped_moe(const tcf4_moe *m, const uint16_t *x, int32_t T, const int32_t *topk_ids,
                                const float *topk_w, int32_t k, uint16_t *out, void *workspace, size_t ws_bytes,
                                void *stream) {
  int gu_seg = 1, dn_seg = 1;
  tcf4_status st = check_moe(m, T, k, &gu_seg, &dn_seg);
  if (st != TCF4_OK) return st;
  if (T == 0) return TCF4_OK;
  if (x == nullptr || topk_ids == nullptr || topk_w == nullptr || out == nullptr) return TCF4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return TCF4_ERR_MISALIGNED;
  const bool mma = moe_uses_mma(m, gu_seg, dn_seg, T);
  const size_t need = mma ? moe_mma_workspace_layout(*m, T, k).total : moe_workspace_layout(m->E, T, k, m->H, m->I).total;
  if (workspace == nullptr || ws_bytes < need) return TCF4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TCF4_ERR_MISALIGNED;
  clear_pending_error();
  if (mma)
    return from_cuda(launch_moe_mma(*m, x, T, topk_ids, topk_w, k, out, workspace, static_cast<cudaStream_t>(stream)));
  return from_cuda(launch_moe(*m, gu_seg, dn_seg, x, T, topk_ids, topk_w, k, out, workspace,
                              static_cast<cudaStream_t>(stream)));
}

size_t mxfp4_gemv_workspace(tcf4_mxfp4 w, int32_t T) {
  if (check_mx(w) != TCF4_OK || T <= 0 || T > kMaxTokens || w.rows == 0 || w.cols == 0) return 0;
  return mx_gemv_workspace(mx_view(w), T);
}

tcf4_status mxfp4_gemv(tcf4_mxfp4 w, const uint16_t *x, int32_t T, uint16_t *y, void *workspace, size_t ws_bytes,
                       void *stream) {
  tcf4_status st = check_mx(w);
  if (st != TCF4_OK) return st;
  if (T < 0) return TCF4_ERR_INVALID_ARG;
  if (T == 0 || w.rows == 0) return TCF4_OK;
  if (T > kMaxTokens) return TCF4_ERR_UNSUPPORTED;
  if (w.cols == 0) return TCF4_ERR_INVALID_ARG;
  if (x == nullptr || y == nullptr) return TCF4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return TCF4_ERR_MISALIGNED;
  const MatView v = mx_view(w);
  if (!mx_gemv_supported(v, T)) return TCF4_ERR_UNSUPPORTED;
  if (workspace == nullptr || ws_bytes < mx_gemv_workspace(v, T)) return TCF4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TCF4_ERR_MISALIGNED;
  clear_pending_error();
  return from_cuda(launch_mx_gemv(v, x, T, y, workspace, static_cast<cudaStream_t>(stream)));
}

// The layer as a tcf4_moe whose stream fields point at the nibble matrices (host arrays of this
// thread, valid until its next MXFP4 MoE call).
static tcf4_status mx_moe_view(const tcf4_mxfp4_moe *m, int32_t T, int32_t k, tcf4_moe *out) {
  static thread_local tcf4_matrix gu[kMaxExperts], dn[kMaxExperts];
  if (m == nullptr || m->gate_up == nullptr || m->down == nullptr) return TCF4_ERR_INVALID_ARG;
  if (m->E < 1 || m->H < 32 || m->I < 32 || m->H % 32 != 0 || m->I % 32 != 0) return TCF4_ERR_INVALID_ARG;
  if (T < 0 || k < 1 || k > m->E) return TCF4_ERR_INVALID_ARG;
  if (m->E > kMaxExperts || k > kMaxTopK || T > kMaxTokens || m->H > kMaxCols || m->I > kMaxCols)
    return TCF4_ERR_UNSUPPORTED;
  for (int e = 0; e < m->E; e++) {
    const tcf4_mxfp4 &g = m->gate_up[e], &d = m->down[e];
    if (g.rows != 2 * (int64_t)m->I || g.cols != m->H || d.rows != m->H || d.cols != m->I) return TCF4_ERR_INVALID_ARG;
    tcf4_status s1 = check_mx(g), s2 = check_mx(d);
    if (s1 != TCF4_OK) return s1;
    if (s2 != TCF4_OK) return s2;
    gu[e] = mx_as_matrix(g);
    dn[e] = mx_as_matrix(d);
  }
  out->gate_up = gu;
  out->down = dn;
  out->E = m->E;
  out->H = m->H;
  out->I = m->I;
  return TCF4_OK;
}

size_t mxfp4_grouped_moe_workspace(const tcf4_mxfp4_moe *m, int32_t T, int32_t k) {
  tcf4_moe v;
  if (mx_moe_view(m, T, k, &v) != TCF4_OK || T == 0) return 0;
  return moe_mma_workspace_layout(v, T, k).total;
}

size_t mxfp4_grouped_moe_hidden_offset(const tcf4_mxfp4_moe *m, int32_t T, int32_t k) {
  tcf4_moe v;
  if (mx_moe_view(m, T, k, &v) != TCF4_OK || T == 0) return 0;
  return moe_mma_workspace_layout(v, T, k).hidden;
}

tcf4_status mxfp4_grouped_moe(const tcf4_mxfp4_moe *m, const uint16_t *x, int32_t T, const int32_t *topk_ids,
                              const float *topk_w, int32_t k, uint16_t *out, void *workspace, size_t ws_bytes,
                              void *stream) {
  tcf4_moe v;
  tcf4_status st = mx_moe_view(m, T, k, &v);
  if (st != TCF4_OK) return st;
  if (T == 0) return TCF4_OK;
  if (x == nullptr || topk_ids == nullptr || topk_w == nullptr || out == nullptr) return TCF4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return TCF4_ERR_MISALIGNED;
  if (!moe_mx_supported(v, T)) return TCF4_ERR_UNSUPPORTED;
  if (workspace == nullptr || ws_bytes < moe_mma_workspace_layout(v, T, k).total) return TCF4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TCF4_ERR_MISALIGNED;
  clear_pending_error();
  return from_cuda(launch_moe_mx(v, x, T, topk_ids, topk_w, k, out, workspace, static_cast<cudaStream_t>(stream)));
}

static tcf4_status check_encode(int64_t rows, int64_t cols, int32_t seg_len) {
  if (rows < 0 || cols < 0 || cols % 32 != 0) return TCF4_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return TCF4_OK;
  if (seg_len <= 0 || seg_len % 32 != 0 || cols % seg_len != 0) return TCF4_ERR_INVALID_ARG;
  if (rows * cols >= ((int64_t)1 << 31)) return TCF4_ERR_UNSUPPORTED;
  return TCF4_OK;
}

size_t trellis_encode_workspace(int64_t rows, int64_t cols, int32_t seg_len) {
  if (check_encode(rows, cols, seg_len) != TCF4_OK || rows == 0 || cols == 0) return 0;
  return encode_workspace((int)rows, (int)cols, seg_len);
}

tcf4_status trellis_encode(const double *target, const double *D, const uint8_t *scales, int64_t rows, int64_t cols,
                           int32_t seg_len, uint32_t *stream_out, double *cost_out, void *workspace, size_t ws_bytes,
                           void *stream) {
  tcf4_status st = check_encode(rows, cols, seg_len);
  if (st != TCF4_OK) return st;
  if (rows == 0 || cols == 0) return TCF4_OK;
  if (target == nullptr || D == nullptr || scales == nullptr || stream_out == nullptr) return TCF4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(target) | reinterpret_cast<uintptr_t>(D)) & 7u) return TCF4_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(stream_out) & 7u) || (reinterpret_cast<uintptr_t>(cost_out) & 7u))
    return TCF4_ERR_MISALIGNED;
  if (workspace == nullptr || ws_bytes < encode_cta_bytes(seg_len)) return TCF4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TCF4_ERR_MISALIGNED;
  clear_pending_error();
  return from_cuda(launch_encode(target, D, scales, (int)rows, (int)cols, seg_len, stream_out, cost_out, workspace,
                                 ws_bytes, static_cast<cudaStream_t>(stream)));
}

unsigned int tcf4_device_timeouts(void) {
  cudaDeviceSynchronize();
  return take_timeouts_gemv() + take_timeouts_moe() + take_timeouts_mma();
}

}  // extern "C"
