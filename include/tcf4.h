/*
 * tcf4.h -- C ABI of the trellis-coded FP4 (XOR-Trellis / HEPH) decode library for B200.
 *
 * The library decodes weights stored as an XOR-Trellis bitstream ("XOR-Trellis: Hadamard-free
 * FP4 LLM quantization" news page, bullet "XOR-Trellis FP4 decoder": 16-bit sliding state, four
 * masked parities 0x1089/0x2112/0x0A24/0x2441 giving p0,p1,q0,q1, palettes P0..P3) under HEPH's
 * grid-aligned convention ("HEPH: 3-Bit Grid-Aligned Trellis Quantization of MXFP4
 * Mixture-of-Experts ...", abstract): each decoded weight is an E2M1 value times its 32-weight
 * block's UE8M0 scale 2^(E-127), i.e. a valid MXFP4 element. HEPH serves such weights in two
 * modes, both exported here: the stream stays resident and is decoded inside the product kernels
 * (trellis_gemv, trellis_grouped_moe), or it is expanded once into a resident packed MXFP4 tensor
 * (trellis_decode_to_mxfp4).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout. A matrix W is [rows][cols] row-major, cols % 32 == 0, scales run along cols.
 *   stream: uint32 [rows][cols/32][2]; for 32-weight block j of row n, word 0 holds the low bit
 *           and word 1 the high bit of the 2-bit branch symbols (bit i = symbol 32j+i).
 *   scales: uint8 [rows][cols/32], UE8M0 (value 2^(E-127); 0xFF is NaN and propagates).
 *   seg_len: the trellis state is 0 at the start of every seg_len-weight segment of a row;
 *           seg_len is a positive multiple of 32 that divides cols (32 = one MXFP4 block).
 *   Decoder reading: the new symbol b enters the state at bits 14-15 (s = s>>2 | b<<14);
 *   p = p0 + 2*p1 picks the palette, q = q0 + 2*q1, entry = b XOR q; P3's zero is -0.
 *   Activations and outputs are bf16 passed as their uint16 bit patterns.
 * Memory. Every data pointer is DEVICE memory owned by the caller. The library never allocates,
 *   frees or synchronizes; every call is asynchronous on `stream` (a cudaStream_t, NULL = the
 *   legacy default stream). Inputs must stay valid until the work on `stream` completes.
 * Alignment. stream, x and y pointers must be 16-byte aligned; MXFP4 outputs too.
 * Errors. Arguments are checked on the host before anything is launched: a bad argument returns
 *   TCF4_ERR_INVALID_ARG / TCF4_ERR_MISALIGNED / TCF4_ERR_UNSUPPORTED / TCF4_ERR_WORKSPACE and
 *   launches nothing. A valid call first clears a pending non-sticky CUDA error left by earlier
 *   calls (cudaGetLastError), so that it is not mistaken for its own; a failed launch then returns
 *   TCF4_ERR_CUDA with the CUDA error left set for the caller to read. Empty problems (rows == 0,
 *   T == 0) return TCF4_OK and launch nothing.
 * Stream order. Kernels are launched as programmatic dependents of the preceding work on the
 *   stream: each waits for its predecessor before it reads what that predecessor may write (x,
 *   routing, workspace) or writes what it may still read (y, workspace). The product kernels read
 *   their weights (stream words, scales, scale tiles, MXFP4 nibbles) before that wait, while the
 *   preceding kernel may still run; the weights must therefore be complete when the call is
 *   enqueued, or be written by work that has completed by then in stream order without releasing
 *   its dependents early. The library's own weight-writing calls (trellis_repack_interleaved,
 *   trellis_make_scale_tiles, trellis_decode_to_mxfp4, trellis_encode) release no dependents
 *   early, so a product call right after one of them reads the finished weights.
 * Threads. Calls are reentrant. The only process state the library writes is a one-time
 *   per-device kernel attribute (the dynamic shared-memory limit of its kernels).
 */
#ifndef TCF4_H
#define TCF4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TCF4_API __attribute__((visibility("default")))
#else
#define TCF4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TCF4_OK = 0,
  TCF4_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, cols % 32, bad seg_len, bad k/E/T */
  TCF4_ERR_MISALIGNED = 2,   /* a pointer that must be 16-byte aligned is not */
  TCF4_ERR_UNSUPPORTED = 3,  /* a size beyond the limits stated below */
  TCF4_ERR_WORKSPACE = 4,    /* workspace missing or smaller than trellis_grouped_moe_workspace */
  TCF4_ERR_CUDA = 5          /* a kernel launch failed */
} tcf4_status;

/* One trellis-coded matrix (all pointers device memory). */
typedef struct {
  const uint32_t *stream; /* [rows][cols/32][2] planar trellis words */
  const uint8_t *scales;  /* [rows][cols/32] UE8M0 block scales */
  int64_t rows;
  int64_t cols;           /* multiple of 32 */
  int32_t seg_len;        /* multiple of 32 dividing cols */
} tcf4_matrix;

/* HEPH abstract, second serving mode: expand the stream into a resident packed MXFP4 tensor.
 *   out_nibbles: uint8 [rows][cols/2]; byte u of a row holds element 2u in its low nibble and
 *                element 2u+1 in its high nibble (OCP E2M1 codes, sign in bit 3).
 *   out_scales:  uint8 [rows][cols/32], a byte-for-byte copy of w.scales.
 * Bit-exact with the decoder definition. out_nibbles must be 16-byte aligned. */
TCF4_API tcf4_status trellis_decode_to_mxfp4(tcf4_matrix w, uint8_t *out_nibbles, uint8_t *out_scales,
                                    void *stream);

/* The second stream packing: each row one bit string, symbol k at bits 2k (its low bit) and 2k+1
 * (its high bit), LSB-first in 32-bit words, so block j of a row owns words 2j (its symbols 0..15)
 * and 2j+1 (symbols 16..31). The XOR-Trellis page's 16-bit sliding state ("XOR-Trellis FP4
 * decoder" bullet) is then a window of that string. Every other call here reads the planar packing
 * (tcf4_matrix.stream); this call converts, bit for bit, once at load time.
 *   in:  uint32 [rows][cols/32][2] interleaved words (device); out: the same shape, planar words.
 *   in == out converts in place; otherwise the two buffers must not overlap (TCF4_ERR_INVALID_ARG).
 *   Both pointers 8-byte aligned (TCF4_ERR_MISALIGNED); 32-byte alignment of both takes the widest
 *   accesses. rows * cols / 32 < 2^31 (TCF4_ERR_UNSUPPORTED). rows or cols 0: nothing to do. */
TCF4_API tcf4_status trellis_repack_interleaved(const uint32_t *in, int64_t rows, int64_t cols, uint32_t *out,
                                                void *stream);

/* HEPH abstract, first serving mode: fused decode + product.
 *   y[t][n] = bf16( sum_k w[n][k] * x[t][k] ), fp32 accumulation, round to nearest even.
 *   x: bf16 bits [T][cols]; y: bf16 bits [T][rows]; 1 <= T <= 32 (T == 0 is a no-op).
 * Two kernels behind one call: when cols is a multiple of 64 (any seg_len; segments longer than a
 * block carry the trellis state from block to block) and the scales are 2-byte aligned, the product
 * runs on the tensor cores (block-scaled MXFP4 x MXFP4 MMA: each 32-block of x is written as a sum of six
 * E2M1 terms with their own UE8M0 scales, which leaves at most 5^-6 of the block's largest |x|
 * unrepresented) and needs `workspace`; otherwise it runs on CUDA cores and needs none.
 * trellis_gemv_workspace tells which (0 bytes = none needed).
 *   workspace: device scratch of at least trellis_gemv_workspace(w, T) bytes, 256-byte aligned,
 *   owned by the caller (may be NULL when that size is 0).
 * Accuracy: |y - exact| <= 2e-3 * ||w_row||_2 * ||x_t||_2 per output plus the bf16 rounding.
 * Limits: cols <= 16384. */
TCF4_API size_t trellis_gemv_workspace(tcf4_matrix w, int32_t T);
TCF4_API tcf4_status trellis_gemv(tcf4_matrix w, const uint16_t *x, int32_t T, uint16_t *y, void *workspace,
                                  size_t ws_bytes, void *stream);

/* Scale tiles: the weights' UE8M0 scales rearranged once, at load time, into the layout the tensor
 * cores' scale-factor copies read (HEPH abstract, first serving mode: the grid-aligned scale of each
 * 32-weight block; the bytes are the same, only their order changes). For 128-row tile t and
 * 4-block group g (g < 8 * ceil(cols / 1024), a whole number of 32-block stages per tile) a
 * 512-byte tile at byte offset (t * groups + g) * 512 whose byte 16 r + 4 q + i is the scale of
 * row 128 t + 32 q + r, block 4 g + i, or 0 past the matrix.
 *   trellis_scale_tiles_bytes: the size (0 for an invalid or empty matrix).
 *   trellis_make_scale_tiles: writes them from w.scales; tiles 16-byte aligned, caller-owned. */
TCF4_API size_t trellis_scale_tiles_bytes(tcf4_matrix w);
TCF4_API tcf4_status trellis_make_scale_tiles(tcf4_matrix w, uint8_t *tiles, void *stream);

/* trellis_gemv with the weights' scales read from scale tiles (w.scales is not read and may be
 * NULL). Same result, accuracy, workspace (trellis_gemv_workspace) and limits as trellis_gemv, on
 * the tensor-core path only: cols a multiple of 64 and tiles 16-byte aligned, else
 * TCF4_ERR_UNSUPPORTED. The decode then does no scale work: the scale tiles of each stage are
 * bulk-copied beside its stream words and moved to the tensor memory by the MMA issuers. */
TCF4_API tcf4_status trellis_gemv_tiled(tcf4_matrix w, const uint8_t *tiles, const uint16_t *x, int32_t T,
                                        uint16_t *y, void *workspace, size_t ws_bytes, void *stream);

/* The XOR-Trellis news page's grouping format: E2M1 elements with E5M3 block scales (its paragraph
 * on the format; no encoding given). w.scales holds one E5M3 byte per 32-weight block, read as: no
 * sign bit, exponent bits 7..3 with bias 15, mantissa bits 2..0, exponent 0 subnormal (2^-14 m/8),
 * exponent 31 NaN. Otherwise as trellis_gemv: y[t][n] = bf16( sum_k w[n][k] * x[t][k] ), same
 * shapes, alignment, limits and accuracy bound, and the same two paths. On the tensor cores (cols a
 * multiple of 64) each E5M3 scale is written as the sum of at most four powers of two (the implicit
 * bit and each set significand bit), so a block's product is four block-scaled MMAs of the same
 * decoded weights, one per power; an absent power adds the block's product times 2^-127. That path
 * needs trellis_gemv_e5m3_workspace(w, T) bytes of workspace (256-byte aligned, caller-owned);
 * otherwise the CUDA-core kernel scales each block's partial sum once and needs none (0 bytes). */
TCF4_API size_t trellis_gemv_e5m3_workspace(tcf4_matrix w, int32_t T);
TCF4_API tcf4_status trellis_gemv_e5m3(tcf4_matrix w, const uint16_t *x, int32_t T, uint16_t *y, void *workspace,
                                       size_t ws_bytes, void *stream);

/* trellis_gemv without a caller-provided workspace (the source pages have no counterpart; this is
 * a convenience of this library). Same arguments, result and accuracy as trellis_gemv.
 * For callers that cannot hand over device scratch memory: a host program that holds only the
 * device pointers it was given and has no device allocator of its own, or a serving loop that must
 * not allocate while it runs because its memory was reserved up front.
 * The scratch is one 2 MiB array per device, inside this library. Every call looks up that array's
 * address on the current device through the CUDA runtime (nothing is cached, so the address stays
 * right after a cudaDeviceReset). The first lookup on a device may load the library's module there,
 * so make the first call on each device before beginning any stream capture. All calls on a device
 * share the array and leave in it whatever they last wrote; nothing in it has to start at zero, as
 * each call writes the scratch it reads. Calls that overlap in time on one device (other streams or
 * host threads) race on the array: the caller must serialize them.
 * Returns TCF4_ERR_WORKSPACE when the call would need more than 2 MiB of scratch (not reached
 * within the limits of trellis_gemv), TCF4_ERR_CUDA when the address lookup fails. */
TCF4_API tcf4_status trellis_gemv_noalloc(tcf4_matrix w, const uint16_t *x, int32_t T, uint16_t *y, void *stream);

/* Router for the MoE layer: for each token, the k experts with the largest logits (ties to the
 * lower expert index) and softmax weights over those k logits (fp32).
 *   logits: fp32 [T][E]; topk_ids: int32 [T][k]; topk_w: fp32 [T][k].
 * Non-finite logits: a NaN ranks below every number (-inf included), so k valid ids in [0, E)
 * always come out, and weighs as -inf. When a token's largest selected logit is -inf all its
 * weights are 0; when it is +inf the +inf logits share the weight equally.
 * Limits: 1 <= k <= 8, k <= E <= 256, T <= 32. */
TCF4_API tcf4_status trellis_moe_route(const float *logits, int32_t T, int32_t E, int32_t k, int32_t *topk_ids,
                              float *topk_w, void *stream);

/* One MoE layer: E experts, hidden size H, intermediate size I.
 *   gate_up: HOST array of E descriptors, each [2I][H] (gate rows 0..I-1, up rows I..2I-1);
 *   down:    HOST array of E descriptors, each [H][I].
 * All gate_up matrices share one seg_len, and all down matrices share one seg_len. The host
 * arrays are read during the call only. */
typedef struct {
  const tcf4_matrix *gate_up;
  const tcf4_matrix *down;
  int32_t E;
  int32_t H;
  int32_t I;
} tcf4_moe;

/* Bytes of device workspace trellis_grouped_moe needs for T tokens and top-k routing
 * (0 when the arguments are invalid). */
TCF4_API size_t trellis_grouped_moe_workspace(const tcf4_moe *m, int32_t T, int32_t k);

/* HEPH abstract, first serving mode for a routed MoE layer: for every token t and every selected
 * expert j = topk_ids[t][*]: g,u = gate_up_j . x_t, h = bf16(silu(g) * u), y_j = down_j . h, and
 *   out[t] = bf16( sum_j topk_w[t][j] * y_j )   (fp32 accumulation and combine).
 * Tokens routed to the same expert share one decode of its weights.
 *   x: bf16 bits [T][H]; topk_ids: int32 [T][k] (device); topk_w: fp32 [T][k] (device);
 *   out: bf16 bits [T][H]; workspace: device scratch of at least
 *   trellis_grouped_moe_workspace(m, T, k) bytes, 256-byte aligned, owned by the caller.
 * After the call the workspace holds, among other things, h as bf16 [T*k][I] in (t, j) order at
 * offset trellis_grouped_moe_hidden_offset(m, T, k).
 * Limits: 1 <= T <= 32, 1 <= k <= 8, E <= 256, H and I <= 16384. Expert ids outside [0, E) in
 * topk_ids make the affected (t, j) contribute nothing. */
TCF4_API tcf4_status trellis_grouped_moe(const tcf4_moe *m, const uint16_t *x, int32_t T, const int32_t *topk_ids,
                                const float *topk_w, int32_t k, uint16_t *out, void *workspace,
                                size_t ws_bytes, void *stream);

/* Byte offset of h (bf16 [T*k][I]) inside the workspace of trellis_grouped_moe. */
TCF4_API size_t trellis_grouped_moe_hidden_offset(const tcf4_moe *m, int32_t T, int32_t k);

/* ------------------------------------------------------------------------------------------------
 * HEPH abstract, second serving mode, consumer side: products straight from the resident MXFP4
 * tensor that trellis_decode_to_mxfp4 writes (expand once, then every product reads 4.25 bits per
 * weight with no decode). Same operations and accuracy contract as trellis_gemv and
 * trellis_grouped_moe, on the tensor cores (block-scaled MXFP4 x MXFP4 MMA with the activations
 * written as six E2M1 terms per 32-block; the same workspaces).
 * ------------------------------------------------------------------------------------------------ */

/* One resident MXFP4 matrix W [rows][cols]:
 *   nibbles: uint8 [rows][cols/2], byte u of a row holds element 2u in its low nibble and element
 *            2u+1 in its high nibble (OCP E2M1 codes); 16-byte aligned.
 *   scales:  uint8 [rows][cols/32] UE8M0, element k of a row scaled by 2^(scales[k/32] - 127);
 *            2-byte aligned.
 *   cols:    a multiple of 64 (whole K = 64 MMAs), at most 16384. Device memory owned by the
 *            caller. */
typedef struct {
  const uint8_t *nibbles;
  const uint8_t *scales;
  int64_t rows;
  int64_t cols;
} tcf4_mxfp4;

/* y[t][n] = bf16( sum_k w[n][k] * x[t][k] ), fp32 accumulation; x bf16 bits [T][cols], y bf16 bits
 * [T][rows], 1 <= T <= 32 (T == 0 is a no-op); x and y 16-byte aligned.
 *   workspace: device scratch of at least mxfp4_gemv_workspace(w, T) bytes, 256-byte aligned, owned
 *   by the caller. Accuracy: |y - exact| <= 2e-3 * ||w_row||_2 * ||x_t||_2 plus the bf16 rounding.
 * Errors: TCF4_ERR_UNSUPPORTED when cols is not a multiple of 64 or exceeds 16384, or when T > 32;
 * TCF4_ERR_MISALIGNED for pointers that break the alignment above. */
TCF4_API size_t mxfp4_gemv_workspace(tcf4_mxfp4 w, int32_t T);
TCF4_API tcf4_status mxfp4_gemv(tcf4_mxfp4 w, const uint16_t *x, int32_t T, uint16_t *y, void *workspace,
                                size_t ws_bytes, void *stream);

/* A routed MoE layer of resident MXFP4 experts: gate_up[e] is [2I][H] (gate rows 0..I-1, up rows
 * I..2I-1), down[e] is [H][I]; host arrays of E descriptors. */
typedef struct {
  const tcf4_mxfp4 *gate_up;
  const tcf4_mxfp4 *down;
  int32_t E;
  int32_t H;
  int32_t I;
} tcf4_mxfp4_moe;

/* The same layer computation as trellis_grouped_moe (SwiGLU between gate/up and down, fp32
 * combine of the k routed experts, bf16 out) from resident MXFP4 experts. Limits: 1 <= T <= 32,
 * 1 <= k <= 8, E <= 256, H and I multiples of 64 up to 16384. The workspace holds h as bf16
 * [T*k][I] in (t, j) order at offset mxfp4_grouped_moe_hidden_offset(m, T, k) after the call. */
TCF4_API size_t mxfp4_grouped_moe_workspace(const tcf4_mxfp4_moe *m, int32_t T, int32_t k);
TCF4_API size_t mxfp4_grouped_moe_hidden_offset(const tcf4_mxfp4_moe *m, int32_t T, int32_t k);
TCF4_API tcf4_status mxfp4_grouped_moe(const tcf4_mxfp4_moe *m, const uint16_t *x, int32_t T,
                                       const int32_t *topk_ids, const float *topk_w, int32_t k, uint16_t *out,
                                       void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------------------------------
 * The upstream (offline) step: "XOR-Trellis: Hadamard-free FP4 LLM quantization" news page, bullet
 * "Curvature-aware Viterbi objective". Each segment of seg_len weights of a row is encoded as the
 * trellis path, starting in state 0 and ending in any state, that minimises
 *   sum_k D[k] * (target[k] - value_k * 2^(E_k - 127))^2
 * where value_k is the palette value of the state after symbol k (the decoder of trellis_gemv) and
 * E_k the UE8M0 scale byte of weight k's 32-block (chosen by the caller, e.g. the grid-aligned
 * convention: the block's own MXFP4 exponent). The sum is evaluated in fp64, term by term in that
 * order with no fused operations. Among equal-cost paths the lower predecessor window (the 7
 * previous symbols read as a number, newest symbol in the top bits) wins at each step, and the
 * lowest final window at the end.
 *   target, D:  fp64 [rows][cols], device.       scales: uint8 [rows][cols/32], device.
 *   stream_out: uint32 [rows][cols/32][2] planar words (the layout of tcf4_matrix.stream), device.
 *   cost_out:   fp64 [rows][cols/seg_len], the minimum of each segment, device (may be NULL).
 *   workspace:  device scratch; trellis_encode_workspace(rows, cols, seg_len) bytes run one segment
 *               per SM at a time, fewer bytes (at least seg_len * 4 KiB) fewer segments. 256-byte
 *               aligned, owned by the caller.
 * Compute-bound: 2^16 candidate paths per weight. Limits: cols a multiple of 32, seg_len a
 * multiple of 32 dividing cols, rows * cols < 2^31. */
TCF4_API size_t trellis_encode_workspace(int64_t rows, int64_t cols, int32_t seg_len);
TCF4_API tcf4_status trellis_encode(const double *target, const double *D, const uint8_t *scales, int64_t rows,
                                    int64_t cols, int32_t seg_len, uint32_t *stream_out, double *cost_out,
                                    void *workspace, size_t ws_bytes, void *stream);

/* Bounded waits that gave up inside the library's kernels since the last call, then resets the
 * count. Kernels that stage weights with bulk copies wait on shared-memory barriers with an
 * iteration limit; a wait that runs out is counted and the affected outputs are invalid. Never
 * expected in a correct run. Synchronous: it waits for the current device's work to finish. */
TCF4_API unsigned int tcf4_device_timeouts(void);

/* A static, human-readable description of a status code. */
TCF4_API const char *tcf4_status_string(tcf4_status s);

#ifdef __cplusplus
}
#endif

#endif /* TCF4_H */
