/*
 * mxc.h -- C ABI of the MXCode W4A4 linear-layer library for NVIDIA B200 (sm_100a).
 *
 * Method: "MXCode: Vector Quantization for MX-Native Inference at Scale".
 * Weights are stored at about 2 bits each: a uint8 index per d=4 consecutive
 * weights along the input-channel axis selects one of K=256 FP4 (E2M1)
 * centroids of the weight's QBlock (abstract; Table 4 caption), and the
 * centroid's codes are scaled by MX block scales (Table 1): E8M0 per 32
 * weights, or E4M3 per 16 weights with an FP32 tensor scale.  PostScale and
 * PreScale store the block scales directly; PreScale+ VQ-codes groups of 8
 * scales with a 256-entry scale codebook (Table 4 caption).  The library
 * decodes indices straight into MX-native FP4 operand tiles in shared memory
 * and multiplies them with FP4-quantized activations on the tcgen05
 * block-scaled tensor cores (W4A4, abstract and Table 2 caption); it never
 * materialises BF16 weights.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Ownership: the caller allocates and owns every buffer and the stream.
 *   The library keeps no allocation of its own apart from one 4-byte device
 *   error word per device (a module global).  Pointers marked "device" must be
 *   device memory of the current device; "host" pointers are host memory.
 * - Asynchrony: GPU calls enqueue work on the given stream and return.  They
 *   do not synchronize.  Argument, shape and alignment problems are reported
 *   synchronously by the return value and nothing is enqueued.
 * - Programmatic dependent launch: mxc_quantize_act (M*K <= 16*8192) and the
 *   M <= 16 path of mxc_linear / mxc_native_linear let the next kernel of the
 *   stream start early, and the decode path loads and decodes its weight
 *   buffers before waiting for the previous kernel.  Weight buffers are
 *   therefore constants of the stream: they must not be written by a kernel
 *   that itself launches with programmatic dependent launch right before the
 *   call (host copies, ordinary kernels, this library's packing and decode
 *   calls are fine).  Activation, scale and output buffers follow plain stream
 *   order.
 * - Device-side problems (malformed MoE offsets, a pipeline wait that ran
 *   out) set the device error word; read it with mxc_get_device_error().
 * - No exception crosses this ABI; every entry point returns mxc_status.
 * - Shapes: K (input channels) must be a multiple of 256, N (output channels)
 *   a multiple of 128.  Buffers passed to the GPU must be 16-byte aligned.
 *
 * Layouts
 * -------
 * FP4 matrix  [R, K] as bytes [R, ld] (ld >= K/2, ld % 16 == 0): byte i of a
 *             row holds elements 2i (low nibble) and 2i+1 (high nibble);
 *             nibble = E2M1 code, bit 3 = sign.
 * SF layout   block-scale bytes of an [R, K/B] scale matrix, grouped the way
 *             the tcgen05 block-scaled MMA reads them: rows are padded to a
 *             multiple of 128; byte (r, kb) sits at
 *                 ((r/128) * (K/B/4) + kb/4) * 512
 *               + (r%32) * 16 + ((r/32)%4) * 4 + (kb%4).
 *             mxc_sf_bytes(R, K, fmt) gives the size.
 * Packed VQ weight (mxc_pack_weight writes it; see mxc_weight below).
 */
#ifndef MXC_H_
#define MXC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mxc_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum mxc_status {
  MXC_OK = 0,
  MXC_ERR_INVALID_ARG = 1,    /* null pointer, bad enum, inconsistent shapes        */
  MXC_ERR_UNSUPPORTED = 2,    /* e.g. the UE5M3 scale format, or M beyond limits    */
  MXC_ERR_ALIGNMENT = 3,      /* K % 256, N % 128, QBlock sizes, 16-byte pointers   */
  MXC_ERR_WORKSPACE = 4,      /* workspace missing or smaller than required         */
  MXC_ERR_CUDA = 5,           /* a CUDA runtime/driver call failed                  */
  MXC_ERR_DEVICE_INVALID = 6, /* device found malformed data (e.g. MoE offsets)     */
  MXC_ERR_TIMEOUT = 7,        /* a bounded pipeline wait on the device expired      */
  MXC_ERR_NO_DEVICE = 8       /* no sm_100 device is current                         */
} mxc_status;

/* Block-scaled FP4 formats (Table 1).  UE5M3-B16 has no native tensor-core
 * path on this GPU and is rejected with MXC_ERR_UNSUPPORTED. */
typedef enum mxc_format {
  MXC_FMT_E8M0_B32 = 0, /* E8M0 scale per 32 elements, no tensor scale          */
  MXC_FMT_E4M3_B16 = 1, /* E4M3 scale per 16 elements, FP32 tensor scale        */
  MXC_FMT_UE5M3_B16 = 2 /* not supported                                        */
} mxc_format;

/* MXCode strategies (abstract).  PostScale and PreScale share one decode path
 * (the Figure 4 and Table 3 captions describe a single FP4 projection backend
 * serving both); the strategy only selects where block scales come from. */
typedef enum mxc_strategy {
  MXC_POSTSCALE = 0,     /* direct block scales                                */
  MXC_PRESCALE = 1,      /* direct block scales                                */
  MXC_PRESCALE_PLUS = 2, /* VQ-coded block scales (groups of 8, 256 entries)   */
  MXC_POSTSCALE_QB = 3   /* PostScale with one scale per QBlock: the codebook's
                            own MX scale, shared by every block of the QBlock
                            (the 2.06 / 2.25 bits per weight of Table 2)       */
} mxc_strategy;

typedef enum mxc_dtype { MXC_OUT_F32 = 0, MXC_OUT_BF16 = 1 } mxc_dtype;

/* An MX-quantized matrix: FP4 codes + block scales (+ FP32 tensor scale).
 * Activations are passed this way, and so are native-FP4 weights. */
typedef struct mxc_mx_tensor {
  const uint8_t* q;      /* device, FP4 matrix [rows, ldq bytes]                      */
  const uint8_t* sf;     /* device, SF layout (see above) of the [rows, K/B] scales    */
  const float* tscale;   /* device, one FP32 tensor scale; NULL means 1.0              */
  int64_t rows;          /* M for activations, N for native weights                    */
  int64_t K;             /* elements per row                                           */
  int64_t ldq;           /* row stride of q in bytes                                   */
  mxc_format fmt;
} mxc_mx_tensor;

/* A VQ-coded weight W[N, K] in the packed device layout.
 *   idx     device, [N/128][K/256][4][128][16] bytes: each 128-row x 256-column
 *           tile (8 KB, tiles in row-major tile order) holds four K-quarter slabs
 *           of 64 input channels; slab c holds, for each of the 128 rows, its 16
 *           uint8 indices (index j covers k = 256 ks + 64 c + 4j .. + 3).
 *   cb      device, [N/qn][K/qk][256] uint16 FP4 codebooks; centroid element t
 *           (k mod 4) in bits 4t..4t+3.  512 bytes per QBlock.
 *   scales  device (PostScale/PreScale), SF layout of the [N, K/B] scale bytes;
 *           (MXC_POSTSCALE_QB) [N/qn][K/qk] bytes, one scale per QBlock.
 *   sidx    device (PreScale+), [N/128][U][128][G] bytes: the scale-codebook index
 *           of each group of ds consecutive block scales along K (ds = scale_group).
 *           With ds*B <= 256 a unit is one 256-channel stage holding G = 256/(ds*B)
 *           groups of each row (U = K/256); with ds*B > 256 a unit is one group
 *           (G = 1, U = K/(ds*B)).  Either way U*G = K/(ds*B).
 *   scb     device (PreScale+), [256][ds] scale bytes.
 *   qn, qk  QBlock size; 0 means the whole dimension.  qn must be 64 or a
 *           multiple of 128 (or N); qk must be 64, 128 or a multiple of 256 (or K).
 *           QBlocks of 64 rows or 64 input channels (down to 64 x 64, the fine end
 *           of Figure 3's sweep) are decoded once per call into the workspace and
 *           run on the native GEMM at every M (see mxc_linear_workspace_bytes_for);
 *           the grouped (MoE) calls do not take them.
 *   w_tscale  FP32 tensor scale (E4M3-B16); use 1.0 for E8M0-B32.
 *   scale_group  PreScale+: ds, the block scales one scale index covers (Table 4
 *           caption: 8; 16 and 32 are Figure 3's higher scale-compression ratios);
 *           0 means 8.  K must be a multiple of ds*B.  Ignored by other strategies. */
typedef struct mxc_weight {
  mxc_strategy strategy;
  mxc_format fmt;
  int64_t N, K, qn, qk;
  const uint8_t* idx;
  const uint16_t* cb;
  const uint8_t* scales;
  const uint8_t* sidx;
  const uint8_t* scb;
  float w_tscale;
  int32_t scale_group;
} mxc_weight;

/* The same weight in its logical host layout, as produced by a quantizer:
 *   idx [N, K/4] uint8, cb [N/qn, K/qk, 256] uint16, scales [N, K/B] uint8
 *   (direct), [N/qn, K/qk] uint8 (PostScale-QB), or sidx [N, K/(ds*B)] uint8 +
 *   scb [256, ds] uint8 (PreScale+, ds = scale_group). */
typedef struct mxc_weight_host {
  mxc_strategy strategy;
  mxc_format fmt;
  int64_t N, K, qn, qk;
  const uint8_t* idx;
  const uint16_t* cb;
  const uint8_t* scales;
  const uint8_t* sidx;
  const uint8_t* scb;
  float w_tscale;
  int32_t scale_group;
} mxc_weight_host;

/* Byte sizes of the packed buffers (host-side arithmetic only). */
typedef struct mxc_packed_sizes {
  size_t idx, cb, scales, sidx, scb;
} mxc_packed_sizes;

/* ---- version / status ------------------------------------------------------------- */

const char* mxc_status_string(mxc_status s);
int mxc_version(void); /* 100 * major + minor */

/* ---- host-side layout helpers (no GPU needed) ------------------------------------ */

/* Bytes of an SF-layout buffer for an [rows, K/B] scale matrix (rows padded to 128). */
size_t mxc_sf_bytes(int64_t rows, int64_t K, mxc_format fmt);

/* Sizes of the packed buffers of a weight.  Returns MXC_ERR_* for bad shapes. */
mxc_status mxc_packed_weight_sizes(const mxc_weight_host* w, mxc_packed_sizes* out);

/* Reorders a logical host weight into the packed layout, host to host.
 * idx_out, scales_out (direct) or sidx_out (PreScale+) must hold the sizes
 * that mxc_packed_weight_sizes() reports; cb and scb are used as they are
 * (their logical layout is already the packed one).  Unused outputs may be
 * NULL.  Pure host code: safe without a GPU. */
mxc_status mxc_pack_weight(const mxc_weight_host* w, uint8_t* idx_out, uint8_t* scales_out,
                           uint8_t* sidx_out);

/* Workspace bytes each GPU call needs (0 if none).  M = activation rows;
 * for mxc_moe_linear M is the total number of (token, expert) rows.
 * mxc_linear: a workspace it uses starts with 4 KiB of split-K arrival counters,
 * which only the split-K below touches and which every call leaves zero: zero a
 * workspace once after allocating it, and it stays valid whichever mxc_linear /
 * mxc_native_linear calls use it.  Up to 16 rows, when the 128-row output tiles are
 * split along K into more than two ranks (ranks s = min(4, 148 / (N/128)), at
 * least 1) or into slices longer than 2048 input channels: the counters, then
 * N/128 x R x 8 KiB of FP32 partial tiles, R = the fewest ranks (at least s, at
 * most 16) whose slices are at most 2048 input channels long, provided
 * N/128 x R <= 148 (one CTA per SM) and N/128 <= 1024; else 0.  Without that room
 * the call runs on split-K clusters (slower for those shapes), not an error.  17
 * to 128 rows (128-token tiles of the fused kernel), when N/128 <= 1024 and the
 * 128-row output tiles can be split along K into R = min(4, 148 / (N/128), K/256)
 * >= 2 ranks (R recomputed as the number of slices of ceil(K/256 / R) stages): the
 * counters, then N/128 x R x 64 KiB of FP32 partial tiles; else 0.  Without that
 * room the call runs one CTA per output tile (slower), not an error.  The
 * partials are added in rank order, so a result depends on the room given, not on
 * timing.  Above 128 rows when N is a multiple of 256 (else from 1024
 * rows): the counters, then the room for the weight decoded once per call (N*K/2
 * bytes of FP4 codes rounded up to 1 KiB, then N*K/B bytes of SF-layout scales).
 * A smaller workspace is not an error there: the call then runs the fused
 * decode-in-GEMM kernel, which is slower at those sizes.
 * mxc_moe_linear and mxc_moe_gate_up_swiglu: the expert tile and chunk tables,
 * 2 (E+1) int32 rounded up to whole 256-byte units. */
size_t mxc_quantize_act_workspace_bytes(int64_t M, int64_t K, mxc_format fmt);
size_t mxc_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, mxc_format fmt);
size_t mxc_moe_workspace_bytes(int64_t M, int32_t E, int64_t N, int64_t K, mxc_format fmt);
/* The workspace mxc_linear needs for this weight at M rows: mxc_linear_workspace_bytes,
 * except for QBlocks of 64 rows or 64 input channels, which need the decoded weight's
 * room (N*K/2 rounded up to 1 KiB, plus N*K/B) after the counter area at every M --
 * without it mxc_linear returns MXC_ERR_WORKSPACE for them -- followed, up to 16
 * rows, by the split-K partial tiles described above.  0 for an invalid weight. */
size_t mxc_linear_workspace_bytes_for(const mxc_weight* w, int64_t M);

/* Rows of the SF layout that mxc_quantize_act_grouped writes:
 * sum over groups of ceil(rows_g / 128) * 128, bounded by M + 128*E. */
int64_t mxc_grouped_sf_rows_bound(int64_t M, int32_t E);

/* ---- GPU calls ----------------------------------------------------------------------- */

/* Activation MX quantization, BF16 -> FP4 codes + block scales (W4A4: abstract,
 * Table 2 caption; formats: Table 1).  Rule (the pages give none; OCP MX):
 *   E8M0-B32: per block of 32, e = floor(log2 amax) - 2 clamped to [-127,127]
 *             (amax = 0 -> byte 0), codes = RNE_E2M1(x / 2^e) saturating at +-6.
 *   E4M3-B16: s = amax_tensor / 2688 in FP32 (1 if amax = 0), unless
 *             act_tscale_in gives it; per block of 16,
 *             sb = E4M3_RNE_satfinite(fp32(fp32(amax/6) / s)),
 *             codes = RNE_E2M1(x / fp32(sb * s)) decided exactly; sb = 0 -> +-0.
 *   Signs are kept, so -0 becomes code 0x8.  NaN/Inf inputs are undefined.
 * x_bf16        device, [M, ldx] BF16 elements (ldx >= K)
 * act_tscale_in device FP32 or NULL (E4M3 only; ignored for E8M0)
 * q_out         device, FP4 matrix [M, ldq] (ldq >= K/2, multiple of 16)
 * sf_out        device, SF layout, mxc_sf_bytes(M, K, fmt) bytes; padding rows get 0
 * act_tscale_out device FP32 (E4M3: receives s; may be NULL for E8M0)
 * ws            device workspace of mxc_quantize_act_workspace_bytes() bytes */
mxc_status mxc_quantize_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, mxc_format fmt,
                            const float* act_tscale_in, uint8_t* q_out, int64_t ldq, uint8_t* sf_out,
                            float* act_tscale_out, void* ws, size_t ws_bytes, mxc_stream_t stream);

/* As mxc_quantize_act for rows sorted by group (MoE experts): row r belongs to
 * group g when d_offsets[g] <= r < d_offsets[g+1].  q_out is dense [M, ldq];
 * sf_out places each group's scale rows at the next multiple of 128 rows
 * (mxc_grouped_sf_rows_bound(M, E) rows are enough), which is what
 * mxc_moe_linear reads.  d_offsets is device int32 [E+1], offsets[0] = 0,
 * non-decreasing, offsets[E] = M; violations set MXC_ERR_DEVICE_INVALID. */
mxc_status mxc_quantize_act_grouped(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                    mxc_format fmt, const int32_t* d_offsets, int32_t E,
                                    const float* act_tscale_in, uint8_t* q_out, int64_t ldq,
                                    uint8_t* sf_out, float* act_tscale_out, void* ws,
                                    size_t ws_bytes, mxc_stream_t stream);

/* MXCode W4A4 linear layer: y[M, N] = A[M, K] . W[N, K]^T, where A is the
 * MX-quantized activation and W the VQ weight reconstructed on the fly (the
 * abstract's point: the VQ storage becomes MX-native FP4 operands directly, with
 * no high-precision copy of the weight in between).  Accumulation is FP32 on the
 * tensor cores; y = acc * w_tscale * a_tscale, written as FP32 or BF16 (RNE).
 * a         activation, a->fmt must equal w->fmt; a->rows = M; a->sf in SF layout
 * w         packed VQ weight (device pointers inside)
 * y         device, [M, ldy] elements of y_dtype (ldy >= N)
 * ws        device workspace of mxc_linear_workspace_bytes() bytes (16-byte aligned)
 * M <= 16 takes the split-K decode path; larger M the tiled prefill path, which
 * decodes each weight tile inside the GEMM (17 to 128 rows: split along K through
 * the workspace when it has the room, see mxc_linear_workspace_bytes).  Above 128 rows when N is a multiple
 * of 256 (else from 1024 rows), with the workspace given, the call instead decodes
 * the weight once into it (MX-native FP4 codes and scales, the output of
 * mxc_decode_weight) and runs the native block-scaled GEMM on that: the same
 * operands in the same K order, so the same result bits. */
mxc_status mxc_linear(const mxc_mx_tensor* a, const mxc_weight* w, void* y, int64_t ldy,
                      mxc_dtype y_dtype, void* ws, size_t ws_bytes, mxc_stream_t stream);

/* Native block-scaled FP4 linear layer on the same pipeline, with the weight
 * given as an MX tensor (w->rows = N): the "Native FP4" baseline of Table 2
 * and Table 3.  Same output contract as mxc_linear. */
mxc_status mxc_native_linear(const mxc_mx_tensor* a, const mxc_mx_tensor* w, void* y, int64_t ldy,
                             mxc_dtype y_dtype, void* ws, size_t ws_bytes, mxc_stream_t stream);

/* Grouped-expert (MoE) MXCode linear: rows of `a` are sorted by expert, expert e
 * owning rows [d_offsets[e], d_offsets[e+1]); y[r, :] = A[r, :] . W_e^T.  The
 * weights are MoE expert tensors, as in the paper's evaluation (Table 4 caption:
 * the VQ-coded tensors are the experts of Qwen3's MoE layers); every expert is a
 * VQ weight of the same shape and coding.
 * a         quantized with mxc_quantize_act_grouped (grouped SF layout)
 * d_offsets device int32 [E+1] (validated on the device)
 * experts   host array of E packed weights that share strategy, format, N, K,
 *           qn, qk (their device pointers may differ); E <= 256, larger E
 *           returns MXC_ERR_UNSUPPORTED
 * y         device, [M, ldy]
 * ws        device workspace of mxc_moe_workspace_bytes() bytes
 * Checks, in this order: the activation (INVALID_ARG / ALIGNMENT / UNSUPPORTED),
 * null pointers and E <= 0 (INVALID_ARG), E > 256 (UNSUPPORTED), each expert
 * weight, consistency with the activation, the output, then the device
 * (NO_DEVICE) and the workspace (WORKSPACE). */
mxc_status mxc_moe_linear(const mxc_mx_tensor* a, const int32_t* d_offsets, const mxc_weight* experts,
                          int32_t E, void* y, int64_t ldy, mxc_dtype y_dtype, void* ws,
                          size_t ws_bytes, mxc_stream_t stream);

/* The gate/up projection of a MoE layer fused with SwiGLU and with the MX
 * quantization of its result, which is the down projection's W4A4 activation
 * (the experts are Qwen3's MoE FFN tensors: Table 4 caption).  Each expert's
 * gate/up weight is [2F, K]: rows [0, F) are the gate projection, rows [F, 2F)
 * the up projection.  For every row r of expert e, with g and u the FP32 outputs
 * of the two projections (accumulator times the FP32 tensor scales, as
 * mxc_moe_linear returns them):
 *   h = SiLU(g) * u = (g / (1 + exp(-g))) * u,
 * evaluated one IEEE FP32 operation at a time, with exp(x) computed as
 * 2^n * P(r), x = n ln2 + r (Cody-Waite reduction, ln2 split into a 9-bit head
 * and the rest), P the degree-7 Taylor polynomial of e^r by Horner's rule, no
 * fused multiply-add; exp(x) = +inf above 88 and 0 below -86.  h is then
 * quantized exactly as mxc_quantize_act quantizes BF16 input (blocks of B
 * consecutive channels of h), in the activation's format:
 *   E8M0-B32: no tensor scale;
 *   E4M3-B16: with the given FP32 tensor scale *h_tscale_in (a calibrated scale:
 *             h's global maximum is unknown while its tiles are produced).
 * h is never written in a wider type.
 * a, d_offsets, experts, E, ws, ws_bytes: as for mxc_moe_linear (N = 2F, F a
 *           multiple of 128)
 * h_tscale_in device FP32, required for E4M3-B16, ignored for E8M0-B32
 * h_q       device, FP4 matrix [M, ldh] (ldh >= F/2, a multiple of 16)
 * h_sf      device, grouped SF layout of h's [rows, F/B] scales (the layout of
 *           mxc_quantize_act_grouped over the same offsets: each expert's rows
 *           start at the next multiple of 128 rows; mxc_grouped_sf_rows_bound(M, E)
 *           rows are enough); the padding rows of every expert tile get zero
 *           scales.  (h_q, h_sf, h_tscale_in) is the activation of the down
 *           projection's mxc_moe_linear over the same d_offsets. */
mxc_status mxc_moe_gate_up_swiglu(const mxc_mx_tensor* a, const int32_t* d_offsets, const mxc_weight* experts,
                                  int32_t E, const float* h_tscale_in, uint8_t* h_q, int64_t ldh, uint8_t* h_sf,
                                  void* ws, size_t ws_bytes, mxc_stream_t stream);

/* mxc_moe_linear for callers that cannot allocate device memory: plugins whose
 * host owns all device memory and hands out none, real-time serving loops that
 * forbid allocator calls (an allocation may block or synchronize the device
 * mid-step), or C callers with no device allocator at hand.
 * The paper has no counterpart to this entry point; it exists for the calling
 * environment only.  It takes the same arguments as mxc_moe_linear minus the
 * workspace, checks them in the same order with the same statuses, and runs
 * the same kernels, so its output is bit-identical to mxc_moe_linear's.
 * Scratch: the per-call expert tile and chunk tables live in a fixed
 * module-global array of 2304 bytes in device memory (room for the largest
 * tables, E = 256 experts),
 * held by every GPU that loads the library until the process exits.  Limit:
 * E <= 256 experts, as for mxc_moe_linear; larger E returns MXC_ERR_UNSUPPORTED
 * and enqueues nothing.
 * The first call on each device looks up that array's device address (no
 * allocation); make the first call on a device before any stream capture that
 * includes this entry point.  Every call rewrites the tables before reading them,
 * so nothing needs clearing between calls, but all calls on a device share the
 * array: calls whose executions overlap on the GPU (e.g. on two streams without
 * ordering between them) race.  The function calls no cudaMalloc, cudaFree or
 * other allocating routine. */
mxc_status mxc_moe_linear_noalloc(const mxc_mx_tensor* a, const int32_t* d_offsets, const mxc_weight* experts,
                                  int32_t E, void* y, int64_t ldy, mxc_dtype y_dtype, mxc_stream_t stream);

/* Runs the weight decode of mxc_linear (index -> codebook -> FP4 tile and
 * scale decode, through shared memory) and writes the result out in plain
 * layouts: q_out FP4 matrix [N, ldq], sf_out the SF layout of [N, K/B].
 * Used to check the decode bit for bit and to build native-FP4 weights that
 * hold exactly the same values. */
mxc_status mxc_decode_weight(const mxc_weight* w, uint8_t* q_out, int64_t ldq, uint8_t* sf_out,
                             mxc_stream_t stream);

/* Self-test of the device timeout path (test infrastructure; the paper has no
 * counterpart).  Enqueues one tiny kernel whose single bounded pipeline wait --
 * the same wait every kernel of this library uses -- is on a barrier that nothing
 * completes, with a limit of limit_cycles SM clocks (1 .. 2e9) instead of the
 * pipelines' two billion.  The wait runs out, the kernel records MXC_ERR_TIMEOUT
 * in the device error word and returns normally: no fault, no hang, nothing left
 * in flight, the context stays usable.  mxc_get_device_error() then returns
 * MXC_ERR_TIMEOUT.  Returns MXC_ERR_INVALID_ARG for a limit out of range. */
mxc_status mxc_selftest_wait_timeout(int64_t limit_cycles, mxc_stream_t stream);

/* Waits for the stream, then reads and clears the device error word of the
 * current device: MXC_OK, MXC_ERR_DEVICE_INVALID or MXC_ERR_TIMEOUT. */
mxc_status mxc_get_device_error(mxc_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MXC_H_ */
