/*
 * qlora.h -- C ABI of the NF4 + double-quantized QLoRA linear layer on B200.
 *
 * The layer (cited by web-page title and section):
 *
 *     Y = X . dequant(W)^T + s . (X . A^T) . B^T ,     s = alpha / r
 *
 *   - the frozen base weight W is stored in 4 bits and dequantized block by
 *     block to bf16 for each matrix product ["QLoRA", Storage precision is not
 *     calculation precision; "QLoRA and Quantized Training", The idea;
 *     "A 65B fine-tune on the GPU you already have", figure 2];
 *   - the 16 code levels sit at normal quantiles (NF4) ["QLoRA and Quantized
 *     Training", The idea; "QLoRA Explained", 1. 4-bit NormalFloat];
 *   - one absmax constant per block of 64 weights, and those constants are
 *     themselves quantized to 8 bits in blocks of 256 with one fp32 constant
 *     each ["A 65B fine-tune on the GPU you already have", figure 4;
 *     "QLoRA > Summary"];
 *   - only the low-rank adapters A, B (bf16) receive gradients; the input
 *     gradient flows through the frozen dequantized weight ["QLoRA", Follow
 *     one QLoRA training step; "QLoRA Explained", What is QLoRA?].
 *
 * Entry points: qlora_quantize_nf4_dq / qlora_quantize_4bit_dq (fp32 W ->
 * codes), qlora_dequant (codes -> bf16 W^), qlora_linear_fwd (and its
 * _noalloc form), qlora_linear_bwd_dx, qlora_lora_bwd (adapter gradients),
 * qlora_linear_bwd (the whole backward, rank-r intermediates formed once),
 * qlora_merge_adapter (W^ + s B A for export), qlora_lora_dropout and the
 * _dropout forms of the forward and input gradient; helpers for workspace sizes,
 * codebook levels, errors, versions and launch counts.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers, allocated and owned by the
 *     caller.  The library never allocates, frees or retains memory; scratch
 *     space is a caller-provided workspace sized by qlora_workspace_bytes().
 *   - Matrices are dense row-major.  bf16 tensors are passed as uint16_t bit
 *     patterns (the layout of __nv_bfloat16).  W is [n x k] (out x in),
 *     X [m x k], Y [m x n], A [r x k], B [n x r].
 *   - Every tensor pointer must be 16-byte aligned.
 *   - Shapes: n > 0, k > 0, k % 64 == 0; the linear operations also need
 *     n % 8 == 0 (16-byte bf16 rows of Y and dY);
 *     r % 16 == 0 with 0 <= r <= 256 (r == 0, or A == B == NULL, means no
 *     adapter), m >= 0 (m == 0 is an empty batch: nothing is launched).
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream);
 *     inputs must stay valid and outputs untouched until the stream reaches
 *     the call.  All arguments are validated on the host before any launch:
 *     a call that returns an error has launched nothing.  No kernel traps.
 *   - Return value: QLORA_OK or one of the negative codes below.  After
 *     QLORA_ERR_CUDA, qlora_last_cuda_error() returns the cudaError_t.
 *   - Inputs must be finite (NaN/Inf weights are a documented precondition,
 *     not checked on the device).
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; a cudaStream_t can be passed directly. */
typedef struct CUstream_st *qlora_stream_t;

enum qlora_status {
  QLORA_OK = 0,
  QLORA_ERR_NULL = -1,      /* a required pointer is NULL                  */
  QLORA_ERR_SHAPE = -2,     /* a size breaks the shape rules above         */
  QLORA_ERR_ALIGN = -3,     /* a pointer is not 16-byte aligned            */
  QLORA_ERR_WORKSPACE = -4, /* workspace missing or smaller than required  */
  QLORA_ERR_CUDA = -5,      /* a CUDA call failed (see last_cuda_error)    */
  QLORA_ERR_DEVICE = -6,    /* the current device is not sm_100            */
  QLORA_ERR_CODEBOOK = -7,  /* codebook id not one of qlora_codebook       */
  QLORA_ERR_FORMAT = -8     /* dq_format not one of qlora_dq_format         */
};

/* The sixteen 4-bit values a weight's codes index.  NF4 is the method's own
 * ("QLoRA and Quantized Training", The idea; "A 65B fine-tune on the GPU you
 * already have", figure 3).  FP4 and INT4 are the uniform-bin baselines the
 * pages say NF4 beats on normally distributed weights ("QLoRA Explained", The
 * three ideas behind QLoRA; "A 65B fine-tune", figure 3); the pages do not
 * define them, and these are the formats taken:
 *   QLORA_CODEBOOK_FP4   e2m1 float (1 sign, 2 exponent bits with bias 1,
 *                        1 mantissa bit): magnitudes 0 .. 6 divided by 6,
 *                        ascending; code 7 is -0, code 8 is +0.
 *   QLORA_CODEBOOK_INT4  symmetric integers i/7, i = -7..7, at codes 0..14;
 *                        code 15 repeats +1 and is never produced.
 * Every codebook is used with the same blocks, double quantization and
 * decision rule; only the levels and their midpoints change.               */
enum qlora_codebook { QLORA_CODEBOOK_NF4 = 0, QLORA_CODEBOOK_FP4 = 1, QLORA_CODEBOOK_INT4 = 2 };

/* How the block absmax constants are stored (double quantization).
 *   QLORA_DQ_LINEAR8   unsigned linear 8-bit codes, group_scale[g] = max of
 *                      the group's absmax (the pages' format, 0.127 bit/weight):
 *                      c' = fp32(q * fp32(group_scale[g] / 255))
 *   QLORA_DQ_FP8_MEAN  the cited paper's variant, which the pages name but
 *                      do not define ("QLoRA Explained", What is QLoRA?;
 *                      arXiv:2305.14314): the tensor's mean absmax mu is
 *                      subtracted first and the offsets are stored as E4M3
 *                      8-bit floats per group of 256.  mu = fp32 of the fp64
 *                      sum of the absmax values (each group summed by
 *                      pairwise halving, then the group sums the same way)
 *                      over nb; S_g = max |c - mu| over the group;
 *                      absmax_q = E4M3_rn(fp32(fp32((c - mu) / S_g) * 448));
 *                      group_scale[g] = fp32(S_g / 448) for g < ng and
 *                      group_scale[ng] = mu (ng + 1 floats):
 *                      c' = fp32(fp32(E4M3(absmax_q) * group_scale[g]) + mu)  */
enum qlora_dq_format { QLORA_DQ_LINEAR8 = 0, QLORA_DQ_FP8_MEAN = 1 };

/* Quantized weight: three flat buffers plus the shape and the codebook.
 *   codes       uint8 [n*k/2]   4-bit codes, two per byte in row-major element
 *                               order: byte j = (code[2j] << 4) | code[2j+1]
 *   absmax_q    uint8 [n*k/64]  8-bit code of each block's absmax
 *   group_scale fp32  [ceil(n*k/64/256)]  max absmax of each group of 256
 *   block == 64 and group == 256 are the only supported values.
 *   codebook    qlora_codebook the codes index (0 == NF4, so a zeroed field
 *               means NF4); any other value gives QLORA_ERR_CODEBOOK.
 *   dq_format   qlora_dq_format of absmax_q / group_scale (0 == linear 8-bit,
 *               so a zeroed field means the pages' format; QLORA_DQ_FP8_MEAN
 *               has ng + 1 group_scale entries); any other value gives
 *               QLORA_ERR_FORMAT.
 * Dequantization ["A 65B fine-tune on the GPU you already have", figure 4;
 * "QLoRA", Storage precision is not calculation precision]:
 *   c'  = fp32(float(absmax_q[b]) * fp32(group_scale[b/256] / 255))
 *         (QLORA_DQ_LINEAR8; the c' of QLORA_DQ_FP8_MEAN is given above)
 *   W^  = bf16_rne(fp32(L[code] * c')), L the weight's codebook            */
typedef struct {
  const uint8_t *codes;
  const uint8_t *absmax_q;
  const float *group_scale;
  int64_t n, k;
  int32_t block;
  int32_t group;
  int32_t codebook;
  int32_t dq_format;
} qlora_nf4_weight;

/* Operation ids for qlora_workspace_bytes. */
enum qlora_op { QLORA_OP_FWD = 0, QLORA_OP_BWD_DX = 1, QLORA_OP_LORA_BWD = 2 };

/* Blockwise NF4 quantization with double-quantized absmax.
 * ["QLoRA and Quantized Training", The idea and Worked example (blocks of 64,
 *  one fp32 scale each, 0.5 byte per weight); "A 65B fine-tune on the GPU you
 *  already have", figures 3 and 4 (NF4 levels; 8-bit constants in blocks of
 *  256); "QLoRA > Summary" (scales quantized to 8-bit integers)]
 *   W              in   fp32 [n x k]
 *   codes          out  uint8 [n*k/2]
 *   absmax_q       out  uint8 [n*k/64]
 *   group_scale    out  fp32  [ceil(n*k/64/256)]
 *   absmax_fp32    out  fp32  [n*k/64] block absmax before double
 *                       quantization; may be NULL
 * Per block b of 64 consecutive row-major weights: c_b = max|w|;
 * code = #{i : fp32(w / c_b) > T_i} over the 15 fp32 midpoints T_i of the
 * sorted NF4 levels (a value on a midpoint takes the lower code; c_b == 0
 * gives code 7, the zero level).  Per group g of 256 blocks: S_g = max c_b,
 * absmax_q = rint_even(fp32(fp32(c_b / S_g) * 255)) (0 when S_g == 0).     */
int qlora_quantize_nf4_dq(const float *W, int64_t n, int64_t k,
                          uint8_t *codes, uint8_t *absmax_q, float *group_scale,
                          float *absmax_fp32, qlora_stream_t stream);

/* The same quantization with the levels and midpoints of `codebook`
 * (qlora_codebook); qlora_quantize_nf4_dq is codebook QLORA_CODEBOOK_NF4.
 * The weight it fills is used with that codebook in qlora_nf4_weight.     */
int qlora_quantize_4bit_dq(const float *W, int64_t n, int64_t k, int32_t codebook,
                           uint8_t *codes, uint8_t *absmax_q, float *group_scale,
                           float *absmax_fp32, qlora_stream_t stream);

/* The same quantization with the absmax constants stored in `dq_format`
 * (qlora_dq_format); qlora_quantize_4bit_dq is QLORA_DQ_LINEAR8.  With
 * QLORA_DQ_FP8_MEAN, group_scale has ng + 1 entries and the call reads W
 * twice (the mean of all block absmax values is needed before any group's
 * codes); absmax_q doubles as scratch between the passes.                  */
int qlora_quantize_4bit_dq_format(const float *W, int64_t n, int64_t k, int32_t codebook, int32_t dq_format,
                                  uint8_t *codes, uint8_t *absmax_q, float *group_scale,
                                  float *absmax_fp32, qlora_stream_t stream);

/* Standalone dequantization to bf16 ["QLoRA", Storage precision is not
 * calculation precision; "A 65B fine-tune on the GPU you already have",
 * figure 2].
 *   w       in   quantized weight [n x k]
 *   W_bf16  out  bf16 [n x k], bit-exact W^ as defined at qlora_nf4_weight. */
int qlora_dequant(const qlora_nf4_weight *w, uint16_t *W_bf16, qlora_stream_t stream);

/* Adapter merge (export): W' = W^ + s . B . A
 * ["QLoRA", Training setup versus deployment setup (serve the quantized base
 *  with the adapter, or merge into another checkpoint); Common misconception
 *  (LoRA's matrices merge back into the frozen weight)]
 *   w       in   quantized weight [n x k] (any codebook)
 *   A, B    in   bf16 [r x k], [n x r]; NULL/NULL or r == 0: W' = W^ bit for
 *                bit (FP4's -0 level included)
 *   scale   in   s = alpha / r
 *   W_bf16  out  bf16 [n x k] = bf16_rne(W'), or NULL
 *   W_f32   out  fp32 [n x k] = W', or NULL (e.g. to re-quantize it with
 *                qlora_quantize_4bit_dq into a new 4-bit checkpoint)
 * At least one output.  W' = fma(s, acc, W^) in fp32, acc the fp32 sum of the
 * rank-r product; W^ exactly as qlora_dequant returns it.                   */
int qlora_merge_adapter(const qlora_nf4_weight *w, const uint16_t *A, const uint16_t *B, int32_t r,
                        float scale, uint16_t *W_bf16, float *W_f32, qlora_stream_t stream);

/* Forward: Y = bf16( X . W^T + T . B^T ),  T = bf16(s . X . A^T)
 * ["QLoRA and Quantized Training", The idea (compute in bf16, each block
 *  dequantized, used, discarded); "A 65B fine-tune on the GPU you already
 *  have", figure 2; LoRA r and alpha from "QLoRA and Quantized Training",
 *  In code]
 *   X      in   bf16 [m x k]
 *   w      in   quantized weight [n x k]
 *   A, B   in   bf16 [r x k], [n x r]; NULL/NULL or r == 0: no adapter
 *   scale  in   s = alpha / r
 *   Y      out  bf16 [m x n]
 *   ws     scratch, ws_bytes >= qlora_workspace_bytes(QLORA_OP_FWD, m, n, k, r);
 *          contents on entry are ignored; when the call returns (in stream
 *          order) its first m*r*2 bytes hold T [m x r], which
 *          qlora_linear_bwd can take instead of recomputing it.
 * Products accumulate in fp32.  m <= 16 runs a weight-streaming kernel; larger
 * m runs the tcgen05 tensor-core kernel with dequantization in its main loop. */
int qlora_linear_fwd(const uint16_t *X, int64_t m, const qlora_nf4_weight *w,
                     const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                     uint16_t *Y, void *ws, size_t ws_bytes, qlora_stream_t stream);

/* Input gradient: dX = bf16( dY . W^ + U . A ),  U = bf16(s . dY . B)
 * ["QLoRA", Follow one QLoRA training step, step 4 (gradients flow into the
 *  adapters, not the frozen base); "QLoRA Explained", What is QLoRA?
 *  (backpropagates through a frozen, 4-bit quantized base model)]
 *   dY     in   bf16 [m x n]
 *   w      in   quantized weight [n x k]
 *   A, B   in   bf16 [r x k], [n x r] (as in the forward)
 *   dX     out  bf16 [m x k]
 *   ws     scratch, ws_bytes >= qlora_workspace_bytes(QLORA_OP_BWD_DX, m, n, k, r) */
int qlora_linear_bwd_dx(const uint16_t *dY, int64_t m, const qlora_nf4_weight *w,
                        const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                        uint16_t *dX, void *ws, size_t ws_bytes, qlora_stream_t stream);

/* Adapter gradients ["QLoRA and Quantized Training", The idea (the adapters
 * hold the gradients and optimizer state); "QLoRA", Follow one QLoRA training
 * step, step 4]:
 *   dA = bf16( s . (dY . B)^T . X )      [r x k]
 *   dB = bf16( dY^T . T ),  T = bf16(s . X . A^T)     [n x r]
 *   X, dY  in   bf16 [m x k], [m x n]
 *   A, B   in   bf16 [r x k], [n x r], r > 0
 *   dA, dB out  bf16; overwritten (not accumulated)
 *   ws     scratch, ws_bytes >= qlora_workspace_bytes(QLORA_OP_LORA_BWD, m, n, k, r)
 * m == 0 writes zeros to dA and dB.  For r <= 64, U = bf16(s . dY . B) and
 * dB come from one read of dY (one kernel forms both products, then a small
 * kernel adds the fp32 partials of U in a fixed order); results do not
 * depend on the launch configuration's timing (no atomics).                */
int qlora_lora_bwd(const uint16_t *X, const uint16_t *dY, int64_t m, int64_t n, int64_t k,
                   const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                   uint16_t *dA, uint16_t *dB, void *ws, size_t ws_bytes,
                   qlora_stream_t stream);

/* The whole backward of the layer in one call: dX, dA and dB, with the
 * rank-r intermediates formed once ["QLoRA", Follow one QLoRA training step,
 * step 4; "QLoRA and Quantized Training", The idea]:
 *   U  = bf16(s . dY . B)   computed once, used by dX and by dA
 *   dX = bf16(dY . W^ + U . A)          (skipped when dX is NULL)
 *   dA = bf16(U^T . X),  dB = bf16(dY^T . T)
 *   T  = bf16(s . X . A^T): pass the forward's (qlora_linear_fwd leaves it at
 *        the start of its workspace, [m x r] row-major), or NULL to compute it
 *        here.  With dropout, X is the forward's Xd and T its workspace.
 *   dY, X  in   bf16 [m x n], [m x k];  A, B as in the forward, r > 0
 *   dX, dA, dB out  (dX may be NULL); ws >= qlora_workspace_bytes(QLORA_OP_LORA_BWD, m, n, k, r)
 * m == 0 writes zeros to dA and dB.  Same results as qlora_linear_bwd_dx
 * followed by qlora_lora_bwd, with two fewer rank-r projections; for r <= 64
 * U and dB share one read of dY, as in qlora_lora_bwd.                     */
int qlora_linear_bwd(const uint16_t *dY, const uint16_t *X, const uint16_t *T, int64_t m,
                     const qlora_nf4_weight *w, const uint16_t *A, const uint16_t *B, int32_t r,
                     float scale, uint16_t *dX, uint16_t *dA, uint16_t *dB, void *ws, size_t ws_bytes,
                     qlora_stream_t stream);

/* LoRA dropout on the adapter input ["QLoRA and Quantized Training", In code:
 * LoraConfig(r=16, lora_alpha=32, lora_dropout=0.05, ...)].  The pages give
 * only the probability; the reading taken is inverted dropout on the
 * adapter's input, as in the LoRA configuration they use:
 *     Xd = D . X . c,   c = fp32(1 / fp32(1 - p)),   kept: bf16_rne(fp32(x . c)), dropped: +0
 *     Y  = X . W^T + s . (Xd . A^T) . B^T              (the frozen product keeps X)
 *     dX = dY . W^ + D . (s . (dY . B) . A) . c
 *     dA = s . (dY . B)^T . Xd,   dB = s . dY^T . (Xd . A^T)   (qlora_lora_bwd with Xd for X)
 * The keep mask D is counter-based, so the backward regenerates it from the
 * forward's (seed, offset): element e of the row-major [m x k] tensor draws
 * 16-bit lane e % 16 (bits 16 (i % 4) of word i / 4 for lane i) of
 * Philox4x64-10 (Salmon et al., SC 2011) for counter (e / 16, offset, 0, 0)
 * under key (seed, 0), and is kept when that value is >= round_half_even(
 * fp32(p) . 65536).  `offset` separates the masks of different calls (steps,
 * layers).  0 <= p < 1, else QLORA_ERR_SHAPE; k % 64 == 0.
 *
 * qlora_lora_dropout:       Xd [m x k] bf16 from X [m x k] bf16.
 * qlora_linear_fwd_dropout: writes Xd (keep it for the backward) and Y; an
 *   adapter is required (A, B non-NULL, r > 0); ws as for qlora_linear_fwd.
 * qlora_linear_bwd_dx_dropout: dX as above, computed as
 *   bf16(bf16(dY . W^) + D . (U . A) . c) with U = bf16(s . dY . B); an
 *   adapter is required; ws as for qlora_linear_bwd_dx.                     */
int qlora_lora_dropout(const uint16_t *X, int64_t m, int64_t k, float p, uint64_t seed, uint64_t offset,
                       uint16_t *Xd, qlora_stream_t stream);
int qlora_linear_fwd_dropout(const uint16_t *X, int64_t m, const qlora_nf4_weight *w,
                             const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                             float p, uint64_t seed, uint64_t offset, uint16_t *Xd, uint16_t *Y,
                             void *ws, size_t ws_bytes, qlora_stream_t stream);
int qlora_linear_bwd_dx_dropout(const uint16_t *dY, int64_t m, const qlora_nf4_weight *w,
                                const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                                float p, uint64_t seed, uint64_t offset, uint16_t *dX,
                                void *ws, size_t ws_bytes, qlora_stream_t stream);

/* Forward with no caller workspace, for callers that cannot allocate device
 * memory: code whose host owns every device allocation (an engine plugin), a
 * deployment that forbids allocation on its serving path, or a C caller with
 * no device allocator.  The pages have no counterpart: this is a convenience
 * of this library around qlora_linear_fwd.
 *   Same arguments, checks (in the same order), results and errors as
 *   qlora_linear_fwd, minus `ws`.
 *   The rank-r scratch T lives in a fixed device array of
 *   QLORA_NOALLOC_SCRATCH_BYTES inside the library; every device that loads
 *   the library holds it until the process exits.  Calls whose scratch
 *   (m*r*2 bytes rounded up to 256) exceeds it return QLORA_ERR_WORKSPACE and
 *   launch nothing.  The call allocates nothing: no cudaMalloc, no cudaFree,
 *   no allocating library routine.
 *   The first call with an adapter on a device looks up the array's device
 *   address (cudaGetSymbolAddress) with that device current, and looks it up
 *   again whenever another driver context is current on that device; make
 *   that first call before any stream capture.  Calls after cudaDeviceReset
 *   in the same process are not supported.
 *   All calls on a device share the array and it keeps the last call's
 *   contents; T is fully written before it is read, so nothing in it needs to
 *   start at zero.  Calls that may run at the same time on one device (other
 *   streams, other host threads) race on the array: serialize them.        */
#define QLORA_NOALLOC_SCRATCH_BYTES (1u << 20)
int qlora_linear_fwd_noalloc(const uint16_t *X, int64_t m, const qlora_nf4_weight *w,
                             const uint16_t *A, const uint16_t *B, int32_t r, float scale,
                             uint16_t *Y, qlora_stream_t stream);

/* Workspace bytes an operation needs (0 if none); SIZE_MAX for an unknown op
 * or invalid sizes.  A workspace may be reused across calls on one stream;
 * two calls that may run concurrently need separate workspaces.
 * QLORA_OP_LORA_BWD (also qlora_linear_bwd): U and T ([m x r] bf16 each,
 * 256-byte aligned), then for r <= 64 the fp32 partials of U, one [m x r]
 * block per n-range of the one-pass kernel (at most one range per 128
 * columns of n; the bound holds for any device).                           */
size_t qlora_workspace_bytes(int op, int64_t m, int64_t n, int64_t k, int32_t r);

/* cudaError_t of the last failing CUDA call on this host thread (0 if none). */
int qlora_last_cuda_error(void);

/* Device-side status: kernels never trap; a wait inside a kernel that gives
 * up after its time limit sets a bit in a per-device error word instead and
 * the kernel exits early (its outputs are then undefined).  This call
 * synchronizes `stream`, writes the word to *flags (host memory; 0 = no
 * error) and clears it.  QLORA_ERR_NULL if flags is NULL.  Bits: which wait
 * gave up (a pipeline stage's operands, the expanded weight tile, a free
 * stage, the accumulator, the final drain of copies, the self-test).        */
enum qlora_device_error {
  QLORA_DEVERR_OPERANDS = 1u << 0,
  QLORA_DEVERR_WEIGHT_TILE = 1u << 1,
  QLORA_DEVERR_FREE_STAGE = 1u << 2,
  QLORA_DEVERR_ACCUMULATOR = 1u << 3,
  QLORA_DEVERR_DRAIN = 1u << 4,
  QLORA_DEVERR_SELFTEST = 1u << 5
};
int qlora_poll_device_error(qlora_stream_t stream, unsigned *flags);

/* Self-tests of the device-side guards (no counterpart on the pages).
 * qlora_selftest_bounded_wait launches one thread that waits, through the
 * same bounded mbarrier wait the pipelined kernels use, on a barrier nothing
 * arrives at: after limit_ns nanoseconds (1 .. 2e9) the wait gives up, sets
 * QLORA_DEVERR_SELFTEST in the device error word and the kernel returns,
 * writing 1 to *expired (device memory, 4-byte aligned; may be NULL).  Nothing
 * faults and the context stays usable.
 * qlora_selftest_div255 adds to *mismatches (device memory, 8-byte aligned)
 * the number of fp32 bit patterns in [first_bits, first_bits + count) (all
 * positive and finite) whose fp32(s / 255) by the library's division
 * (Markstein's method with the correctly rounded reciprocal of 255, used for
 * the double-quantization constant) differs from IEEE division.             */
int qlora_selftest_bounded_wait(uint64_t limit_ns, unsigned *expired, qlora_stream_t stream);
int qlora_selftest_div255(uint32_t first_bits, uint32_t count, unsigned long long *mismatches,
                          qlora_stream_t stream);

/* Profiling hook.  While set, qlora_linear_fwd and qlora_linear_bwd_dx
 * record `start` on their stream right before launching their main kernel
 * (the fused tensor-core GEMM, or the weight-streaming kernel for small m)
 * and `stop` right after it, so the caller can time that kernel alone with
 * cudaEventElapsedTime.  Both are cudaEvent_t handles owned by the caller;
 * the setting is per host thread; pass NULL, NULL to clear.  Returns
 * QLORA_ERR_NULL if exactly one of the two is NULL.                         */
int qlora_set_profile_events(void *start, void *stop);

/* Number of CUDA kernels this library has launched in this process so far
 * (all threads, all devices).  Lets a caller count the launches inside a
 * timed region.                                                             */
uint64_t qlora_launch_count(void);

/* Static, human-readable name of a status code. */
const char *qlora_status_string(int status);

/* The library's own fp32 NF4 codebook, derived at load time from the normal
 * quantile construction (16 ascending levels, index 7 == 0, 0 == -1,
 * 15 == +1).  Host function; writes 16 floats to `levels` (host memory).   */
void qlora_nf4_levels(float *levels);

/* The 16 fp32 levels of `codebook` in code order (host function, host
 * memory); QLORA_ERR_CODEBOOK for an unknown id, QLORA_ERR_NULL for NULL. */
int qlora_codebook_levels(int32_t codebook, float *levels);

/* ABI version: (major << 16) | minor. */
int qlora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
