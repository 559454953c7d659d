/*
 * ifq.h -- C ABI of libifq: PhaseQuant quantization of complex weights to the
 * fourth roots of unity {1, i, -1, -i} and the multiplication-free complex
 * product that consumes the codes, on one NVIDIA B200 (sm_100a).
 *
 * Method sources, by page and section:
 *   "Fairy2i write-up" (hotelren.com): §2.1 widely-linear transform y = Ux + W conj(x),
 *     §3.1 phase rule, §3.2 axis-aligned scales, §4.1 recursive residual stages,
 *     §4.2 multiplication-free product.
 *   "iFairy article" (bestcxt.com): §二.1 codebook and 2-bit storage, §二.2 GEMM by add/sub/swap.
 *   "iFairy talk notes" (43b.com.cn): §2.2.2 phase rule, §2.3.1 x i = swap + negate.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers into caller-owned memory.  The
 *     library allocates nothing, keeps no state between calls, never
 *     synchronizes the host, and enqueues all work on the caller's stream.
 *     Descriptor arrays (ifq_qtensor*, ifq_layer*) are HOST pointers; they
 *     are read during the call and may be freed when it returns.
 *   - Every argument error is reported by the return value before anything
 *     is enqueued.  Conditions that only the GPU can see set bits in the
 *     caller's device status word (dev_status), which the caller reads after
 *     synchronizing; no kernel traps or asserts.
 *   - Complex tensors are planar: a real plane and an imaginary plane.
 *   - Code k in {0,1,2,3} stands for the codebook entry [1, i, -1, -i][k]
 *     (the list order of the §3.1 phase-rule sketch).  Bit 0 of k is the axis
 *     (0: real, +-1; 1: imaginary, +-i), bit 1 the sign.
 *   - Packed codes: uint8 [T][N][K/4], row-major; code j of row n of stage t
 *     is bits 2(j%4) and 2(j%4)+1 of byte [t][n][j/4].  2 bits per complex
 *     weight per stage.
 *   - Scales: float32 [T][2] = {s_re, s_im} per stage, per tensor (§3.2).
 *     Stage t's dequantized weight is w_hat_t = s_re Re(b) + i s_im Im(b).
 *   - Activations: bf16 bit patterns, planar, token-major [B or M][K].
 *     Outputs: float32, planar, token-major [B or M][N], OVERWRITTEN.
 */
#ifndef IFQ_H
#define IFQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t passed as an opaque pointer (NULL = the legacy default stream). */
typedef void* ifq_stream_t;

typedef enum {
  IFQ_OK = 0,
  IFQ_ERR_NULL = 1,        /* a required pointer is NULL */
  IFQ_ERR_SHAPE = 2,       /* a size is zero, negative, odd where it must be even, or not a multiple the call needs */
  IFQ_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  IFQ_ERR_STAGES = 4,      /* T outside 1..IFQ_MAX_STAGES */
  IFQ_ERR_BATCH = 5,       /* B outside 1..IFQ_MAX_GEMV_BATCH, or M < 1 */
  IFQ_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than ifq_quantize_workspace_bytes() */
  IFQ_ERR_CUDA = 7,        /* a CUDA runtime call failed (launch error, no device, ...) */
  IFQ_ERR_UNSUPPORTED = 8, /* the device is not sm_100 */
  IFQ_ERR_COUNT = 9,       /* descriptor count outside 1..IFQ_MAX_GROUP */
  IFQ_ERR_STATIC_LIMIT = 10 /* the call needs more scratch than IFQ_QUANT_STATIC_SCRATCH_BYTES */
} ifq_status;

#define IFQ_MAX_STAGES 8
#define IFQ_MAX_GEMV_BATCH 16
#define IFQ_MAX_GROUP 32

/* Device status bits, OR-ed into *dev_status by kernels. */
#define IFQ_DEV_NONFINITE 0x1u /* a weight was NaN or Inf; it was quantized as 0 (code 0) */
#define IFQ_DEV_TIMEOUT 0x2u   /* a bounded pipeline wait gave up; outputs of that call are invalid */

const char* ifq_status_string(ifq_status s);

/* ---------------------------------------------------------------------------
 * ifq_widely_linear_from_real  ("Fairy2i write-up" §2.1)
 *
 * Splits a real layer R (rows = 2n outputs, cols = 2m inputs, float32
 * row-major) into complex n x m matrices U and W with R [x_re; x_im] =
 * U x + W conj(x):
 *   U_re = (R11 + R22)/2, U_im = (R21 - R12)/2,
 *   W_re = (R11 - R22)/2, W_im = (R12 + R21)/2,
 * with R11 = R[:n,:m], R12 = R[:n,m:], R21 = R[n:,:m], R22 = R[n:,m:].
 * Each output is the float32 sum or difference rounded to nearest-even, then
 * halved, which equals the exact value rounded once.
 *
 *   R                     [rows][cols] float32, device, read-only
 *   rows, cols            even, >= 2
 *   U_re, U_im, W_re, W_im  [rows/2][cols/2] float32, device, written
 * Pointers must be 16-byte aligned.  The four outputs must not overlap R.
 * ------------------------------------------------------------------------- */
ifq_status ifq_widely_linear_from_real(const float* R, int64_t rows, int64_t cols,
                                       float* U_re, float* U_im, float* W_re, float* W_im,
                                       ifq_stream_t stream);

/* ---------------------------------------------------------------------------
 * ifq_quantize_pack  ("Fairy2i write-up" §3.1, §3.2, §4.1)
 *
 * T-stage PhaseQuant of `count` complex tensors.  Stage t quantizes the
 * residual r_t = w - sum_{u<t} w_hat_u (r_1 = w), computed in float64 from w
 * and the codes and float32 scales of the earlier stages:
 *   k = sector of r_t: floor(2 arg(r)/pi + 0.5) mod 4, evaluated exactly by
 *       comparisons (a tie on a diagonal goes counter-clockwise; r = 0 -> 0);
 *   s_re = mean |Re r| over entries coded +-1, s_im = mean |Im r| over
 *       entries coded +-i (float64 sums, rounded to float32; 0 if none).
 * An entry with a NaN or Inf part is quantized as 0 and sets IFQ_DEV_NONFINITE.
 * Sums are reduced in a fixed order, so results are bit-reproducible.
 *
 *   tensors[i].w_re, w_im   [N][K] float32, device, read-only, 16-byte aligned
 *   tensors[i].N, K         N >= 1, K >= 4, K % 4 == 0
 *   tensors[i].codes        [T][N][K/4] uint8, device, written, 16-byte aligned
 *   tensors[i].scales       [T][2] float32, device, written
 *   count                   1..IFQ_MAX_GROUP tensors, processed together
 *   T                       1..IFQ_MAX_STAGES
 *   workspace               device scratch of ifq_quantize_workspace_bytes()
 *                           bytes, 16-byte aligned, owned by the caller; no
 *                           initial contents needed; must not be used by
 *                           anything else until the enqueued work finishes
 *   dev_status              device uint32, bits OR-ed in (may be NULL)
 * ------------------------------------------------------------------------- */
typedef struct {
  const float* w_re;
  const float* w_im;
  int64_t N;
  int64_t K;
  uint8_t* codes;
  float* scales;
} ifq_qtensor;

size_t ifq_quantize_workspace_bytes(const ifq_qtensor* tensors, int count, int T);

ifq_status ifq_quantize_pack(const ifq_qtensor* tensors, int count, int T, void* workspace,
                             size_t workspace_bytes, uint32_t* dev_status, ifq_stream_t stream);

/* ---------------------------------------------------------------------------
 * ifq_quantize_stage, ifq_quantize_finish  ("Fairy2i write-up" §3.2, §4.1; rows
 * of a tensor split across GPUs)
 *
 * ifq_quantize_pack in two halves per stage, for a tensor whose rows are split
 * across GPUs.  A stage's scales are means over the whole tensor (§3.2), so the
 * shards exchange the stage's tile partials before the next stage:
 *   1. every GPU: ifq_quantize_stage(shard, t) -- stage t's codes of its rows and
 *      one 32-byte partial (class sums and count) per 4096-weight tile of the
 *      shard, in `partials`;
 *   2. gather the partials of all shards in row order (e.g. an all-gather);
 *   3. every GPU: ifq_quantize_finish(gathered partials of the whole tensor, t)
 *      -- stage t's scales, by the same reduction over the same tiles in the
 *      same order as ifq_quantize_pack.
 * When every shard but the last holds a multiple of 4096 weights (rows * K),
 * the shards' tiles are exactly the whole tensor's tiles and codes and scales
 * equal those of ifq_quantize_pack on the whole tensor bit for bit.
 *
 *   tensors[i]      the shard: w_re, w_im [N_shard][K]; codes [T][N_shard][K/4]
 *                   (stage t written, stages < t read); scales [T][2] (stages
 *                   < t read: the whole tensor's scales, from earlier finish
 *                   calls).  Sizes and alignment as for ifq_quantize_pack.
 *   t               the stage, 1..IFQ_MAX_STAGES (stage 1 reads no codes)
 *   partials        device buffer of ifq_quantize_workspace_bytes(tensors,
 *                   count, t) bytes (the shard's tile partials, tensor after
 *                   tensor), 16-byte aligned; no initial contents needed
 *   parts[i]        .partials: the gathered partials of a whole tensor
 *                   (quantizer tiles of N x K weights, 32 bytes each, in row
 *                   order); .N: the whole tensor's rows; .K; .scales: [T][2],
 *                   stage t written (4-byte aligned)
 * Errors as for ifq_quantize_pack; t outside 1..IFQ_MAX_STAGES is
 * IFQ_ERR_STAGES.
 * ------------------------------------------------------------------------- */
typedef struct {
  const void* partials;
  int64_t N;
  int64_t K;
  float* scales;
} ifq_qpartials;

ifq_status ifq_quantize_stage(const ifq_qtensor* tensors, int count, int t, void* partials, size_t partials_bytes,
                              uint32_t* dev_status, ifq_stream_t stream);

ifq_status ifq_quantize_finish(const ifq_qpartials* parts, int count, int t, ifq_stream_t stream);

/* ---------------------------------------------------------------------------
 * ifq_quantize_pack_static
 *
 * The write-ups have no counterpart of this call: it is ifq_quantize_pack
 * (same kernels, same results bit for bit) with its scratch in a fixed array
 * inside the library instead of a caller workspace, for callers that cannot
 * hand over device memory -- a plain C weight loader with no device allocator
 * of its own, or a serving process that has reserved all free device memory
 * for its caches before it quantizes.  Nothing is allocated: no cudaMalloc,
 * no cudaFree, no allocating library call.
 *
 *   tensors, count, T, dev_status, stream   as for ifq_quantize_pack
 *
 * Limit: ifq_quantize_workspace_bytes(tensors, count, T) must not exceed
 * IFQ_QUANT_STATIC_SCRATCH_BYTES (2 MiB: 32 bytes per 4096 complex weights,
 * about 2.7e8 complex weights per call in total); larger calls return
 * IFQ_ERR_STATIC_LIMIT before anything is launched.
 * The scratch needs no initial contents: every call writes each part of it
 * before reading it.
 * The first call on a device (with that device current) looks up the array's
 * device address (cudaGetSymbolAddress) and may load the library's device code;
 * make that first call before anything that must not see such set-up, such as
 * a stream capture.  The address is kept per device together with the driver
 * context it belongs to, and looked up again when a call runs in another
 * context (a context of the caller's own, or the new primary context after a
 * device reset).
 * There is one array per device: calls whose work may overlap on the GPU
 * (unordered streams, or several host threads) race on it and give wrong
 * results.  Order such calls on one stream.
 * ------------------------------------------------------------------------- */
#define IFQ_QUANT_STATIC_SCRATCH_BYTES ((size_t)2 << 20)

ifq_status ifq_quantize_pack_static(const ifq_qtensor* tensors, int count, int T, uint32_t* dev_status,
                                    ifq_stream_t stream);

/* ---------------------------------------------------------------------------
 * ifq_widely_linear_quantize_pack  ("Fairy2i write-up" §2.1, then §3.1, §3.2, §4.1)
 *
 * ifq_widely_linear_from_real followed by ifq_quantize_pack of the resulting
 * U and W, with the conversion and stage 1 done in one pass over R: every
 * output -- the four planes, the codes and the scales of every stage -- is
 * bit for bit what the two calls give.  Per complex position at stage 1 this
 * moves 32.5 bytes of HBM traffic instead of 48.5 (R is read once; U and W are
 * written and not read back until stage 2).  Stages 2..T run as in
 * ifq_quantize_pack.
 *
 *   layers[i].R                  [rows][cols] float32, device, read-only
 *   layers[i].rows, cols         rows even >= 2; cols >= 8, cols % 8 == 0
 *                                (U, W are n x m = rows/2 x cols/2, m % 4 == 0)
 *   layers[i].U_re .. W_im       [n][m] float32, device, written (the
 *                                conversion's output and the quantizer's input)
 *   layers[i].codes_u, codes_w   [T][n][m/4] uint8, device, written
 *   layers[i].scales_u, scales_w [T][2] float32, device, written
 *   count                        1..IFQ_MAX_GROUP/2 layers (U and W count as
 *                                two tensors of one ifq_quantize_pack call)
 *   T                            1..IFQ_MAX_STAGES
 *   workspace                    device scratch of
 *                                ifq_widely_linear_quantize_workspace_bytes()
 *                                bytes, 16-byte aligned, owned by the caller;
 *                                no initial contents needed
 *   dev_status                   device uint32, bits OR-ed in (may be NULL)
 * Pointers must be 16-byte aligned (scales: 4-byte).  No output may overlap R
 * or another output.
 * ------------------------------------------------------------------------- */
typedef struct {
  const float* R;
  int64_t rows;
  int64_t cols;
  float* U_re;
  float* U_im;
  float* W_re;
  float* W_im;
  uint8_t* codes_u;
  float* scales_u;
  uint8_t* codes_w;
  float* scales_w;
} ifq_wl_layer;

size_t ifq_widely_linear_quantize_workspace_bytes(const ifq_wl_layer* layers, int count, int T);

ifq_status ifq_widely_linear_quantize_pack(const ifq_wl_layer* layers, int count, int T, void* workspace,
                                           size_t workspace_bytes, uint32_t* dev_status, ifq_stream_t stream);

/* ---------------------------------------------------------------------------
 * ifq_dequantize  ("Fairy2i write-up" §3.2, §4.1; "iFairy talk notes" §2.2.1)
 *
 * The dequantized weight W_hat = sum_t (s_re,t Re b_t + i s_im,t Im b_t) of each
 * tensor as bf16 planes, for the forward pass of quantization-aware training
 * (the straight-through backward passes the gradient unchanged and needs no
 * call).  Per entry the stage terms are added in float32 in stage order from +0
 * and the sum is rounded once to bf16, nearest-even.
 *
 *   tensors[i].codes        [T][N][K/4] uint8, device, read-only
 *   tensors[i].scales       [T][2] float32, device, read-only (4-byte aligned)
 *   tensors[i].N, K         N >= 1, K >= 4, K % 4 == 0
 *   tensors[i].w_re, w_im   [N][K] bf16 bit patterns, device, written
 *   count                   1..IFQ_MAX_GROUP tensors, one launch
 *   T                       1..IFQ_MAX_STAGES (the stages summed)
 * Pointers must be 16-byte aligned (scales: 4-byte).
 * ------------------------------------------------------------------------- */
typedef struct {
  const uint8_t* codes;
  const float* scales;
  int64_t N;
  int64_t K;
  uint16_t* w_re;
  uint16_t* w_im;
} ifq_dqtensor;

ifq_status ifq_dequantize(const ifq_dqtensor* tensors, int count, int T, ifq_stream_t stream);

/* ---------------------------------------------------------------------------
 * Product layers ("Fairy2i write-up" §2.1, §4.2; "iFairy article" §二.2)
 *
 *   y = sum_t ( U_hat_t x + W_hat_t conj(x) ),  per token,
 * where U_hat_t, W_hat_t are stage t of the two code sets.  Each code adds or
 * subtracts the real or imaginary part of x into a per-class float32
 * accumulator (no multiplications by weights); the scales are applied once per
 * (stage, branch) in the epilogue.
 *
 *   codes_u, scales_u   stage codes and scales of U (required)
 *   codes_w, scales_w   of W, applied to conj(x); both NULL = no conjugate branch
 *   N, K                outputs, inputs: N >= 1, K >= 4, K % 4 == 0 (the tensor-core
 *                       kernels take K % 64 == 0; a call with another K runs a
 *                       plain CUDA-core kernel with float64 sums, and ifq_gemv
 *                       then needs no workspace)
 *   x_re, x_im          [rows][K] bf16 bit patterns, device, 16-byte aligned
 *   y_re, y_im          [rows][N] float32, device, overwritten
 *                       ("device" means an address the GPU can use: x and y may
 *                       also be pinned host memory in the unified address space,
 *                       which the kernels then read and write over PCIe; for
 *                       ifq_gemv at B <= 2 x is read once, by the preparation
 *                       kernel, so that costs little)
 *   rot_re, rot_im      optional epilogue rotation, both NULL = none: when set,
 *                       output [r][n] is multiplied by the complex number
 *                       rot_re[r][n] + i rot_im[r][n] ([rows][N] float32,
 *                       device, 16-byte aligned) before it is stored.  This is
 *                       the complex rotary position encoding of the q and k
 *                       projections, one complex multiply per output ("iFairy
 *                       article" §三; "iFairy talk notes" §2.1.3): the caller
 *                       passes e^{i theta} for each token position and output.
 *                       Setting only one of the two is IFQ_ERR_NULL.
 * rows = B for ifq_gemv and M for ifq_gemm.
 *
 * The attention score of the complex model, Re(q^T conj(k)) ("Fairy2i write-up"
 * §2.2; "iFairy talk notes" §2.1.4), equals the real dot product of the stacked
 * vectors [q_re, q_im] and [k_re, k_im], so the planar outputs feed a standard
 * real attention kernel directly; the library has no score kernel of its own.
 * ------------------------------------------------------------------------- */
typedef struct {
  const uint8_t* codes_u;
  const float* scales_u;
  const uint8_t* codes_w;
  const float* scales_w;
  int64_t N;
  int64_t K;
  const uint16_t* x_re;
  const uint16_t* x_im;
  float* y_re;
  float* y_im;
  const float* rot_re;
  const float* rot_im;
} ifq_layer;

/* Decode product for B = 1..IFQ_MAX_GEMV_BATCH tokens per layer; all `count`
 * layers (1..IFQ_MAX_GROUP) run in one launch.  Codes stream from HBM once.
 *   B <= 2: exact integer tensor-core path.  Each code becomes two 0/1 planes
 *           of its Gray re-coding (g1 = sign, g0 = axis XOR sign, so that
 *           Re b = 1 - g0 - g1 and Im b = g0 - g1 are affine in the bits); the
 *           activations of each 2048-wide K block are scaled by a power of two
 *           and split into four signed 8-bit digits by a small preparation
 *           kernel; int32 accumulation is exact, and the only rounding is that
 *           of the activation scaling (below 2^-29 of the block's largest |x|
 *           per position, per token).  Partial sums are combined in a fixed
 *           order through the workspace, so results are bit-reproducible.
 *           B = 2 shares each operand's extraction between the tokens.
 *   B >= 3: codes expanded in registers to exact {-2, 0, +2} bf16 operands,
 *           float32 accumulation per axis class; a layer longer than 2048
 *           positions is cut into K segments whose partial sums are added in
 *           segment order through the workspace.
 * workspace: device scratch of ifq_gemv_workspace_bytes() bytes, 16-byte
 *           aligned, owned by the caller; no initial contents needed.  Calls
 *           that share a workspace must not overlap on the GPU.  May be NULL
 *           when ifq_gemv_workspace_bytes() returns 0 (B >= 3 with every
 *           K <= 2048).
 * dev_status may be NULL.  A NaN or Inf activation sets IFQ_DEV_NONFINITE
 * (B <= 2: the affected outputs are NaN); a lost pipeline wait sets
 * IFQ_DEV_TIMEOUT. */
size_t ifq_gemv_workspace_bytes(const ifq_layer* layers, int count, int T, int B);

ifq_status ifq_gemv(const ifq_layer* layers, int count, int T, int B, void* workspace, size_t workspace_bytes,
                    uint32_t* dev_status, ifq_stream_t stream);

/* Prepared decode calls, for a caller that repeats the same call (a decode loop): ifq_gemv_prepare
 * validates the arguments and stores everything the launches need -- the routing, and for the integer
 * tensor-core path (B <= 2) the finished kernel parameters with their tensor maps -- in a caller-owned HOST
 * buffer of ifq_gemv_plan_bytes() bytes, 64-byte aligned; ifq_gemv_run(plan, stream) then only
 * launches, and gives the same outputs as ifq_gemv with the same arguments.  Every tensor named by
 * the layers, the workspace and dev_status must stay allocated and in place while the plan is used
 * (new activations are written into the same x buffers).  The library keeps nothing: the plan is
 * the caller's, may be copied bytewise, and runs on any stream of the device it was made on.
 * Errors: ifq_gemv's; plan NULL is IFQ_ERR_NULL, too small IFQ_ERR_WORKSPACE, misaligned
 * IFQ_ERR_ALIGN; ifq_gemv_run of a buffer that ifq_gemv_prepare did not fill is IFQ_ERR_NULL. */
size_t ifq_gemv_plan_bytes(void);

ifq_status ifq_gemv_prepare(const ifq_layer* layers, int count, int T, int B, void* workspace,
                            size_t workspace_bytes, uint32_t* dev_status, void* plan, size_t plan_bytes);

ifq_status ifq_gemv_run(const void* plan, ifq_stream_t stream);

/* Prefill product for M >= 1 tokens (meant for M >= 128) on the tensor cores:
 * codes are expanded straight into TMEM as exact {-2, 0, +2} bf16 operands (the
 * MMA's A operand), the +-1 and +-i classes accumulate in separate rows of a
 * float32 TMEM accumulator, and the scales are applied per (stage, branch) in
 * the epilogue.  All layers of the call run in one persistent launch (one CTA
 * per SM over every layer's tiles, the layers with the longest K first).
 * dev_status may be NULL (timeouts then go unreported). */
ifq_status ifq_gemm(const ifq_layer* layers, int count, int T, int64_t M, uint32_t* dev_status,
                    ifq_stream_t stream);

/* As ifq_gemm, with every pipeline wait of the tensor-core kernel bounded by
 * wait_limit_ns (> 0) instead of 2 s.  A wait that runs out sets IFQ_DEV_TIMEOUT
 * in *dev_status; the kernel then lets its copies and MMAs in flight finish
 * (waits of up to 2 s), frees its TMEM and returns, so the context stays usable
 * and the next call runs normally.  The outputs of a call that timed out are
 * invalid.  For failure-detection tests and for callers with a tighter watchdog
 * than 2 s; ifq_gemm is this call with 2 s.  wait_limit_ns == 0 is
 * IFQ_ERR_SHAPE. */
ifq_status ifq_gemm_wait_limit(const ifq_layer* layers, int count, int T, int64_t M, uint64_t wait_limit_ns,
                               uint32_t* dev_status, ifq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* IFQ_H */
