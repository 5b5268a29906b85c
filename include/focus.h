/*
 * focus.h -- C ABI of libfocus.so: the FOCUS NVFP4 weight fake-quantizer on
 * NVIDIA B200 (sm_100a).
 *
 * FOCUS (Coupled-Relaxation and Dual-Granularity Scaling) learns, for every
 * linear weight W[out, in] of a frozen BF16 model, one factor m per 16-element
 * block and one logit q per 8-element sub-block.  The source of every formula
 * is the model card "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct (our
 * reproduction)", section "What this is" (field table, layout sentence and the
 * three equations with the rules that follow them) and section "Calibration"
 * (optimizer and learning rates); the straight-through estimator is named in
 * "Technische Samenvatting: FOCUS ...", section "Methodologie", item 1.
 *
 * Per block b (16 weights along in_features) with sub-blocks k = 0, 1 (8 each):
 *   A_b  = max |w_i|
 *   x_b  = fl(fl(A_b * m_b) / fl(6 * s2));  x_b == 0 -> 1
 *   S_b  = e4m3_rne(clamp(x_b, 2^-6, 448))
 *   D_k  = fl(fl(S_b * sigmoid(q_k)) * s2)
 *   y_i  = fl(w_i / D_k)
 *   c_i  = E2M1_rne(clamp(y_i, -6, 6))             (ties to even, sign kept)
 *   w'_i = bf16_rne(fl(fl(c_i * S_b) * s2))
 * All arithmetic is IEEE binary32 with one rounding per operation; sigmoid is
 * the binary32 rounding of 1/(1+exp(-q)) evaluated in binary64.
 *
 * Besides the FOCUS calls (s2, forward, straight-through backward, AdamW, the
 * fused step, the NVFP4 pack; single tensors or a whole model as a table) the
 * library has the rows around them: FourOverSix and plain NVFP4 round to
 * nearest of weights and of activations with one scale per token, the MXFP4
 * variant of FOCUS, the 128x4 scale layout of sm_100 block-scaled GEMMs, and
 * the fused step over tensors held in host memory.
 *
 * Conventions for every call:
 *  - Tensors are dense row-major.  W, dW' and W' are bf16, passed as uint16_t
 *    bit patterns.  m is float[out][in/16], q is float[out][in/8]: m[r][b]
 *    belongs to W[r][16b..16b+15], q[r][2b+k] to W[r][16b+8k..16b+8k+7].
 *  - Pointers named *_dev, and every tensor pointer, are device pointers
 *    (cudaMalloc / PyTorch CUDA memory) on the current device; their base
 *    addresses must be 16-byte aligned.  Parameters passed by value or through
 *    a host pointer are read before the call returns.  (focus_step_host is the
 *    one exception: its tensors are in host memory; see there.)
 *  - The caller owns every buffer and the stream.  The library allocates no
 *    device or host memory of its own; temporary storage is passed in as a
 *    workspace.
 *  - Every call only enqueues work on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and returns at once, except focus_get_error and
 *    focus_step_host, which block.  The return value reports the argument
 *    checks (done on the host, before anything is enqueued) and the launch
 *    status; a failed check enqueues nothing.
 *  - Non-finite values in W, m or q, and an invalid s2 read from device
 *    memory, are outside the contract: kernels never trap on them, they set a
 *    sticky device flag that focus_get_error() reports.  Every wait inside a
 *    kernel is bounded in time; a wait that runs out sets the flag too.
 *  - in must be a multiple of 16; out >= 0 (an empty tensor is a no-op).
 */
#ifndef FOCUS_H
#define FOCUS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void *focus_stream_t; /* a cudaStream_t */

typedef enum focus_status {
    FOCUS_OK = 0,
    FOCUS_ERR_NULL = 1,             /* a required pointer is NULL */
    FOCUS_ERR_SHAPE = 2,            /* in % 16 != 0, out < 0, n < 0, or a tensor of more than
                                       2^31 - 2^16 blocks (out*in/16) */
    FOCUS_ERR_ALIGN = 3,            /* a tensor base address is not 16-byte aligned */
    FOCUS_ERR_VALUE = 4,            /* s2 <= 0 or not finite, lr < 0, step < 1, beta outside [0,1) ... */
    FOCUS_ERR_WORKSPACE = 5,        /* workspace missing or smaller than required */
    FOCUS_ERR_CUDA = 6,             /* a CUDA runtime call or a launch failed */
    FOCUS_ERR_NONFINITE_INPUT = 7,  /* reported by focus_get_error(): a kernel met a non-finite input
                                       or gradient, or an invalid s2 in a table */
    FOCUS_ERR_DEVICE_TIMEOUT = 8    /* reported by focus_get_error(): a kernel's staging pipeline
                                       gave up waiting (2 s) and left its work unfinished */
} focus_status;

/* Human-readable name of a status code (static storage; never NULL). */
const char *focus_status_string(int status);

/* ---------------------------------------------------------------------------
 * Per-tensor scale s2 = amax(|W|) / (6 * 448).
 * Card, field table, row "s2": one FP32 scale per tensor, frozen, computed from
 * the base weights.  Two passes: every CTA writes the max |w| of its tile into
 * the workspace, then one CTA reduces those maxima and divides once by 2688.
 * The result is exact (max is order-free; one correctly rounded division).
 *   W       [out, in] bf16, device
 *   s2_dev  one float, device, written
 *   ws_dev  device workspace of at least focus_s2_workspace_bytes(out, in)
 *           bytes, 16-byte aligned; its contents on entry do not matter.
 * An all-zero W gives s2 = 0, which the other calls reject.
 * ------------------------------------------------------------------------- */
size_t focus_s2_workspace_bytes(int64_t out, int64_t in);
int focus_s2(const uint16_t *W, int64_t out, int64_t in, float *s2_dev, void *ws_dev,
             size_t ws_bytes, focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * s2 without a workspace: the same result as focus_s2, for callers that
 * cannot give the library device memory (a runtime whose own memory pool owns
 * every device allocation, or a path that must never call cudaMalloc, which
 * can synchronize the device).  The pages describe nothing like it; it only
 * changes where the per-tile maxima live: in a 256 KB array inside the
 * library's device image, held on every GPU that loads the library until the
 * process exits.  This call allocates nothing.  (The CUDA runtime loads the
 * library's device code on a device when any of its entry points first runs
 * there, which reserves its device globals, this array among them, and may
 * synchronize; a caller that must avoid that on its critical path makes one
 * warm-up call beforehand.  Later calls allocate nothing.)
 *   W       [out, in] bf16, device; at most FOCUS_S2_NOALLOC_MAX_WEIGHTS
 *           weights, else FOCUS_ERR_WORKSPACE and nothing is enqueued;
 *           out = 0 gives s2 = 0, as focus_s2
 *   s2_dev  one float, device, written
 * The first call on a device (with that device current) looks up the array's
 * device address; make that first call before any stream capture.  If the
 * lookup fails the call returns FOCUS_ERR_CUDA and the next call tries again.
 * All calls share the array: calls whose work may overlap on the GPU
 * (different streams without ordering between them) race and must not be
 * issued.
 * ------------------------------------------------------------------------- */
#define FOCUS_S2_NOALLOC_MAX_WEIGHTS 268435456 /* 65,536 tiles of 4096 weights */
int focus_s2_noalloc(const uint16_t *W, int64_t out, int64_t in, float *s2_dev, focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * Forward fake-quantization W -> W'.
 * Card, "What this is": the S_b, c_i and w'_i equations.
 *   W   [out, in] bf16, device (read)
 *   m   [out, in/16] float, device (read)
 *   q   [out, in/8] float, device (read)
 *   s2  the tensor scale, by value: finite and > 0, else FOCUS_ERR_VALUE
 *   Wq  [out, in] bf16, device (written; must not overlap W)
 * ------------------------------------------------------------------------- */
int focus_fwd(const uint16_t *W, const float *m, const float *q, float s2, int64_t out, int64_t in,
              uint16_t *Wq, focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * Straight-through backward for m and q.
 * "Technische Samenvatting: FOCUS ...", "Methodologie" item 1 (scales learned
 * through the straight-through estimator), applied to the card's equations:
 * rounding (E2M1 and E4M3) acts as the identity; the clamps pass the gradient
 * at and inside their bounds and block it outside; the zero-block rule blocks
 * it.  With g_i the gradient of w'_i, in_i = [-6 <= y_i <= 6] and
 * inS_b = [x_b != 0 and 2^-6 <= x_b <= 448]:
 *   dL/dm_b   = inS_b * (A_b/6) * sum_{i in b} g_i * (in_i ? c_i - y_i : c_i)
 *   dL/dq_k   = -(1 - sigmoid(q_k)) * S_b * s2 * sum_{i in k} in_i * g_i * y_i
 *   W, dWq     [out, in] bf16, device (read); dWq is dL/dW'
 *   m, q       as in focus_fwd (read)
 *   dm         [out, in/16] float, device; dq [out, in/8] float, device
 *   accumulate 0: dm, dq are overwritten; 1: the gradients are added to them
 * Sums are formed in binary32 (order fixed per block).
 * ------------------------------------------------------------------------- */
int focus_ste_bwd(const uint16_t *W, const uint16_t *dWq, const float *m, const float *q, float s2,
                  int64_t out, int64_t in, float *dm, float *dq, int accumulate, focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * AdamW update of a parameter vector, in place.
 * Card, "Calibration": AdamW with betas 0.9/0.999, weight decay 0 and a
 * constant learning rate (5e-3 for m, 1e-3 for q).  Decoupled weight decay and
 * bias correction, step counted from 1:
 *   p <- p*(1 - lr*wd); v1 <- b1*v1 + (1-b1)*g; v2 <- b2*v2 + (1-b2)*g^2
 *   p <- p - (lr/(1-b1^t)) * v1 / (sqrt(v2)/sqrt(1-b2^t) + eps)
 *   p, exp_avg, exp_avg_sq  n floats, device (read and written)
 *   g                       n floats, device (read)
 *   lr >= 0, 0 <= beta1, beta2 < 1, eps >= 0, weight_decay >= 0, step >= 1
 * ------------------------------------------------------------------------- */
int focus_adamw_step(float *p, const float *g, float *exp_avg, float *exp_avg_sq, int64_t n, float lr,
                     float beta1, float beta2, float eps, float weight_decay, int64_t step,
                     focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * NVFP4 export pack.
 * Card, "What this is": the deployed model is plain NVFP4 -- E2M1 elements,
 * one E4M3 scale per 16 elements, one FP32 scale per tensor.  Byte layout (the
 * card gives none; this is the common one):
 *   codes             [out, in/2] uint8, device: byte j of a row holds element
 *                     2j in bits 0-3 and element 2j+1 in bits 4-7 (sign bit 3/7)
 *   scales            [out, in/16] uint8, device: the E4M3 byte of S_b
 *   tensor_scale_dev  one float, device: s2 (a dequantization multiplier,
 *                     w' = c * S_b * s2)
 * Other arguments as in focus_fwd.
 * ------------------------------------------------------------------------- */
int focus_pack_nvfp4(const uint16_t *W, const float *m, const float *q, float s2, int64_t out, int64_t in,
                     uint8_t *codes, uint8_t *scales, float *tensor_scale_dev, focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * Multi-tensor interface: every linear weight of a model in one launch.
 *
 * A table of focus_tensor_desc lives in DEVICE memory.  The caller fills the
 * table on the host, calls focus_table_prepare() on it (which checks every
 * entry and fills the two *_begin fields), copies it to device memory and then
 * passes the device copy to the calls below, step after step.  The table must
 * not change without being prepared again.
 * ------------------------------------------------------------------------- */
typedef struct focus_tensor_desc {
    const uint16_t *W;     /* [out, in] bf16 base weight (read) */
    const uint16_t *dWq;   /* [out, in] bf16 dL/dW' (read by focus_step_fused; may be NULL otherwise) */
    uint16_t *Wq;          /* [out, in] bf16 W' (written when not NULL) */
    float *m;              /* [out, in/16] */
    float *q;              /* [out, in/8] */
    float *m_exp_avg;      /* AdamW first moment of m  (focus_step_fused) */
    float *m_exp_avg_sq;   /* AdamW second moment of m (focus_step_fused) */
    float *q_exp_avg;      /* AdamW first moment of q  (focus_step_fused) */
    float *q_exp_avg_sq;   /* AdamW second moment of q (focus_step_fused) */
    float *s2;             /* one float: written by focus_s2_multi, read by the others */
    uint8_t *codes;        /* [out, in/2] NVFP4 codes (written when not NULL) */
    uint8_t *scales;       /* [out, in/16] E4M3 scale bytes (written when not NULL) */
    float *dm;             /* [out, in/16] gradient buffer, see FOCUS_STEP_* flags (may be NULL) */
    float *dq;             /* [out, in/8]  gradient buffer, see FOCUS_STEP_* flags (may be NULL) */
    int64_t out;
    int64_t in;
    int64_t block_begin;   /* filled by focus_table_prepare: sum of out*in/16 over earlier entries */
    int64_t tile_begin;    /* filled by focus_table_prepare: first work tile of this entry */
} focus_tensor_desc;

typedef struct focus_hparams {
    float lr_m;            /* 5e-3 on the card */
    float lr_q;            /* 1e-3 on the card */
    float beta1;           /* 0.9 */
    float beta2;           /* 0.999 */
    float eps;             /* 1e-8 */
    float weight_decay;    /* 0 */
} focus_hparams;

/* focus_table_prepare purpose of a table for the MXFP4 multi-tensor calls. */
#define FOCUS_PURPOSE_MX 4
/* focus_table_prepare purposes of a table of activation tensors for the
 * per-token calls focus_fouroversix_act_multi / focus_nvfp4_act_multi: block
 * scales row-major (5) or in the 128x4-atom layout (6). */
#define FOCUS_PURPOSE_ACT 5
#define FOCUS_PURPOSE_ACT_SWIZZLED 6

/* Flags of focus_step_fused. */
#define FOCUS_STEP_ACCUMULATE 1u  /* add dm/dq (earlier micro-batches) to this step's gradients */
#define FOCUS_STEP_WRITE_GRAD 2u  /* write the gradients used by the update into dm/dq */
#define FOCUS_STEP_PACK_UPDATED 4u /* codes/scales receive the NVFP4 export of the UPDATED m and q (what
                                      focus_pack_multi would write after this call) instead of the
                                      forward's; W is not read again */
#define FOCUS_STEP_WQ_UPDATED 8u   /* W' receives the forward of the UPDATED m and q (what focus_fwd_multi
                                      would write after this call: the next step's fake-quantized
                                      weight) instead of the forward's */

/* Checks every entry (pointers, alignment, shapes, which inputs are present
 * for `purpose`: 0 = s2/forward/pack, 1 = also focus_step_fused (dWq and the
 * four moments), 2 = also focus_ste_bwd_multi (dWq, dm, dq), 3 = s2 and
 * FourOverSix only (W and s2; m and q may be NULL; codes+scales or Wq),
 * FOCUS_PURPOSE_MX (4) = the MXFP4 calls focus_mx_*_multi (in % 32 == 0; W,
 * m and q present; s2 unused; the other pointers optional here and checked by
 * the kernels: an entry lacking one its call needs is skipped and flagged),
 * FOCUS_PURPOSE_ACT (5) and FOCUS_PURPOSE_ACT_SWIZZLED (6) = the per-token
 * calls focus_*_act_multi (W = X [tokens = out, hidden = in] with hidden at
 * most 16384, s2 = the token scales [tokens], codes and scales present, Wq =
 * X' optional))
 * and fills block_begin and tile_begin (for purpose 4 in 32-blocks and tiles
 * of 128 of them: 4096 weights, as for the other purposes; for purposes 5 and
 * 6 the work unit is a bundle of consecutive rows of one entry -- as many as
 * 256 threads cover with at most 4 blocks each, e.g. 4 rows of 4096 values, 1
 * of 14336 -- tile_begin is the entry's first bundle, and the rows of every
 * entry count padded to a multiple of 128 for purpose 6).  Host memory in,
 * host memory out.
 * *total_tiles receives the number of work units (tiles; for purposes 5 and
 * 6 bundles of rows), passed to the calls below.
 * A device-resident table cannot be checked again at call time: a kernel that
 * meets an entry lacking a pointer it needs skips that entry and sets the
 * device flag (FOCUS_ERR_NONFINITE_INPUT from focus_get_error). */
int focus_table_prepare(focus_tensor_desc *descs_host, int n_tensors, int purpose, int64_t *total_tiles);

/* Workspace bytes focus_s2_multi needs for a prepared table. */
size_t focus_s2_multi_workspace_bytes(int64_t total_tiles);

/* s2 of every entry (two launches). */
int focus_s2_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles, void *ws_dev,
                   size_t ws_bytes, focus_stream_t stream);

/* One calibration step of every entry in one launch, W read once:
 * forward (W' when desc.Wq != NULL, codes/scales when present), straight-
 * through backward, AdamW on m and q (lr_m for m, lr_q for q) at step `step`.
 * hp is a host pointer.  flags: FOCUS_STEP_ACCUMULATE, FOCUS_STEP_WRITE_GRAD
 * (both need desc.dm and desc.dq), FOCUS_STEP_PACK_UPDATED,
 * FOCUS_STEP_WQ_UPDATED.  W', codes and scales are the forward's, i.e. of m
 * and q before the update, unless FOCUS_STEP_WQ_UPDATED / _PACK_UPDATED make
 * them those of the updated m and q. */
int focus_step_fused(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles,
                     const focus_hparams *hp, int64_t step, unsigned flags, focus_stream_t stream);

/* The same step, also computing each entry's s2 for the next step: the step
 * reduces the block maxima it computes anyway into the tensor's max |w|
 * (bf16 magnitude bits, atomically maximised into amax_ws[i] for entry i), and
 * focus_s2_from_amax then writes desc.s2 = fl(max / 2688) -- card, field
 * table, row s2 -- and clears amax_ws.  W is frozen, so this is the s2 a
 * separate focus_s2_multi pass would compute, without a second read of W.
 *   amax_ws  n_tensors uint32 words, device, 16-byte aligned; zero before the
 *            first step (focus_s2_from_amax leaves it zero for the next one).
 * The step itself reads desc.s2 as focus_step_fused does (the previous value,
 * or one from focus_s2_multi before the first step). */
int focus_step_fused_amax(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles,
                          const focus_hparams *hp, int64_t step, unsigned flags, uint32_t *amax_ws,
                          focus_stream_t stream);
int focus_s2_from_amax(const focus_tensor_desc *descs_dev, int n_tensors, uint32_t *amax_ws, focus_stream_t stream);

/* Forward of every entry in one launch: W' (desc.Wq), and the codes and
 * scales when present.  Card, "What this is": the S_b, c_i and w'_i
 * equations. */
int focus_fwd_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles,
                    focus_stream_t stream);

/* Straight-through backward of every entry in one launch (as focus_ste_bwd):
 * desc.dm/dq receive the gradients, added to what they hold when
 * accumulate = 1 -- the micro-batches of a step before the one that runs
 * focus_step_fused with FOCUS_STEP_ACCUMULATE.  The table needs purpose 2. */
int focus_ste_bwd_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles, int accumulate,
                        focus_stream_t stream);

/* NVFP4 pack of every entry with codes and scales present (desc.s2 holds the
 * tensor scale, which the caller exports). */
int focus_pack_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles,
                     focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * FourOverSix round to nearest: plain NVFP4 (E2M1 codes, one E4M3 scale per
 * 16 elements, an FP32 scale per tensor or per token) in which every block's
 * scale maps the block maximum to 6 or to 4, whichever gives the lower
 * squared error.  Model card "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct",
 * section "Calibration" (activation bullet: one scale per token) and section
 * "Perplexity" (round-to-nearest FourOverSix weights, the reference row);
 * "Llama-3.1-8B-Instruct FlipQuant MixFP4 maps", section "What this is".
 * Per block, for the targets T = 6 and T = 4 (s the tensor or token scale):
 *   x_T = fl(A_b / fl(T*s));  x_T == 0 -> 1;  S_T = e4m3_rne(clamp(x_T, 2^-6, 448))
 *   c_i = E2M1_rne(clamp(fl(w_i / fl(S_T*s)), -6, 6))
 *   err_T = sum_i (w_i - c_i*S_T*s)^2, the exact squared error
 * The target 4 is taken when err_4 < err_6 exactly (a tie keeps 6; exact ties
 * occur, about one block in 10^7 of Gaussian weights).  The kernels screen the
 * choice with binary32 sums and decide the blocks within 2^-19 of a tie by an
 * exact comparison.  The dequantized value is bf16(fl(fl(c_i*S)*s)).  Outputs use the focus_pack_nvfp4 layout
 * (codes [rows][cols/2], element 2j in the low nibble; scales [rows][cols/16]).
 * ------------------------------------------------------------------------- */

/* Weights with the tensor scale s2 (by value: finite and > 0, else
 * FOCUS_ERR_VALUE).  W [out, in] bf16, device; codes/scales (both or
 * neither) and Wq [out, in] bf16 (nullable) are device outputs; at least one
 * of codes or Wq is required.  Non-finite weights set the device flag. */
int focus_fouroversix_weight(const uint16_t *W, int64_t out, int64_t in, float s2, uint8_t *codes,
                             uint8_t *scales, uint16_t *Wq, focus_stream_t stream);

/* The same over every entry of a table (purpose 3, or any purpose whose
 * entries carry codes+scales or Wq) in one launch: desc.W, desc.s2 (device,
 * as focus_s2_multi writes it), desc.codes/scales and desc.Wq. */
int focus_fouroversix_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles,
                            focus_stream_t stream);

/* Plain NVFP4 round to nearest of weights with the tensor scale s2 (the
 * card's NVFP4 baseline, section "Perplexity": round-to-nearest NVFP4
 * weights): the block equations with m = 1 and sigmoid = 1, i.e. the target 6
 * alone; arguments and outputs exactly as focus_fouroversix_weight and
 * focus_fouroversix_multi. */
int focus_nvfp4_weight(const uint16_t *W, int64_t out, int64_t in, float s2, uint8_t *codes, uint8_t *scales,
                       uint16_t *Wq, focus_stream_t stream);
int focus_nvfp4_weight_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles,
                             focus_stream_t stream);

/* Activations with one scale per token: X [tokens, hidden] bf16, device
 * (hidden % 16 == 0); token_scales [tokens] float, device, receives
 * s_t = fl(max_row |x| / 2688); codes [tokens][hidden/2], scales
 * [tokens][hidden/16] and Xq [tokens, hidden] bf16 (nullable) are device
 * outputs.  A row whose maximum is 0 gets s_t = 0, scale bytes 0x38, codes 0
 * and values 0.  A row holding a non-finite value sets the device flag and
 * its outputs are left unwritten.  One launch; X is read from HBM once
 * (rows of up to 16384 values are staged in shared memory, longer rows are
 * read a second time from L2). */
int focus_fouroversix_act(const uint16_t *X, int64_t tokens, int64_t hidden, float *token_scales,
                          uint8_t *codes, uint8_t *scales, uint16_t *Xq, focus_stream_t stream);

/* The same, with the block scales written straight into the 128x4-atom layout
 * that focus_scales_swizzle produces (declared below), the layout an sm_100
 * block-scaled GEMM reads for its activation operand: scales_swz (device, at
 * least focus_scales_swizzled_bytes(tokens, hidden/16) bytes, else
 * FOCUS_ERR_WORKSPACE) receives every byte, padding rows and columns 0.  The
 * result equals focus_fouroversix_act followed by focus_scales_swizzle, in one
 * launch.  A row holding a non-finite value sets the device flag and leaves
 * its outputs, padding columns included, unwritten. */
int focus_fouroversix_act_swizzled(const uint16_t *X, int64_t tokens, int64_t hidden, float *token_scales,
                                   uint8_t *codes, uint8_t *scales_swz, size_t scales_bytes, uint16_t *Xq,
                                   focus_stream_t stream);

/* The same over every entry of a table of activation tensors prepared with
 * FOCUS_PURPOSE_ACT (block scales row-major; swizzled = 0) or
 * FOCUS_PURPOSE_ACT_SWIZZLED (the 128x4-atom layout, each entry's scales
 * buffer at least focus_scales_swizzled_bytes(tokens, hidden/16) bytes;
 * swizzled = 1), in one launch: total_rows = the work count
 * focus_table_prepare returned (bundles of rows),
 * max_hidden at least every entry's hidden (a multiple of 16, at most 16384,
 * else FOCUS_ERR_SHAPE; an entry wider than max_hidden is skipped and sets
 * the device flag).  Every entry as the single-tensor call: desc.W = X,
 * desc.s2 = token scales (written), desc.codes, desc.scales, desc.Wq = X'
 * (nullable).  Rows of up to 16384 values are staged in shared memory, so X
 * is read from HBM once. */
int focus_fouroversix_act_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_rows,
                                int64_t max_hidden, int swizzled, focus_stream_t stream);

/* Plain NVFP4 round to nearest with one scale per token: the NVFP4 baseline
 * of the card's section "Perplexity" (NVFP4 activations with one scale per
 * token), read as the block equations with m = 1 and sigmoid = 1 and the
 * token's scale s_t = fl(max_row |x| / 2688) in place of s2:
 *   S_b = e4m3(clamp(fl(A_b / fl(6*s_t)), 2^-6, 448)) (x == 0 -> 1)
 *   c_i = E2M1_rne(clamp(fl(x_i / fl(S_b*s_t)), -6, 6));  x'_i = bf16(fl(fl(c_i*S_b)*s_t))
 * Arguments, layouts, the zero-row and non-finite rules exactly as
 * focus_fouroversix_act / focus_fouroversix_act_swizzled. */
int focus_nvfp4_act(const uint16_t *X, int64_t tokens, int64_t hidden, float *token_scales, uint8_t *codes,
                    uint8_t *scales, uint16_t *Xq, focus_stream_t stream);
int focus_nvfp4_act_swizzled(const uint16_t *X, int64_t tokens, int64_t hidden, float *token_scales, uint8_t *codes,
                             uint8_t *scales_swz, size_t scales_bytes, uint16_t *Xq, focus_stream_t stream);
/* ... and over a table, as focus_fouroversix_act_multi. */
int focus_nvfp4_act_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_rows, int64_t max_hidden,
                          int swizzled, focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * MXFP4 variant: 32-element blocks with an E8M0 scale and four sub-blocks of
 * 8, no tensor scale.  "Technische Samenvatting: FOCUS ...", sections
 * "Probleemstelling" (MXFP4 shares an E8M0 scale per 32 values) and
 * "Methodologie" items 2-3 (hardware scale x learnable coefficient; sub-blocks
 * of 8 inside each hardware block of 32); the card's equations give the
 * structure.  The pages give no MXFP4 formula; the scale follows the OCP
 * Microscaling rule on the scaled maximum.  Per block b, sub-blocks k = 0..3:
 *   x_b = fl(A_b * m_b);  S_b = 2^(floor(log2 x_b) - 2), exponent clamped to
 *   [-127, 127]; S_b = 1 when x_b == 0
 *   D_k = fl(S_b * sigmoid(q_k));  c_i = E2M1_rne(clamp(fl(w_i/D_k), -6, 6))
 *   w'_i = bf16(fl(c_i * S_b))
 *   dm_b = [x_b >= 2^-125] (A_b/4) sum_i g_i (in_i ? c_i - y_i : c_i)
 *   dq_k = -(1 - sigma_k) S_b sum_{i in k} in_i g_i y_i
 * Layout: W, dW', W' bf16 [out][in] with in % 32 == 0 (else FOCUS_ERR_SHAPE);
 * m and its moments float [out][in/32]; q and its moments float [out][in/8]
 * (q[r][4b+k]); codes [out][in/2] (element 2j in the low nibble); scales
 * [out][in/32] E8M0 bytes (exponent + 127).  All device pointers, 16-byte
 * aligned; one tensor per call.
 * ------------------------------------------------------------------------- */

/* Forward: Wq (nullable) and codes+scales (both or neither; at least one
 * output). */
int focus_mx_fwd(const uint16_t *W, const float *m, const float *q, int64_t out, int64_t in, uint16_t *Wq,
                 uint8_t *codes, uint8_t *scales, focus_stream_t stream);

/* Straight-through backward into dm [out][in/32], dq [out][in/8] (added to
 * what they hold when accumulate = 1). */
int focus_mx_ste_bwd(const uint16_t *W, const uint16_t *dWq, const float *m, const float *q, int64_t out,
                     int64_t in, float *dm, float *dq, int accumulate, focus_stream_t stream);

/* One fused step of one tensor: forward (W' when Wq != NULL), straight-through
 * backward, AdamW on m (lr_m) and q (lr_q) in place.  flags:
 * FOCUS_STEP_ACCUMULATE, FOCUS_STEP_WRITE_GRAD (both need dm and dq),
 * FOCUS_STEP_WQ_UPDATED (Wq receives the forward of the UPDATED m and q: what
 * focus_mx_fwd would write after the call); other bits give FOCUS_ERR_VALUE. */
int focus_mx_step(const uint16_t *W, const uint16_t *dWq, float *m, float *q, float *m_exp_avg,
                  float *m_exp_avg_sq, float *q_exp_avg, float *q_exp_avg_sq, int64_t out, int64_t in,
                  const focus_hparams *hp, int64_t step, unsigned flags, uint16_t *Wq, float *dm, float *dq,
                  focus_stream_t stream);

/* The same three over every entry of a table prepared with FOCUS_PURPOSE_MX,
 * in one launch each (per entry: W, m, q; the forward writes Wq and/or
 * codes+scales, whichever the entry has; the backward needs dWq, dm, dq; the
 * step needs dWq and the four moments, writes Wq and codes+scales when
 * present, and needs dm, dq under FOCUS_STEP_ACCUMULATE /
 * FOCUS_STEP_WRITE_GRAD).  The step's flags also take FOCUS_STEP_PACK_UPDATED
 * (codes+scales of the UPDATED m and q: what focus_mx_fwd_multi would write
 * after the call; W is not read again) and FOCUS_STEP_WQ_UPDATED (W' of the
 * updated m and q); without them the step writes the forward's.  An entry
 * lacking a pointer its call needs is skipped and sets the device flag. */
int focus_mx_fwd_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles,
                       focus_stream_t stream);
int focus_mx_ste_bwd_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles, int accumulate,
                           focus_stream_t stream);
int focus_mx_step_multi(const focus_tensor_desc *descs_dev, int n_tensors, int64_t total_tiles,
                        const focus_hparams *hp, int64_t step, unsigned flags, focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * Scale factors for sm_100 block-scaled GEMMs.  The pages deploy the export
 * as plain NVFP4 for standard NVFP4 kernels (card, "What this is"); on sm_100
 * those kernels (cuBLASLt's NVFP4 GEMM, the tcgen05 block-scaled MMA; PyTorch
 * calls the layout SWIZZLE_32_4_4) read an operand's E4M3 scales [rows][K/16]
 * in NVIDIA's 128x4 layout: rows padded to 128 and columns to 4, atoms of 128
 * rows x 4 columns (512 bytes) stored band by band with the column groups
 * inner, scale (r, c) of an atom at byte 16*(r mod 32) + 4*(r div 32) + c.
 *   scales  [rows][cols] u8, device, as focus_pack_nvfp4 / the FourOverSix
 *           calls write them (cols = K/16)
 *   out     device, at least focus_scales_swizzled_bytes(rows, cols) bytes
 *           (else FOCUS_ERR_WORKSPACE); every byte is written, padding 0
 * ------------------------------------------------------------------------- */
size_t focus_scales_swizzled_bytes(int64_t rows, int64_t cols);
int focus_scales_swizzle(const uint8_t *scales, int64_t rows, int64_t cols, uint8_t *out, size_t out_bytes,
                         focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * The fused step over tensors held in HOST memory (the same computation as
 * focus_step_fused_amax + focus_s2_from_amax on device-resident tensors).
 *
 * host_descs: n_tensors focus_tensor_desc in host memory whose pointers are
 * HOST pointers: W, dWq (read), m, q and the four moments (read, then
 * overwritten with the updated values), s2 (one float: read unless
 * FOCUS_HOST_S2_FIRST, then overwritten with s2 for the next step), Wq and
 * codes+scales (optional outputs, written); dm and dq must be NULL
 * (FOCUS_ERR_VALUE); block_begin and tile_begin are ignored.  Shapes as in
 * focus_table_prepare (in % 16 == 0); empty tensors are skipped.
 *
 * Per tensor, in three device slots carved from the caller's workspace: the
 * inputs are uploaded, the step (with s2 first under FOCUS_HOST_S2_FIRST, and
 * the tensor maximum) runs on `stream`, and the outputs are read back; the
 * upload and read-back of neighbouring tensors run on two streams of the call
 * while a tensor is stepped.  Host buffers should be pinned (page-locked):
 * pageable buffers give the same results, with the copies serialised by the
 * host.
 *
 * ws_dev: device memory, 256-byte aligned, at least
 * focus_step_host_workspace_bytes(host_descs, n_tensors) bytes (three slots
 * of 8.81 bytes per weight of the largest tensor plus small fields), else
 * FOCUS_ERR_WORKSPACE.  flags: FOCUS_STEP_PACK_UPDATED, FOCUS_STEP_WQ_UPDATED,
 * FOCUS_HOST_S2_FIRST; others give FOCUS_ERR_VALUE.  Every entry is checked on
 * the host before anything is enqueued (a missing pointer: FOCUS_ERR_NULL; a
 * stored s2 that is not finite and > 0 without FOCUS_HOST_S2_FIRST:
 * FOCUS_ERR_VALUE).
 *
 * BLOCKING: the call returns when every result is in host memory (it creates
 * and releases its two copy streams and its events).  The device flag is
 * reported by focus_get_error as for the other calls.  An entry the step
 * skips (an all-zero W under FOCUS_HOST_S2_FIRST gives s2 = 0; the flag is
 * set) gets its m, q and moments back unchanged and s2 = 0; its Wq, codes and
 * scales are then undefined.
 * ------------------------------------------------------------------------- */
#define FOCUS_HOST_S2_FIRST 16u   /* compute s2 from W in the slot before the step (first step) */
size_t focus_step_host_workspace_bytes(const focus_tensor_desc *host_descs, int n_tensors);
int focus_step_host(const focus_tensor_desc *host_descs, int n_tensors, const focus_hparams *hp, int64_t step,
                    unsigned flags, void *ws_dev, size_t ws_bytes, focus_stream_t stream);

/* ---------------------------------------------------------------------------
 * Synchronizes `stream`, then reports and clears the sticky device flag:
 * FOCUS_ERR_DEVICE_TIMEOUT when a kernel's pipeline wait ran out,
 * FOCUS_ERR_NONFINITE_INPUT when any kernel since the last call met a
 * non-finite W/m/q value or gradient or an invalid s2 read from a table,
 * FOCUS_ERR_CUDA when the stream reports an error, else FOCUS_OK.
 * ------------------------------------------------------------------------- */
int focus_get_error(focus_stream_t stream);

/* Library version, "major.minor.patch" (static storage). */
const char *focus_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FOCUS_H */
