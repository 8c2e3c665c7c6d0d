/*
 * pl.h -- C ABI of the B200 (sm_100a) fused GRPO/BNPO policy-loss library (libpl.so).
 *
 * Two forms of one hot path, both defined by the pages this library restates:
 *
 *   pl_loss / pl_loss_ex -- the loss-only kernel on precomputed log-probs:
 *       ratio     = exp(policy_lp - old_lp)
 *       clipped   = clip(ratio, 1 - eps_lo, 1 + eps_hi)
 *       per_token = -adv[b] * min(ratio, clipped)
 *       kl        = exp(ref_lp - policy_lp) - (ref_lp - policy_lp) - 1
 *       BNPO: loss = sum(mask * (per_token + beta*kl)) / max(sum(mask), 1)
 *       GRPO: loss = mean_b( sum_t(mask * (per_token + beta*kl)) / max(sum_t mask, 1) )
 *     ("Geometric-AI Kernels" model card, sections "BNPO Loss" and "GRPO Loss";
 *      the fused forward+backward returning (loss, grad_logprobs) and the
 *      forward-only variant are the card's "Entry points" section).
 *
 *   pl_fused_linear_grpo -- the fused linear path: hidden states x lm_head weight ->
 *     per-token log-prob of the sampled token (logsumexp over the whole vocabulary,
 *     temperature 1.0) for the policy and the reference model -> the loss above ->
 *     grad_logits = g * (onehot - softmax) -> dX, dW, dbias, in row chunks of at
 *     most 1024 with fp32 weight-gradient accumulation across chunks
 *     ("Add SM100 CuTe DSL GRPO fast path", Liger-Kernel PR #1363, sections
 *      "Summary", "Why it is faster and uses less memory" and "Native scope").
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers to contiguous row-major arrays on the
 *     current CUDA device; the caller owns every buffer.  Nothing is freed or
 *     retained by the library except the per-(device, stream) scratch of pl_loss.
 *   - Work is enqueued on `stream` (a cudaStream_t; 0 = legacy default stream) and
 *     the calls return without synchronising the host.
 *   - Host-detectable problems (NULL required pointer, negative size, unsupported
 *     dtype, workspace too small, a device that is not compute capability 10.0)
 *     return an error code before any launch and before any output is written.
 *   - Problems only the device can see (a bounded wait that ran out, a target id
 *     outside [0, V)) set a sticky flag in the workspace; outputs are then
 *     undefined.  Read and clear it with pl_device_status().  After a wait that
 *     ran out, zero-fill a caller-owned workspace again before reusing it (a
 *     call cut short may leave its counters set).
 *   - No exception crosses this boundary.
 */
#ifndef PL_H_
#define PL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so this header needs no CUDA header. */
typedef struct CUstream_st* pl_stream_t;

typedef enum {
  PL_OK = 0,
  PL_ERR_ARG = 1,            /* NULL required pointer, negative size, bad eps/beta/mode bits */
  PL_ERR_DTYPE = 2,          /* dtype field not supported by this entry point */
  PL_ERR_ALIGN = 3,          /* a pitch the tensor-memory-access unit cannot address */
  PL_ERR_WORKSPACE = 4,      /* workspace NULL or smaller than the *_workspace_bytes() size */
  PL_ERR_ARCH = 5,           /* current device is not compute capability 10.0 (B200) */
  PL_ERR_CUDA = 6,           /* a CUDA runtime call or kernel launch failed */
  PL_ERR_DEVICE_TIMEOUT = 7, /* a bounded device-side wait ran out (reported by pl_device_status) */
  PL_ERR_BAD_TARGET = 8      /* a target id outside [0, V) (reported by pl_device_status) */
} pl_status;

/* ---- mode bit-field ----------------------------------------------------------
 * bits 0-1  reduction: PL_BNPO (global token mean) or PL_GRPO (per-sequence mean,
 *           then mean over the bs sequences, fully masked sequences counted).
 * bits 4-7  dtype of the log-probs (pl_loss) or of X/W/Xref/Wref/bias/dX/dW/dbias
 *           (pl_fused_linear_grpo): PL_F32, PL_F16 or PL_BF16.
 * bit 8     PL_ADV_LP_DTYPE: adv is in that dtype instead of fp32.
 * bit 9     PL_CLIP_TWO_SIDED: use -min(A*ratio, A*clipped) instead of the literal
 *           -A*min(ratio, clipped).  (The literal form makes eps_lo inert; the
 *           two-sided form is the standard PPO objective.)
 * bits 16-23 pl_fused_linear_grpo only: rows per chunk / 128; 0 selects 1024.
 */
#define PL_BNPO 0u
#define PL_GRPO 1u
#define PL_REDUCTION_MASK 0x3u
#define PL_F32 (0u << 4)
#define PL_F16 (1u << 4)
#define PL_BF16 (2u << 4)
#define PL_DTYPE_MASK (0xFu << 4)
#define PL_ADV_LP_DTYPE (1u << 8)
#define PL_CLIP_TWO_SIDED (1u << 9)
#define PL_CHUNK_SHIFT 16
#define PL_CHUNK_ROWS(n) ((uint32_t)(((n) / 128) & 0xFF) << PL_CHUNK_SHIFT)

/* ---- loss-only kernel ---------------------------------------------------------
 * pl_loss: fused forward + backward (grad_out != NULL) or forward-only
 * (grad_out == NULL) of the BNPO/GRPO loss above, as ONE kernel launch: the
 * valid-token counts (global for BNPO, per sequence for GRPO) are taken on the
 * device before any gradient is scaled -- in a first phase ordered by a bounded
 * grid barrier, or, for batches of up to 65536 tokens and 1024 sequences, by
 * every block counting the whole mask itself -- and the last block to finish
 * reduces the per-block partial sums in a fixed order (deterministic for a
 * given size).  No host synchronisation.
 *
 *   policy_lp, old_lp, ref_lp : [bs, seq] in the mode's dtype.  ref_lp may be NULL
 *                               only when beta == 0 (the KL branch is then compiled
 *                               out and ref_lp is never read).
 *   adv                       : [bs], fp32 (or the log-prob dtype with PL_ADV_LP_DTYPE).
 *   mask                      : [bs, seq] bytes (bool or int8); nonzero = valid.
 *   eps_lo, eps_hi, beta      : clip band [1-eps_lo, 1+eps_hi] (both >= 0), KL weight (>= 0).
 *   loss_out                  : device fp32 scalar.
 *   grad_out                  : [bs, seq] in the log-prob dtype = dLoss/dpolicy_lp, or NULL.
 * bs*seq == 0 writes loss 0.  Pointers that are not 16-byte aligned take a scalar
 * path; they never fail.
 * Scratch: pl_loss keeps one small zero-initialised buffer per (device, stream),
 * allocated on the first call on that pair, or ahead of time by pl_init (make
 * that first call, or pl_init, outside any stream capture).  Calls on one stream
 * are ordered; calls on different streams use different scratch.
 */
/* pl_init: creates, ahead of the first call, the library-owned scratch that
 * pl_loss (and pl_reverse_kl with a NULL workspace) use on the current device
 * and `stream`, sized for batches of up to max_bs sequences, so that later calls
 * allocate nothing and may be captured into a CUDA graph.  It synchronises
 * `stream` only when it has to grow an existing buffer.  max_bs < 0 is
 * PL_ERR_ARG; a device that is not compute capability 10.0 is PL_ERR_ARCH.
 */
pl_status pl_init(int64_t max_bs, pl_stream_t stream);

pl_status pl_loss(const void* policy_lp, const void* old_lp, const void* ref_lp,
                  const void* adv, const uint8_t* mask, int64_t bs, int64_t seq,
                  float eps_lo, float eps_hi, float beta, uint32_t mode,
                  float* loss_out, void* grad_out, pl_stream_t stream);

/* pl_loss with caller-owned scratch and optional count outputs.
 *   n_valid_out   : device int64 scalar, the global valid-token count, or NULL.
 *   row_valid_out : device int64 [bs], the per-sequence counts, or NULL.
 *   workspace     : device buffer of at least pl_loss_workspace_bytes(bs, seq) bytes,
 *                   256-byte aligned, zero-filled by the caller ONCE after allocation; the kernel
 *                   returns its counters to zero, so it stays reusable.  Calls that
 *                   share a workspace must be ordered on one stream.
 */
pl_status pl_loss_ex(const void* policy_lp, const void* old_lp, const void* ref_lp,
                     const void* adv, const uint8_t* mask, int64_t bs, int64_t seq,
                     float eps_lo, float eps_hi, float beta, uint32_t mode,
                     float* loss_out, void* grad_out, int64_t* n_valid_out,
                     int64_t* row_valid_out, void* workspace, size_t ws_bytes,
                     pl_stream_t stream);

size_t pl_loss_workspace_bytes(int64_t bs, int64_t seq);

/* pl_loss_static: pl_loss_ex for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it exists because some
 * callers must not call cudaMalloc on this path -- for example a process that
 * reserved all free device memory for its own pool at start-up, or code that
 * must not risk the device-wide synchronisation an allocation can cause -- and
 * pl_loss allocates its scratch on first use while pl_loss_ex needs a buffer.
 *
 * Here the kernel's scratch is a fixed 64.25 KB array inside libpl.so's device
 * image (held on every GPU that loads the library until the process exits), so
 * the call allocates nothing: no cudaMalloc, cudaFree or allocating library
 * routine.  Limits: bs <= 4096; a larger bs returns PL_ERR_WORKSPACE before
 * any launch.  All other arguments are those of pl_loss_ex.
 *   status_out : optional device uint32; receives this call's device error bits
 *                (0 = none, 1 = a bounded wait ran out) and clears them.  With
 *                NULL, the bits accumulate until a call passes status_out.
 * The first call on each device looks up the array's device address (with that
 * device current), so make it before any stream capture.  The address is cached
 * per device and context; after a cudaDeviceReset the next call looks it up
 * again (and should again come before any capture).  Every call shares the one
 * array and resets the counters it needs on `stream` before its kernel: calls
 * whose work overlaps on the GPU race, so order them on one stream.
 */
pl_status pl_loss_static(const void* policy_lp, const void* old_lp, const void* ref_lp,
                         const void* adv, const uint8_t* mask, int64_t bs, int64_t seq,
                         float eps_lo, float eps_hi, float beta, uint32_t mode,
                         float* loss_out, void* grad_out, int64_t* n_valid_out,
                         int64_t* row_valid_out, uint32_t* status_out, pl_stream_t stream);

/* ---- fused linear path ----------------------------------------------------------
 * pl_fused_linear_grpo: for the N = bs*T rows (sequence-major),
 *   z      = X W^T (+ bias),  logp = z[target] - logsumexp(z)        (policy)
 *   z_ref  = Xref Wref^T,     ref_logp likewise                        (reference, no bias)
 *   loss   = the BNPO/GRPO loss of pl_loss on (logp, old_lp, ref_logp)
 *   g      = dLoss/dlogp,  dz = g * (onehot(target) - softmax(z))
 *   dX = dz W,  dW = dz^T X,  dbias = sum over rows of dz.
 * Rows are processed in chunks (1024 by default, see the mode bits).  Per chunk a
 * persistent tcgen05 GEMM computes the reference and policy logits tile by tile;
 * its epilogue keeps a per-(row, 256-column tile) running max / sum of exponentials
 * and the target logit, and stores the policy logits into a bounded workspace of
 * chunk x V elements per slot (full-batch logits are never materialised; two
 * slots with several chunks, three with several bf16 chunks and a weight
 * gradient).  The logits are then turned into dz in place and a second
 * persistent GEMM computes dX and dW (with several chunks, chunk c's backward
 * GEMM shares a launch with chunk c+1's forward); dW and dbias are accumulated in
 * fp32 across chunks (the first contribution stores, later ones add, a last pass
 * converts to the model dtype; bf16 chunks 2i and 2i+1 make one dW contribution
 * whose K covers both chunks' rows).
 *
 *   X [N,H], W [V,H], bias [V] or NULL : model dtype (PL_F16 or PL_BF16).
 *   targets [N] int64                  : sampled token ids; a row whose id is outside
 *                                        [0, V) is treated as masked and raises
 *                                        PL_ERR_BAD_TARGET in pl_device_status.
 *   Xref [N,H], Wref [V,H]             : reference model inputs, model dtype; NULL
 *                                        allowed only when beta == 0 (the reference
 *                                        GEMM is then skipped).
 *   old_lp [N] fp32, adv [bs], mask [bs,T] bytes : as for pl_loss.
 *   H must be a multiple of 8 (16-byte row pitch); any V >= 1.
 *   loss                               : device fp32 scalar (required).
 *   dX [N,H], dW [V,H], dbias [V]      : model dtype, each NULL if not needed (its
 *                                        GEMM or reduction is skipped).
 *   logp_out, ref_logp_out [N] fp32    : optional per-token log-probs (the latter is
 *                                        written only when beta != 0).
 *   n_valid_out                        : optional device int64 scalar.
 *   workspace                          : at least pl_fused_linear_grpo_workspace_bytes()
 *                                        bytes, 256-byte aligned, zero-filled once after
 *                                        allocation; calls sharing it must be stream-ordered.
 */
pl_status pl_fused_linear_grpo(const void* X, const void* W, const void* bias,
                               const int64_t* targets, const void* Xref, const void* Wref,
                               const float* old_lp, const void* adv, const uint8_t* mask,
                               int64_t bs, int64_t T, int64_t H, int64_t V,
                               float eps_lo, float eps_hi, float beta, uint32_t mode,
                               float* loss, void* dX, void* dW, void* dbias,
                               float* logp_out, float* ref_logp_out, int64_t* n_valid_out,
                               void* workspace, size_t ws_bytes, pl_stream_t stream);

size_t pl_fused_linear_grpo_workspace_bytes(int64_t bs, int64_t T, int64_t H, int64_t V,
                                            uint32_t mode, int need_dW, int need_dbias);

/* pl_fused_linear_grpo_temp: pl_fused_linear_grpo at a sampling temperature
 * tau > 0 (finite); pl_fused_linear_grpo is this call with tau = 1.  The logits
 * of both models are z = (X W^T (+ bias)) / tau, so logp = log_softmax(z)[target];
 * the gradients returned are with respect to X, W and bias (the 1/tau of the
 * chain rule included).  ("Add SM100 CuTe DSL GRPO fast path", "Native scope",
 * names temperature 1.0 as that design's scope; other temperatures went to its
 * older path.)  Same workspace as pl_fused_linear_grpo.
 */
pl_status pl_fused_linear_grpo_temp(const void* X, const void* W, const void* bias,
                                    const int64_t* targets, const void* Xref, const void* Wref,
                                    const float* old_lp, const void* adv, const uint8_t* mask,
                                    int64_t bs, int64_t T, int64_t H, int64_t V,
                                    float eps_lo, float eps_hi, float beta, float temperature,
                                    uint32_t mode, float* loss, void* dX, void* dW, void* dbias,
                                    float* logp_out, float* ref_logp_out, int64_t* n_valid_out,
                                    void* workspace, size_t ws_bytes, pl_stream_t stream);

/* pl_fused_selective_logprob: the fused linear path without the loss step, the
 * shape of the "fused-linear selective-logprob autograd path" of "Add SM100 CuTe
 * DSL GRPO fast path" (Liger-Kernel PR #1363, "Summary"):
 *   forward  : logp_out[i] = log_softmax(X[i] W^T + bias)[targets[i]]   (fp32, [N])
 *   backward : with grad_logp[i] = dL/dlogp_i supplied (fp32, [N]),
 *              dz = grad_logp * (onehot(target) - softmax(z)),
 *              dX = dz W [N,H], dW = dz^T X [V,H], dbias = sum over rows of dz [V].
 * The same kernels as pl_fused_linear_grpo run: one tcgen05 GEMM per chunk of rows
 * with the logsumexp / target-logit epilogue, then (for the backward) the in-place
 * dlogits pass and the dX / dW GEMMs with fp32 dW accumulation across chunks.
 *   X [N,H], W [V,H], bias [V] or NULL : PL_F16 / PL_BF16 (mode bits 4-7; bits 16-23 chunk rows).
 *   targets [N] int64; an id outside [0, V) gives logp NaN, zero gradient and
 *   PL_ERR_BAD_TARGET in pl_device_status.
 *   grad_logp [N] fp32 or NULL; dX / dW / dbias (model dtype) require it.
 *   logp_out [N] fp32 or NULL (at least one output must be requested).
 *   workspace: pl_fused_selective_logprob_workspace_bytes() bytes, 256-byte aligned,
 *   zero-filled once after allocation.
 */
pl_status pl_fused_selective_logprob(const void* X, const void* W, const void* bias,
                                     const int64_t* targets, int64_t N, int64_t H, int64_t V,
                                     uint32_t mode, const float* grad_logp, float* logp_out,
                                     void* dX, void* dW, void* dbias, void* workspace,
                                     size_t ws_bytes, pl_stream_t stream);

size_t pl_fused_selective_logprob_workspace_bytes(int64_t N, int64_t H, int64_t V, uint32_t mode,
                                                  int need_dW, int need_dbias);

/* pl_reverse_kl: reverse-KL self-distillation ("Geometric-AI Kernels" model card,
 * section "Reverse KL"), forward and, when grad_out is not NULL, the gradient
 * with respect to the student logits, in one launch:
 *   p = softmax(student[r,:]), q = softmax(teacher[r,:]),
 *   kl_r = sum_v p_v (log p_v - log q_v),
 *   loss = sum_r [mask_r != 0] kl_r / max(n_valid, 1),
 *   grad[r,v] = [mask_r != 0] / max(n_valid, 1) * p_v (log p_v - log q_v - kl_r).
 * The card divides by n_valid unclamped (an all-masked batch gives inf/NaN);
 * here the denominator is max(n_valid, 1), so that batch gives loss 0 and a zero
 * gradient, and every other batch is unchanged.
 *   student, teacher [N, V] : one dtype, mode bits 4-7 (PL_F32 / PL_F16 / PL_BF16);
 *                             no other mode bit may be set.  Finite logits.
 *   mask [N] uint8/bool, nonzero = valid, or NULL (every row valid).
 *   loss_out : device fp32 scalar.      grad_out [N, V] student dtype, or NULL (forward only).
 *   kl_rows_out [N] fp32 or NULL : kl_r of each valid row, 0 for masked rows.
 *   n_valid_out : device int64 or NULL.
 *   workspace : pl_reverse_kl_workspace_bytes() bytes, 256-byte aligned and
 *               zero-filled once after allocation; NULL uses a library-owned one
 *               for (device, stream).  Calls sharing a workspace are stream-ordered.
 * Rows that are masked are not read.  Any element alignment is accepted; the
 * 16-byte vector path runs when student, teacher and grad share their address
 * modulo 16.  N = 0 writes loss 0 (student and teacher may then be NULL).
 * Errors: PL_ERR_ARG (NULL loss_out, NULL student/teacher with N > 0, N < 0, V < 1,
 * unknown mode bits), PL_ERR_DTYPE, PL_ERR_ALIGN (a pointer not aligned to its
 * element, or a workspace not 256-byte aligned), PL_ERR_WORKSPACE, PL_ERR_ARCH,
 * PL_ERR_CUDA; all are returned before any launch.
 */
pl_status pl_reverse_kl(const void* student, const void* teacher, const uint8_t* mask, int64_t N,
                        int64_t V, uint32_t mode, float* loss_out, void* grad_out,
                        float* kl_rows_out, int64_t* n_valid_out, void* workspace, size_t ws_bytes,
                        pl_stream_t stream);

size_t pl_reverse_kl_workspace_bytes(int64_t N, int64_t V);

/* pl_scale: x[i] *= *scale for n elements of the mode's dtype (bits 4-7), in place
 * on `stream`; `scale` is a device fp32 scalar, so the host never waits.  It
 * carries the chain rule for the autograd wrappers: the gradient of a scalar
 * loss times the loss's incoming gradient (the card's "Entry points" section:
 * the autograd-aware variant runs the same fused kernel).
 */
pl_status pl_scale(void* x, int64_t n, uint32_t mode, const float* scale, pl_stream_t stream);

/* pl_count_ratio: *factor_out = max(*local, 1) / max(*global_, 1) (fp32), all three
 * device scalars, computed on `stream` with no host synchronisation.
 * Data-parallel callers shard the sequences over ranks.  A rank's loss and
 * gradients come out of the fused call normalised by its own count: its
 * valid-token count n_l for BNPO, its sequence count bs_l for GRPO.  Times this
 * factor (with the all-reduced global count), they are the rank's exact share of
 * the global BNPO / GRPO loss of the "Geometric-AI Kernels" card ("BNPO Loss":
 * sum / max(n, 1); "GRPO Loss": mean over sequences), and summing the shares
 * over ranks gives the loss and dW / dbias of the whole batch.
 * Errors: PL_ERR_ARG (a NULL pointer), PL_ERR_ARCH, PL_ERR_CUDA.
 */
pl_status pl_count_ratio(const int64_t* local, const int64_t* global_, float* factor_out,
                         pl_stream_t stream);

/* ---- status ---------------------------------------------------------------------
 * pl_device_status: synchronises `stream`, reads the sticky device error flag of
 * `workspace` (NULL = pl_loss's own scratch for the current device and `stream`),
 * clears it and returns PL_OK, PL_ERR_DEVICE_TIMEOUT or PL_ERR_BAD_TARGET.
 */
pl_status pl_device_status(const void* workspace, pl_stream_t stream);

/* Static, human-readable name of a status code. */
const char* pl_status_string(pl_status status);

/* Library version as 10000*major + 100*minor + patch. */
int pl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PL_H_ */
