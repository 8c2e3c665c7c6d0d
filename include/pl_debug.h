/*
 * pl_debug.h -- test hooks of libpl.so (not part of the loss path).
 *
 * pl_debug_gemm runs one plain GEMM through the same persistent tcgen05 kernel
 * the fused path uses, so the tensor-core mainloop can be checked in isolation:
 *
 *   D[m, n] = sum_k A(m, k) * B(n, k)            (fp32, row-major [M, N])
 *   A(m, k) = a_mn ? A[k*lda + m] : A[m*lda + k]   (K-major or MN-major)
 *   B(n, k) = b_mn ? B[k*ldb + n] : B[n*ldb + k]
 *
 * A, B: device, 16-bit (mode PL_F16 or PL_BF16), 16-byte aligned, lda/ldb
 * multiples of 8.  D: device fp32.  Enqueued on `stream`; a bounded wait that
 * runs out is reported by pl_device_status(NULL, stream).
 * Returns PL_ERR_ARG / PL_ERR_DTYPE / PL_ERR_ALIGN before any launch on bad input.
 */
#ifndef PL_DEBUG_H_
#define PL_DEBUG_H_

#include "pl.h"

#ifdef __cplusplus
extern "C" {
#endif

pl_status pl_debug_gemm(const void* A, int a_mn, int64_t lda, const void* B, int b_mn, int64_t ldb,
                        float* D, int64_t M, int64_t N, int64_t K, uint32_t mode, pl_stream_t stream);

/*
 * The same GEMM written to D[m*ldd + n] (ldd >= N) through one of the
 * epilogue's three fp32 output paths:
 *   out_path 0: per-thread row stores from registers      D  = A.B
 *   out_path 1: staged in shared memory, TMA tile store   D  = A.B
 *   out_path 2: staged in shared memory, TMA add          D += A.B
 * Paths 1 and 2 need D 16-byte aligned and N and ldd multiples of 4 (else
 * PL_ERR_ALIGN); no path writes D[m*ldd + n] for n >= N or m >= M.  Path 2 is what accumulates dW across the fused
 * path's row chunks.  PL_ERR_ARG for another out_path.
 */
pl_status pl_debug_gemm_out(const void* A, int a_mn, int64_t lda, const void* B, int b_mn, int64_t ldb,
                            float* D, int64_t ldd, int out_path, int64_t M, int64_t N, int64_t K,
                            uint32_t mode, pl_stream_t stream);

/*
 * Kernel timing for the benchmark.  While enabled, every kernel the library
 * launches is bracketed by a pair of CUDA events recorded on the launching
 * stream.  pl_debug_timing_read() waits for the recorded events, returns per
 * kind the summed device milliseconds and launch counts, and clears them.
 * Kinds: 0 = GEMM (tcgen05 kernel), 1 = loss-only kernels (cooperative and
 * small-batch), 2 = every other kernel (the fused path's counts, combine,
 * dlogits, convert and finalize; reverse KL; scale and count ratio).  Arrays
 * have 3 entries.
 * Not thread-safe; meant for one benchmarking thread.
 */
void pl_debug_timing(int enable);
pl_status pl_debug_timing_read(double* ms, int64_t* launches);

/*
 * Failure-detection test knobs, applied to later launches on this process.
 *   wait_ns        : bound on every device-side wait (0 restores the default, 2 s).
 *   extra_arrivals : the loss kernel's grid barrier waits for this many arrivals
 *                    beyond the blocks that exist, so it runs out after wait_ns.
 *   extra_tx       : each GEMM pipeline stage expects this many bytes beyond its
 *                    TMA loads, so its wait runs out after wait_ns.
 * A wait that runs out raises PL_ERR_DEVICE_TIMEOUT (pl_device_status); the
 * kernel then releases tensor memory and returns, and the context stays usable.
 * Pass (0, 0, 0) to restore normal operation.
 */
void pl_debug_set_wait(unsigned long long wait_ns, unsigned extra_arrivals, unsigned extra_tx);

/*
 * Chooses the loss-only kernel for later calls on this process: 1 = the
 * small-batch kernel (no grid barrier; every block counts the whole mask),
 * used when bs * seq <= 65536 and bs <= 1024, else the cooperative kernel;
 * 2 = always the cooperative kernel; 0 restores the default (1).  A
 * pl_debug_set_wait with extra arrivals also selects the cooperative kernel,
 * whose grid barrier it targets.  Returns PL_ERR_ARG for any other value.
 */
int pl_debug_set_loss_path(int path);

/*
 * Forces the reverse-KL kernel's cluster size (CTAs sharing one row: 1, 2, 4 or
 * 8) for later calls on this process, so tests reach every row split; 0
 * restores the host's choice.  Returns PL_ERR_ARG for any other value.
 */
int pl_debug_set_rkl_cluster(int cl);

/*
 * Chooses the reverse-KL kernel for later calls with a gradient on this
 * process: 1 = the streaming kernel (pass 2 re-reads each slice from L2);
 * 2 = the register-resident kernel (each slice read from HBM once) wherever it
 * applies -- 16-bit logits, V a multiple of 8, 16-byte aligned student,
 * teacher and gradient, and a row slice that fits its shared-memory slots --
 * and the streaming kernel otherwise; 0 restores the default (the streaming
 * kernel, measured faster).  Returns PL_ERR_ARG for another value.
 */
int pl_debug_set_rkl_path(int path);

/*
 * Forces the GEMM's pair tile for later launches on this process: 1 = 256 x 256
 * (one N=256 MMA per K step, double-buffered accumulators), 2 = 256 x 512 (two
 * MMAs sharing the A stage); 0 restores the host's choice (256 x 512 when every
 * problem of the launch is at least 512 wide).  Returns PL_ERR_ARG otherwise.
 */
int pl_debug_set_gemm_tile(int nh);

/*
 * The GEMM launcher's tile-width choice (host logic, no device call): for
 * njobs = 1 or 2 problems given as mnk = {M0, N0, K0[, M1, N1, K1]} on `pairs`
 * CTA pairs, returns 1 (256-wide tiles) or 2 (512-wide), or -1 on bad input.
 * The fused path's forward launch is {N, V, H} for the policy and reference;
 * its backward launch is {N, H, V} (dX) and {V, H, N} (dW).
 */
int pl_debug_pick_tile(int njobs, const int64_t* mnk, int pairs);

/*
 * The persistent GEMM's tile schedule, for a host-side check: two problems of
 * t0 tiles (c0 k-steps each) and t1 tiles (c1 k-steps each) over `pairs` CTA
 * pairs.  out_pair[t] (t0 + t1 entries) receives the pair that runs tile t.
 * The schedule balances per-pair loads counting each tile as its k-steps plus
 * a fixed hand-off cost of 8 k-steps.
 * Returns 0, or -1 when some tile would run on no pair or on two.
 */
int pl_debug_pair_tiles(int t0, int t1, int c0, int c1, int pairs, int32_t* out_pair);

/*
 * The backward launch's K-split choice (host logic, no device call): for the two
 * problems mnk = {M0, N0, K0, M1, N1, K1} (dX, then dW) on `pairs` CTA pairs,
 * returns 2 when the dX problem is computed in two K halves (each half's tiles
 * add their fp32 results into a zeroed buffer, which is then rounded to the
 * model dtype), else 1, or -1 on bad input; *nh_out (if not NULL) receives the
 * tile width that goes with it (1: 256 wide, 2: 512 wide).
 */
int pl_debug_pick_split(const int64_t* mnk, int pairs, int* nh_out);

/*
 * Forces the K split of the fused path's backward dX problem for later calls on
 * this process: 1 = never, 2 = always (when its K has at least two 64-wide
 * steps); 0 restores the host's choice.  Returns PL_ERR_ARG for another value.
 */
int pl_debug_set_gemm_split(int mode);

/*
 * Fused path with several row chunks: 0 (the default) = chunk c's backward GEMM
 * and chunk c+1's forward GEMM share one launch, whose CTA pairs claim tiles from
 * a queue (dX tiles first, then the forward tiles interleaved with the dW
 * tiles), with 8 epilogue warps; 1 = separate launches; 2 = shared launches with
 * 4 epilogue warps.  Applies to later calls on this process.  Returns
 * PL_ERR_ARG for another value.
 */
int pl_debug_set_gemm_merge(int mode);

/*
 * 512-wide GEMM launches on the round-robin schedule (the forward launches):
 * 0 (the default) = when the last partial wave holds R <= pairs / 2 tiles, those
 * tiles run as 2R tiles 256 wide, so the wave ends after half a tile's time;
 * 1 = never.  pl_debug_tail_halves returns R for `tiles` equal tiles on `pairs`
 * pairs (0: no split).  Returns PL_ERR_ARG for another mode.
 */
int pl_debug_set_gemm_tail(int mode);
int pl_debug_tail_halves(int tiles, int pairs);

/*
 * Fused path with several row chunks, how dW is finished: 1 = the last chunk
 * adds into the fp32 accumulator like the others and a separate kernel rounds
 * it; 2 = the last chunk's dW epilogue adds the fp32 accumulator of the earlier
 * chunks and stores the model dtype; 0 restores the default (1, measured
 * faster).  Applies to later calls on this process.  Returns PL_ERR_ARG for
 * another value.
 */
int pl_debug_set_dw_finish(int mode);

/*
 * Fused path with several bf16 row chunks run in shared launches, how many
 * rows one dW contribution covers: 1 = each chunk's dW contribution is its own
 * GEMM job (K = the chunk's rows); 2 = chunks 2i and 2i+1 contribute through one
 * job whose K runs over both chunks' rows (the earlier chunk's dlogits wait one
 * launch in the workspace, which then holds three chunks' logits); 0 restores
 * the default (2).  The dlogits of a pair then share the scale 2^0, so one
 * epilogue scale undoes both.  Applies to later calls on this process (the
 * workspace size of pl_fused_linear_grpo_workspace_bytes allows for either).
 * Returns PL_ERR_ARG for another value.
 */
int pl_debug_set_dw_pair(int mode);

/*
 * The GEMM's dynamic tile-queue order (host logic): jobs of tiles[0..njobs)
 * tiles, numbered in job order; queue entry q runs tile out[q].  The tiles of
 * jobs [0, q_f0) come first in order, then those of jobs [q_f0, q_w) spread
 * evenly between those of job q_w (q_w < 0: every tile in order).  Returns 0,
 * or -1 on bad input.
 */
int pl_debug_queue_tiles(int njobs, const int32_t* tiles, int q_f0, int q_w, int32_t* out);

/* Number of kernels this library has launched in this process. */
int64_t pl_debug_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* PL_DEBUG_H_ */
