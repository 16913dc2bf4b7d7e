/*
 * dyra_debug.h - diagnostics for include/dyra.h: read access to a plan's
 * intermediate buffers, so each stage of the forward can be checked on its own.
 * Not needed to run the layer.
 */
#ifndef DYRA_DEBUG_H_
#define DYRA_DEBUG_H_

#include <stddef.h>

#include "dyra.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Workspace buffers, valid after a forward on the same stream has completed.
 * Layouts for a DYRA_BF16 plan and a forward of B instances x T rows (N = B*T):
 *   DYRA_BUF_Z   N x r bf16     X V   ([DyRA] Alg. 1, Inference: first factor of the static part)
 *   DYRA_BUF_L   N x k bf16     X P (the correction's left factor), overwritten per instance by the
 *                solve with L_b (L_b^T L_b + lambda I)^-1
 *   DYRA_BUF_TG  B x k x k fp32 L_b^T L_b per instance (no ridge)
 *   DYRA_BUF_TP  (B*k) x d_in bf16   L_b^T X_b per instance
 *   DYRA_BUF_CT  d_out x (B*k) bf16  Q^T = W_res (L^T X)^T, so that the layer's
 *                correction L R^(1) is the solved L times Q
 * For a DYRA_F32 plan: Z holds N x (r+k) fp32 ([Z | L]), TG holds B x k x
 * (d_in + k) fp32 (columns [0, d_in) L_b^T X_b, then L_b^T L_b), TP the solved
 * (L^T L + lambda I)^-1 L^T X (fp32), and CT holds C = R^(1) as (B*k) x d_out fp32. */
enum {
  DYRA_BUF_Z = 0,
  DYRA_BUF_L = 1,
  DYRA_BUF_TG = 2,
  DYRA_BUF_TP = 3,
  DYRA_BUF_CT = 4
};

/* *ptr receives the device address of buffer `which` and *bytes its capacity
 * (0 and NULL if not allocated). Returns DYRA_OK or DYRA_ERR_INVALID_ARG. */
int dyra_debug_buffer(dyra_plan_t p, int which, const void **ptr, size_t *bytes);

/* Copy `bytes` bytes of buffer `which` to host memory `dst` (synchronous on
 * the plan's device). Returns DYRA_ERR_INVALID_ARG if the buffer is smaller. */
int dyra_debug_copy(dyra_plan_t p, int which, void *dst, size_t bytes);

/* Row splits S and rows per split used by the Gram stage for B x T. */
int dyra_debug_gram_split(dyra_plan_t p, int64_t B, int64_t T, int *splits, int *split_rows);

/* Stage timing. When enabled, every forward records a CUDA event on its stream
 * before each stage and after the last, which serialises the stages (no
 * programmatic overlap between them). Stages of the bf16 path:
 *   0 proj (X [V|P]), 1 gram (L^T [X|L]), 2 solve (L~ = L G^-1),
 *   3 rfactor (Q = T W_res^T), 4 out (Z U^T + L~ Q);
 * they are launched in the order 0 1 3 2 4 and reported in stage order.
 * Stages that did not run (k == 0) report 0. */
int dyra_debug_set_stage_timing(dyra_plan_t p, int enable);

/* Wait limit of one pipeline wait of a stage, in nanoseconds (0 restores the
 * default of 2 s). Every wait inside the tensor-core kernels gives up after
 * its limit: the kernel then raises DYRA_STATUS_WAIT_TIMEOUT, lets the copies
 * and MMAs it already issued finish, frees its tensor memory and returns, so
 * the context stays usable and the next forward is correct. A short limit
 * makes a wait run out on purpose, to test that path. Only stage 1 (gram), a
 * kernel whose every CTA drains its own copies, takes a limit; other stages
 * return DYRA_ERR_UNSUPPORTED. The output of a forward whose wait ran out is
 * not meaningful. */
int dyra_debug_set_wait_limit(dyra_plan_t p, int stage, uint64_t ns);

/* Milliseconds of each of the 5 stages of the last forward (synchronises on
 * its final event). Returns DYRA_ERR_INVALID_ARG if timing was not enabled. */
int dyra_debug_stage_times(dyra_plan_t p, float *ms5);

/* Kernel timelines. When enabled, each CTA of the four tensor-core stages of
 * a bf16 forward (proj, gram, rfactor, out) writes %globaltimer nanosecond
 * stamps at fixed milestones into a plan-owned buffer laid out as
 * [stage 0..4][CTA 0..255][slot 0..63] (uint64):
 *   0 entry, 1 set-up done, 2 inputs of the previous stage visible,
 *   3 first copy issued, 4 last copy issued, 5 first operands arrived,
 *   6 last accumulator committed, 7 first accumulator reached the epilogue,
 *   8 exit, 9 + i epilogue of the CTA's i-th tile done (i < 27),
 *   36 + i MMAs of the CTA's i-th tile committed (i < 20), 56 producer done,
 *   57 last MMA complete, 58 epilogue done, 60..62 split-K partial written,
 *   all partials arrived, slice reduced.
 * The solve stage (2) uses 0 entry, 2 inputs visible, 3 loaded, 4 factored
 * (G^-1 formed), 5 solved, 8 exit, and 40 + j the factorisation's phases.
 * Stamps are read with the timer register, which the assembler may read a
 * little before a preceding barrier.
 * A slot a CTA did not reach stays 0. Disabling frees the buffer. */
int dyra_debug_set_trace(dyra_plan_t p, int enable);
size_t dyra_debug_trace_bytes(void);
int dyra_debug_trace_copy(dyra_plan_t p, void *dst, size_t bytes);

#ifdef __cplusplus
}
#endif

#endif /* DYRA_DEBUG_H_ */
