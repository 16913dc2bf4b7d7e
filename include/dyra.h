/*
 * dyra.h - C ABI of the DyRA approximated linear layer on NVIDIA B200 (sm_100a).
 *
 * Method: "DyRA: Dynamic Residual Approximation for Efficient Matrix
 * Multiplication in DNNs" (Chae, Chung, Lee, Kim), cited as [DyRA].
 *
 * The layer approximates Y = X W^T (PyTorch layout, W is d_out x d_in) by
 *   Y = (X V) U^T + L C,                      [DyRA] Sec. 2.3 Eq. 6
 * where U (d_out x r) and V (d_in x r) are a static rank-r factorisation of W,
 * and L C is a rank-k correction of the residual output X W_res^T fitted to
 * the input with one ridge-regularised ALS step ([DyRA] Sec. 2.2 Eq. 4-5,
 * footnote 2; Appendix A, Algorithm 1, procedure Inference):
 *   L = X P                                    (P precomputed, Eq. 7)
 *   C = (L^T L + lambda I)^-1 (L^T X) W_res^T
 * The correction is fitted separately for each batch instance ([DyRA]
 * Sec. 2.4): X holds B consecutive instances of T rows each.
 *
 * Letters follow this library (static rank r, correction rank k); the paper
 * uses k for the static rank and r for the correction rank.
 *
 * Conventions for every call:
 *  - Matrices are dense, row-major, in the plan's storage type (float for
 *    DYRA_F32, bfloat16 bit patterns for DYRA_BF16). Accumulation is fp32.
 *  - Pointers to matrices are CUDA device pointers on the plan's device,
 *    aligned to 16 bytes. The caller owns them.
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and is asynchronous; no call below synchronises the device
 *    except dyra_last_status and dyra_plan_destroy.
 *  - A plan must not be used from two host threads or two streams at once.
 *  - No call throws; each returns DYRA_OK (0) or a negative DYRA_ERR_* code.
 */
#ifndef DYRA_H_
#define DYRA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *` */
typedef struct CUstream_st *dyra_stream_t;

typedef struct dyra_plan *dyra_plan_t;

typedef enum {
  DYRA_F32 = 0,  /* float storage; SIMT fp32 kernels (no TF32) */
  DYRA_BF16 = 1  /* bfloat16 storage; tcgen05 tensor-core kernels */
} dyra_dtype_t;

enum {
  DYRA_OK = 0,
  DYRA_ERR_INVALID_ARG = -1,    /* null pointer, non-positive or inconsistent size */
  DYRA_ERR_NOT_LOADED = -2,     /* forward before dyra_load_factors */
  DYRA_ERR_ALIGNMENT = -3,      /* pointer not 16-byte aligned, or a bf16 size not a multiple of 8 */
  DYRA_ERR_RANK_DEFICIENT = -4, /* lambda == 0 and T < k: L^T L is singular */
  DYRA_ERR_ALLOC = -5,          /* device allocation failed */
  DYRA_ERR_CUDA = -6,           /* a CUDA runtime/driver call failed */
  DYRA_ERR_UNSUPPORTED = -7,    /* device is not compute capability 10.0 (B200) */
  DYRA_ERR_DEVICE = -8          /* a kernel raised its status word (see dyra_last_status) */
};

/* Device status bits reported by dyra_last_status (OR-ed together). */
enum {
  DYRA_STATUS_NONPOSITIVE_PIVOT = 1, /* Cholesky of L^T L + lambda I met a pivot <= 0 or NaN;
                                        that instance's correction was set to zero */
  DYRA_STATUS_WAIT_TIMEOUT = 2,      /* a kernel's pipeline wait exceeded its time limit and the
                                        kernel returned early; outputs are undefined */
  DYRA_STATUS_BOUNDS = 4             /* bounds-checked build (libdyra_debug.so, compiled with
                                        DYRA_DEBUG) only: a kernel computed a global index outside
                                        its buffer and skipped that access; outputs are undefined */
};

/*
 * Create a plan for one layer shape.
 *   d_in, d_out : layer sizes (>= 1)
 *   r           : static rank, 1 <= r
 *   k           : correction rank, 0 <= k <= 128 (k == 0 gives the weight-only
 *                 layer (X V) U^T, [DyRA] Sec. 2.1)
 *   r + k <= min(d_in, d_out)   (both come from one SVD of W, Alg. 1 offline)
 *   DYRA_BF16 additionally needs d_in, d_out, r, k to be multiples of 8
 *   (16-byte rows for the tensor-memory-access unit), else DYRA_ERR_ALIGNMENT.
 * The plan binds to the current CUDA device. *out receives the handle; it is
 * left unchanged on error.
 */
int dyra_plan_create(dyra_plan_t *out, int d_in, int d_out, int r, int k, dyra_dtype_t dtype);

/*
 * A plan whose static part is a Monarch matrix ([DyRA] App. B) instead of the
 * rank-r factorisation, for a square layer of n = b1 * b2 features (the pages
 * define Monarch for square weights): dyra_plan_create_monarch_rect with
 * b1' = b1 and b2' = b2. Errors as there; DYRA_ERR_INVALID_ARG also when
 * n != b1 * b2.
 */
int dyra_plan_create_monarch(dyra_plan_t *out, int n, int b1, int b2, int k, dyra_dtype_t dtype);

/*
 * A Monarch plan for a rectangular layer, d_in = b1 * b2 and d_out = b1o * b2o
 * (the pages define Monarch for square weights only and also use it on
 * rectangular MLP layers; this is the library's reading of that). In the
 * paper's layout (Y = X W, W of shape d_in x d_out) the static product is
 * X W_hat with W_hat = P1 L P2^T R, L = diag(L_1 .. L_b2) of b1 x b1o blocks,
 * R = diag(R_1 .. R_b1o) of b2 x b2o blocks and P1, P2 the perfect shuffles of
 * the b1 x b2 and b1o x b2 grids:
 *   y[j1*b2o + i2] = sum over m1, j2 of x[m1*b2 + j2] L_j2[m1][j1] R_j1[j2][i2].
 * The correction (rank k, 0 <= k <= min(d_in, d_out), k <= 128) is unchanged.
 * bf16 plans run on the tensor cores (two block-diagonal GEMMs of the output
 * stage's kernel, each behind a shuffle of its input's columns, the second
 * taking the correction), fp32 plans on the CUDA cores. d_in, d_out and
 * b2 * b1o are at most 49152. Errors as dyra_plan_create; DYRA_ERR_ALIGNMENT
 * for bf16 unless d_in, d_out, k, b1 and b2 are multiples of 8.
 * dyra_forward_batched_noalloc returns DYRA_ERR_UNSUPPORTED for these plans,
 * and on the tensor cores dyra_set_als_steps accepts only 2.
 */
int dyra_plan_create_monarch_rect(dyra_plan_t *out, int b1, int b2, int b1o, int b2o, int k,
                                  dyra_dtype_t dtype);

/*
 * Load a Monarch plan's factors (the counterpart of dyra_load_factors):
 *   Lblocks : b2 blocks of b1 x b1o, row-major, one after the other (L_j2[m1][j1])
 *   Rblocks : b1o blocks of b2 x b2o, row-major, one after the other (R_j1[j2][i2])
 *             (b1o = b1 and b2o = b2 for dyra_plan_create_monarch)
 *   P, W_res, lambda : as in dyra_load_factors, with W_res = W - W_hat^T in this
 *                      library's d_out x d_in layout
 * Device pointers in the plan dtype, copied on `stream`. DYRA_ERR_INVALID_ARG
 * for a plan not made by dyra_plan_create_monarch(_rect) (and
 * dyra_load_factors rejects Monarch plans).
 */
int dyra_load_monarch(dyra_plan_t p, const void *Lblocks, const void *Rblocks, const void *P,
                      const void *W_res, float lambda, dyra_stream_t stream);

/*
 * Copy the offline factors into the plan ([DyRA] Alg. 1, Offline Preparation
 * outputs: the structured approximation, W_res and P_L).
 *   U      : d_out x r   (singular values folded in: W_hat = U V^T)
 *   V      : d_in x r
 *   P      : d_in x k    (ignored when k == 0; may be NULL then)
 *   W_res  : d_out x d_in, W - U V^T (ignored when k == 0; may be NULL then)
 *   lambda : ridge constant >= 0 added to L^T L (footnote 2 of Sec. 2.2)
 * The arrays are device pointers in the plan dtype; they are repacked into
 * plan-owned buffers on `stream`, so the caller may free them once the stream
 * has passed this call. May be called again to replace the factors.
 */
int dyra_load_factors(dyra_plan_t p, const void *U, const void *V, const void *P,
                      const void *W_res, float lambda, dyra_stream_t stream);

/*
 * The full linear layer of [DyRA] Sec. 2.4: every later forward computes
 * Y = (X V) U^T + b + alpha * (correction), the correction being the rank-k
 * term of Alg. 1. Before any call there is no bias and alpha = 1 (Alg. 1).
 *   bias  : device pointer to d_out values in the plan dtype, 16-byte aligned,
 *           copied into a plan-owned buffer on `stream` (the caller may free it
 *           once the stream has passed this call); NULL removes the bias.
 *   alpha : finite weight of the correction (0 leaves the static part and b).
 * dyra_forward_weight_only adds the bias too. Errors: DYRA_ERR_INVALID_ARG (NULL
 * plan, non-finite alpha), DYRA_ERR_ALIGNMENT, DYRA_ERR_ALLOC, DYRA_ERR_CUDA;
 * the plan is unchanged on error.
 */
int dyra_set_linear(dyra_plan_t p, const void *bias, float alpha, dyra_stream_t stream);

/*
 * Number of alternating least-squares updates per forward ([DyRA] Sec. 2.2,
 * Eq. 4-5; Sec. 3.3 compares 1, 1.5 and 2 iterations). Updates alternate L and
 * R from Alg. 1's first pair: half_steps = 2 is Alg. 1 (t = 1), 3 adds an L
 * update (t = 1.5: the output uses the newest L with the previous R), 4 an R
 * update (t = 2), and so on. Each L update after the first computes
 * L_b = X_b (R_b W_res)^T (R_b R_b^T + lambda I)^-1, so it costs one more pass
 * over X. Default 2.
 *   half_steps : 2 .. 64, else DYRA_ERR_INVALID_ARG.
 * Every kernel set runs any count. With more than two the bf16 tensor-core
 * forward forms each R update explicitly (the Gram sums kept in fp32 and the
 * small system solved from the left, then the rank-k GEMM) and each further
 * L update as X_b (R_b W_res)^T solved against R_b R_b^T + lambda I, one
 * stage after another without the compensated correction; the workspace then
 * holds B*k*(d_in + k) floats for the Gram sums. dyra_forward_batched_noalloc
 * returns DYRA_ERR_UNSUPPORTED for any count but 2. Takes effect at the next
 * forward.
 */
int dyra_set_als_steps(dyra_plan_t p, int half_steps);

/* Solvers of the per-instance k x k system of the correction. */
enum {
  DYRA_SOLVER_LDL = 0,           /* blocked LDL^T factorisation (the default) */
  DYRA_SOLVER_NEWTON_SCHULZ = 1  /* Newton-Schulz iteration for the inverse */
};

/*
 * Solver of the small ridge system (L_b^T L_b + lambda I) of the correction
 * ([DyRA] Sec. 2.4: a Cholesky solve for small correction ranks, a
 * Newton-Schulz iterative solver for larger ones).
 *   solver    : DYRA_SOLVER_LDL, or DYRA_SOLVER_NEWTON_SCHULZ: from
 *               X_0 = I / ||G||_inf the iteration X <- X (2 I - G X) runs until
 *               the largest entry of I - G X is below 1e-6, stops shrinking
 *               near fp32 rounding, or max_iters steps have run; an instance
 *               whose residual is not below 1e-2 then gets no correction and
 *               raises DYRA_STATUS_NONPOSITIVE_PIVOT.
 *   max_iters : 1 .. 200 (the iteration's limit; ignored by DYRA_SOLVER_LDL).
 * Newton-Schulz runs in fp32 on the CUDA cores, one block per instance, and
 * needs a bf16 tensor-core plan with 1 <= k <= 64 (else DYRA_ERR_UNSUPPORTED);
 * it is used by the one-step forward (dyra_set_als_steps(p, 2)). Errors:
 * DYRA_ERR_INVALID_ARG for a NULL plan or a value out of range. Takes effect at
 * the next forward.
 */
int dyra_set_solver(dyra_plan_t p, int solver, int max_iters);

/*
 * dyra_forward_batched on HOST buffers: X (B*T x d_in) and Y (B*T x d_out) in
 * host memory, ideally page-locked (cudaHostAlloc), since pageable memory
 * makes the copies synchronous. Whole instances move in chunks of at least
 * about 1 MiB of X, at most 16 chunks. On three streams the copy of chunk
 * c + 1 to the device, the forward of chunk c (on `stream`) and the copy of
 * chunk c - 1 back overlap; an instance's result does not depend on the
 * chunking. The call is asynchronous like cudaMemcpyAsync: work enqueued on
 * `stream` afterwards, and a synchronisation of `stream`, see Y complete. The
 * plan owns the device chunk buffers (grown on demand) and the copy streams.
 * Errors as dyra_forward_batched; X and Y must not overlap.
 */
int dyra_forward_batched_host(dyra_plan_t p, const void *X, void *Y, int64_t B, int64_t T,
                              dyra_stream_t stream);

/*
 * Y = DyRA(X) for one instance of N rows (B = 1, T = N).
 *   X : N x d_in input, Y : N x d_out output (overwritten), N >= 0.
 * N == 0 is a no-op. Returns DYRA_ERR_RANK_DEFICIENT if lambda == 0 and N < k.
 */
int dyra_forward(dyra_plan_t p, const void *X, void *Y, int64_t N, dyra_stream_t stream);

/*
 * Y = DyRA(X) with the correction fitted per instance: X and Y hold B
 * consecutive instances of T rows ([DyRA] Sec. 2.4). B*T == 0 is a no-op.
 * Returns DYRA_ERR_RANK_DEFICIENT if lambda == 0 and T < k.
 */
int dyra_forward_batched(dyra_plan_t p, const void *X, void *Y, int64_t B, int64_t T,
                         dyra_stream_t stream);

/*
 * Y = (X V) U^T, the weight-only approximation ([DyRA] Sec. 2.1, first term of
 * Eq. 2) with the plan's static factors, whatever the plan's k.
 */
int dyra_forward_weight_only(dyra_plan_t p, const void *X, void *Y, int64_t N,
                             dyra_stream_t stream);

/*
 * dyra_forward_batched without any device allocation. (No counterpart in the
 * paper: this is a deployment convenience of this library.)
 *
 * Who needs it: callers that must not call cudaMalloc while serving, e.g.
 * code that runs under a memory manager owning every byte of the device,
 * real-time loops where an allocation's implicit synchronisation or its
 * failure mid-run is not acceptable, or embedders that forbid the library
 * from allocating once set-up is over. Instead of the plan's workspace, this
 * call keeps the intermediates (X V, X P, G_b, L_b^T X_b, the factor records
 * and the rank-k factor) in one fixed array of DYRA_STATIC_SCRATCH_BYTES (16 MiB)
 * compiled into the library; every GPU that loads that part of the library
 * holds the array until the process exits.
 *   - Arguments, layouts and results are those of dyra_forward_batched; the
 *     plan (created and loaded beforehand) supplies the factors.
 *   - If the intermediates of B x T rows do not fit in the array the call
 *     returns DYRA_ERR_INVALID_ARG and enqueues nothing. For a bf16 plan they
 *     take about 2*B*T*(r+k) + 4*B*k*k + 2*B*k*(d_in+d_out) + 4*B*F bytes,
 *     each part rounded up to 256, where F = K*K + 5 with K = 32 for
 *     k <= 32, 64 for k <= 64 (F = 0 above), plus 2*B*T*k + 2*B*k*(d_in + d_out)
 *     when the compensated correction is on (a single instance of at most
 *     2048 rows, or DYRA_HILO=1).
 *   - The first call on a device looks the array's device address up
 *     (cudaGetSymbolAddress), and so does the first call after that device's
 *     context was destroyed and created again (the array then has a new
 *     address); make such a call before capturing a stream into a CUDA graph.
 *   - All calls share the one array and it keeps whatever the last call left
 *     there. Nothing in it has to start at zero: every stage overwrites what
 *     the next stage reads. Calls whose execution overlaps on the GPU (other
 *     streams, other host threads, other plans) race on the array and give
 *     wrong results; serialise them.
 */
int dyra_forward_batched_noalloc(dyra_plan_t p, const void *X, void *Y, int64_t B, int64_t T,
                                 dyra_stream_t stream);

#define DYRA_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * Grow the plan's workspace for up to B instances of T rows, so that later
 * forwards of that size allocate nothing (call it before capturing a CUDA
 * graph or timing). Forward calls grow the workspace themselves otherwise.
 */
int dyra_reserve(dyra_plan_t p, int64_t B, int64_t T);

/*
 * Synchronise the plan's device, then return and clear the device status
 * bits (DYRA_STATUS_*) raised since the last call, or a negative error code.
 */
int dyra_last_status(dyra_plan_t p);

/* Free the plan and its device buffers (synchronises the device). NULL is a no-op. */
int dyra_plan_destroy(dyra_plan_t p);

/* Static text for a DYRA_OK / DYRA_ERR_* code. */
const char *dyra_error_string(int code);

/* Bytes of device memory the plan currently owns (factors + workspace). */
size_t dyra_plan_device_bytes(dyra_plan_t p);

#ifdef __cplusplus
}
#endif

#endif /* DYRA_H_ */
