/*
 * mo.h - C ABI of the matrix-aware optimizer-step library (Muon, SOAP and
 * the Newton-Schulz orthogonaliser) for NVIDIA B200 (sm_100a).
 *
 * Conventions for every call below
 * --------------------------------
 *  - Matrices are fp32, row-major and contiguous (leading dimension == cols)
 *    and live in device memory of the context's GPU.  Base pointers must be
 *    4-byte aligned; 16-byte alignment with cols % 4 == 0 enables the
 *    vectorised path.
 *  - The caller owns every buffer: parameters, gradients, optimizer state and
 *    the workspace.  The library never allocates device memory; it owns only
 *    the host-side context.  The workspace is attached with
 *    mo_set_workspace() and must be at least mo_workspace_bytes(.., min) large.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are stream-ordered and asynchronous: they validate on
 *    the host, enqueue kernels and return without synchronising.
 *  - Parameters and state are updated in place; gradients are read only.  A
 *    matrix whose gradient pointer is NULL is skipped entirely (its state is
 *    not advanced), the "grad is None" rule of the LLM Optimizers guide,
 *    section 6.2.
 *  - Errors: invalid arguments are reported before any launch with a
 *    negative status and a message from mo_last_error().  Nothing falls back
 *    to the CPU: a call that cannot run on the GPU fails.
 *  - Non-finite values propagate (as in the published recurrences).  The
 *    optional `nonfinite` arrays receive, per matrix, 1 when the quantity
 *    named in the config is not finite and 0 otherwise, written on the
 *    device without a host synchronisation.
 *  - Kernels never wait without a bound: a wait that exceeds two seconds
 *    records a code in the context's device status word, read back with
 *    mo_device_status().
 *  - The step calls neither allocate nor synchronise, so with the workspace
 *    attached beforehand a sequence of them can be captured into a CUDA
 *    graph and replayed.  The library's kernels let their successors start
 *    their prologue early (programmatic stream serialization); kernels of
 *    the caller on the same stream are ordered as usual.
 *  - Environment: MO_GEMM_PAIR=1 runs tensor-core products with more than
 *    128 rows on pairs of CTAs (256-row tiles) instead of one CTA per
 *    128-row tile; the results are identical up to fp32 rounding of the
 *    accumulation order.
 *  - Each call makes the context's device current while it runs and puts
 *    the calling thread's current device back before it returns.
 *  - One context per host thread.
 */
#ifndef MO_H_
#define MO_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MO_API __attribute__((visibility("default")))
#else
#define MO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MO_OK = 0,
  MO_ERR_INVALID_ARG = -1,   /* null pointer, bad size or hyperparameter */
  MO_ERR_UNSUPPORTED = -2,   /* valid request the library does not support */
  MO_ERR_NO_WORKSPACE = -3,  /* no workspace attached, or too small */
  MO_ERR_CUDA = -4,          /* a CUDA runtime/driver call failed */
  MO_ERR_DEVICE = -5         /* the device status word reports a timeout */
} mo_status;

typedef struct mo_ctx mo_ctx;

/* Create a context bound to CUDA device `device`.  Host memory only. */
MO_API mo_status mo_ctx_create(mo_ctx** ctx, int device);
MO_API void mo_ctx_destroy(mo_ctx* ctx);

/* Last error message of this context (host string, valid until the next
 * call on the same context).  Never NULL. */
MO_API const char* mo_last_error(const mo_ctx* ctx);

/* Library version string. */
MO_API const char* mo_version(void);

/* ------------------------------------------------------------------ workspace
 * Workspace needed by `op` (0 = muon_step, 1 = soap_step, 2 =
 * ns_orthogonalize) for the n matrices of shapes rows[i] x cols[i] (host
 * arrays).  *full_bytes lets every group of equal-shape matrices run in one
 * batch; *min_bytes is the least that works (one matrix at a time).  Either
 * output pointer may be NULL. */
MO_API mo_status mo_workspace_bytes(mo_ctx* ctx, int op, const int64_t* rows, const int64_t* cols, int n,
                             size_t* min_bytes, size_t* full_bytes);

/* Attach caller-allocated device memory (256-byte aligned).  The library
 * keeps the pointer until the next call; the caller keeps ownership and must
 * not free it while work that uses it is in flight.  Attaching a different
 * buffer clears its header with a stream-ordered memset on `stream` and
 * copies the previous workspace's status word into it (a 4-byte device copy
 * on `stream`, which reads the old buffer: keep it alive until that copy has
 * run), so a timeout recorded before the switch is still reported.
 * dev_ptr == NULL with bytes == 0 detaches the workspace: its status word is
 * first read into the context (synchronising `stream`; skipped while
 * `stream` is capturing) and reported by the next mo_device_status; call
 * this before freeing a workspace that will not be replaced. */
MO_API mo_status mo_set_workspace(mo_ctx* ctx, void* dev_ptr, size_t bytes, void* stream);

/* Copy the device status word to *status (0 = no timeout recorded) and clear
 * it.  The word read is the attached workspace's, ORed with that of the
 * fixed scratch array of ns_orthogonalize_static on ctx's device once a
 * static call has set it up there; with neither, MO_ERR_NO_WORKSPACE.
 * Synchronises `stream`.  Returns MO_ERR_DEVICE when the word was set. */
MO_API mo_status mo_device_status(mo_ctx* ctx, void* stream, int32_t* status);

/* ------------------------------------------------------------------ profiling
 * With profiling enabled, every kernel the following calls launch is
 * bracketed by a CUDA event pair on its stream.  mo_profile_read()
 * synchronises those events and returns, per kernel kind k < nkinds (host
 * arrays), the summed elapsed milliseconds, the executed tensor-core flops
 * and the launch count, then forgets the records.  Kinds: 0 Muon momentum /
 * cast, 1 norm finalize, 2 Gram X X^T, 3 polynomial a I + b A + c A A,
 * 4 update P X, 5 apply / store, 6 SOAP elementwise, 7 SOAP rotations, 8 SOAP
 * power step and QR (other), 9 mo_gemm_bf16, 10 SOAP factor EMAs, 11 QR
 * diagonal Cholesky blocks, 12 QR row-block solves, 13 QR trailing updates,
 * 14 fused small-matrix Newton-Schulz / Muon. */
MO_API mo_status mo_profile_enable(mo_ctx* ctx, int enable);
MO_API mo_status mo_profile_read(mo_ctx* ctx, double* ms, double* flops, int64_t* launches, int nkinds);

/* ------------------------------------------------------------------ Muon
 * One Muon step per matrix ("Matrix optimizers: K-FAC, Shampoo and Muon",
 * section "Muon", steps 1-4; "LLM Optimizers: From SGD and AdamW to SOAP,
 * Muon, and Scalable Training", sections 11.3-11.5):
 *   B <- beta B + G            (momentum_ema: B <- beta B + (1 - beta) G)
 *   N  = G + beta B            (nesterov; else N = B)
 *   O  = NS(N): ns_steps quintic Newton-Schulz iterations on
 *        N / (||N||_F + eps), tall matrices transposed so that the Gram
 *        matrix is the smaller one; bf16 operands, fp32 accumulation, every
 *        stored iterate rounded to bf16 (nearest-even); the normalisation
 *        scale is applied in fp32 inside the first iteration
 *   W <- (1 - lr wd) W - lr s O,  s = 0.2 sqrt(max(m, n))  (adjust_lr 0)
 *                                 s = sqrt(max(1, m / n))   (adjust_lr 1)
 * Matrices of equal (oriented) shape are batched into grouped launches. */
typedef struct {
  int64_t rows, cols;   /* m, n */
  float* W;             /* parameter, updated in place */
  const float* G;       /* gradient; NULL skips this matrix */
  float* momentum;      /* momentum buffer B (zero before the first step) */
} mo_muon_mat;

typedef struct {
  float lr, weight_decay, momentum;  /* lr >= 0, wd >= 0, 0 <= momentum < 1 */
  int nesterov;                      /* 1: N = G + beta B (default); 0: N = B */
  int momentum_ema;                  /* 0: B = beta B + G (default); 1: EMA form */
  int ns_steps;                      /* 1..64 (5) */
  float a, b, c;                     /* (3.4445, -4.7750, 2.0315) */
  float eps;                         /* 1e-7 */
  int adjust_lr;                     /* 0: 0.2 sqrt(max(m,n)); 1: sqrt(max(1,m/n)) */
  int32_t* nonfinite;                /* optional device int32[n]: ||N||_F not finite */
} mo_muon_cfg;

MO_API mo_status muon_step(mo_ctx* ctx, const mo_muon_mat* mats /* host array */, int n,
                    const mo_muon_cfg* cfg, void* stream);

/* ------------------------------------------------------------------ Newton-Schulz
 * O_i = NS(in_i) for n matrices of possibly different shapes, with the same
 * iteration and rounding points as muon_step (section 11.4 of the LLM
 * Optimizers guide).  in/out/rows/cols are host arrays of device pointers
 * and sizes; out_i has in_i's shape and receives the bf16 iterate widened to
 * fp32.  in_i and out_i must not overlap. */
typedef struct {
  int ns_steps;         /* 1..64 */
  float a, b, c;
  float eps;
  int32_t* nonfinite;   /* optional device int32[n]: ||in_i||_F not finite */
} mo_ns_cfg;

MO_API mo_status ns_orthogonalize(mo_ctx* ctx, const float* const* in, float* const* out,
                           const int64_t* rows, const int64_t* cols, int n, const mo_ns_cfg* cfg,
                           void* stream);

/* ------------------------------------------------------------------ strided batches
 * The same calls for n matrices of one shape stored at a fixed stride (in
 * elements) from one base pointer, e.g. the per-head matrices of a model
 * held as one [n][rows][cols] tensor: the caller passes O(1) arguments
 * whatever n is.  Matrix i of `in` starts at in + i * in_stride, and
 * likewise for out, W, G and the momentum (one stride for the three).
 * Strides must be at least rows * cols when n > 1.  Everything else,
 * including validation, alignment rules and the nonfinite array (indexed by
 * i), is that of ns_orthogonalize and muon_step. */
MO_API mo_status ns_orthogonalize_strided(mo_ctx* ctx, const float* in, int64_t in_stride, float* out,
                                          int64_t out_stride, int64_t rows, int64_t cols, int n,
                                          const mo_ns_cfg* cfg, void* stream);
MO_API mo_status muon_step_strided(mo_ctx* ctx, float* W, const float* G, float* momentum, int64_t stride,
                                   int64_t rows, int64_t cols, int n, const mo_muon_cfg* cfg, void* stream);

/* ------------------------------------------------------------------ no-allocation variant
 * The pages have no counterpart to this entry point; it serves callers that
 * cannot allocate device memory when they call it: programs whose GPU
 * memory belongs to another allocator with nothing spare, runtimes that
 * forbid allocation after start-up, or plain C hosts with no allocator at
 * hand.  It computes the same mathematics as ns_orthogonalize for ONE matrix
 * (the batched-GEMM engine at every shape, so for m' <= 128 and n' <= 256,
 * where ns_orthogonalize uses its fused small-matrix kernel, the last bits
 * of the rounding may differ), but its scratch is a fixed device array of
 * MO_STATIC_SCRATCH_BYTES inside
 * the library (held by every GPU that loads the library until the process
 * exits) instead of an attached workspace; the caller passes only the input
 * and output.  It calls no allocator.
 *  - Shapes whose scratch exceeds the array (about m' x n' > 1024 x 2048
 *    with m' <= n') are rejected with MO_ERR_UNSUPPORTED and a message.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and caches it: make that first call before any
 *    stream capture.
 *  - All calls share the array and leave their contents behind; each call
 *    writes every scratch value before reading it.  Calls that overlap on
 *    the GPU (for example on unordered streams) race on it.
 *  - The array starts with a status word in which a kernel wait that gives
 *    up records its code; it is not cleared by later calls, and
 *    mo_device_status reads and clears it (no workspace needed).
 *  - ctx supplies the device (made current for the call; the caller's
 *    current device is restored before returning) and receives error
 *    messages. */
#define MO_STATIC_SCRATCH_BYTES (16u << 20)

MO_API mo_status ns_orthogonalize_static(mo_ctx* ctx, const float* in, float* out, int64_t rows,
                                         int64_t cols, const mo_ns_cfg* cfg, void* stream);

/* ------------------------------------------------------------------ SOAP
 * One SOAP step per matrix with a per-step eigenbasis refresh ("Reading
 * notes on SOAP, Muon, and Beyond", sections 1 and 4; "LLM Optimizers",
 * section 11.1; "初探优化器（一）", section 6.2), at step t >= 1:
 *   L <- bs L + (1 - bs) G G^T,   R <- bs R + (1 - bs) G^T G
 *   Q_L <- qr(L Q_L),             Q_R <- qr(R Q_R)
 *                                 (one power step + QR, the current gradient
 *                                  included; diag(R) > 0; fp32-accurate: every
 *                                  refresh product takes fp16 two-plane
 *                                  operands; CholeskyQR passes, plain or
 *                                  shifted per matrix, until the basis is
 *                                  orthonormal to 5e-5.  Where L Q is singular
 *                                  its QR is not unique and the basis is
 *                                  completed arbitrarily (a zero factor gives
 *                                  Q = I, as Householder QR does))
 *   M <- b1 M + (1 - b1) G        (original space)
 *   M' = Q_L^T M Q_R,  G' = Q_L^T G Q_R
 *   V <- b2 V + (1 - b2) G' * G'
 *   Dbar = (M' / (1 - b1^t)) / (sqrt(V / (1 - b2^t)) + eps)
 *   W <- (1 - lr wd) W - lr Q_L Dbar Q_R^T
 * A side with L == NULL (resp. R == NULL) uses the identity basis; Q_* then
 * must be NULL too.  Tensor-core products take bf16 operands with fp32
 * accumulation; L, R, Q_*, M, V stay fp32.  Initial state: L = R = M = V = 0,
 * Q = I. */
typedef struct {
  int64_t rows, cols;   /* m, n */
  float* W;
  const float* G;       /* NULL skips this matrix */
  float* M;             /* first moment, m x n */
  float* V;             /* second moment in the rotated basis, m x n */
  float* L;             /* m x m factor, or NULL (identity left basis) */
  float* QL;            /* m x m basis, or NULL */
  float* R;             /* n x n factor, or NULL (identity right basis) */
  float* QR;            /* n x n basis, or NULL */
} mo_soap_mat;

typedef struct {
  float lr, beta1, beta2, shampoo_beta, eps, weight_decay;
  int bias_correction;  /* 1: divide by 1 - beta^t (default) */
  int32_t* nonfinite;   /* optional device int32[n]: 1 when a basis refresh did
                           not reach an orthonormal basis (non-finite input,
                           or more than 16 CholeskyQR passes needed); that
                           matrix then keeps its previous basis */
  int skip_refresh;     /* 1: update L, R but keep Q_L, Q_R this step (the steps
                           between refreshes when the basis is refreshed only
                           every f steps); 0: refresh every step (default) */
  float damping;        /* 0 (default): the pages' power step qr(L Q).  In
                           (0, 1e-2]: an option that departs from the pages,
                           qr((L + d I) Q) with d = damping * trace(L) (1 when
                           the trace is 0), the damping of the Shampoo family
                           ("Matrix optimizers: K-FAC, Shampoo and Muon",
                           Shampoo); it changes the update */
} mo_soap_cfg;

MO_API mo_status soap_step(mo_ctx* ctx, const mo_soap_mat* mats /* host array */, int n,
                    const mo_soap_cfg* cfg, int64_t step, void* stream);

/* Exact workspace of soap_step for these matrices, sides as given (the
 * shape-only query mo_workspace_bytes(op = 1) assumes both sides are kept).
 * Only rows, cols, L and R are read; no pointer is dereferenced. */
MO_API mo_status mo_soap_workspace_bytes(mo_ctx* ctx, const mo_soap_mat* mats, int n, size_t* bytes);

/* ------------------------------------------------------------------ SOAP-Muon
 * SOAP preconditions the Muon momentum with the bases of the previous step,
 * Newton-Schulz orthogonalises the result and Muon's update applies it; the
 * factors then take the raw gradient and the bases are refreshed for the
 * next step ("初探优化器（一）：从SGD到SOAP-Muon", sections 7.1-7.2; the
 * section's formula was lost, these steps are the plainest reading of its
 * implementation notes).  At step t >= 1:
 *   B <- mu B + G,  N = G + mu B (nesterov) or B
 *   N' = Q_L^T N Q_R,  G' = Q_L^T G Q_R          (bases as passed in)
 *   V <- b2 V + (1 - b2) G' * G'
 *   P = Q_L [N' / (sqrt(V / (1 - b2^t)) + eps)] Q_R^T
 *   O = NS(P)   (quintic Newton-Schulz as in ns_orthogonalize; its Frobenius
 *                normalisation is the rescaling)
 *   W <- (1 - lr wd) W - lr s O   (s as in muon_step's adjust_lr)
 *   L <- bs L + (1 - bs) G G^T,  R likewise;  Q <- qr((F + d I) Q) as in
 *   soap_step (skipped with skip_refresh)
 * Sides, layout, alignment and shape rules are those of soap_step (rows and
 * cols multiples of 8, 16-byte aligned pointers, factor sides <= 16384).
 * Precision: rotations two-plane bf16, P fp32, NS bf16 operands as in
 * muon_step, the refresh fp32-accurate.  Initial state: B = V = L = R = 0,
 * Q = I.  nonfinite[i] is 1 if P was not finite or the QR met a
 * non-positive pivot. */
typedef struct {
  int64_t rows, cols;
  float* W;
  const float* G;       /* NULL skips this matrix */
  float* B;             /* Muon momentum, m x n */
  float* V;             /* second moment in the rotated basis, m x n */
  float* L;             /* m x m factor, or NULL (identity left basis) */
  float* QL;            /* m x m basis, or NULL */
  float* R;             /* n x n factor, or NULL (identity right basis) */
  float* QR;            /* n x n basis, or NULL */
} mo_soap_muon_mat;

typedef struct {
  float lr, weight_decay, momentum;
  int nesterov;
  float beta2;          /* V's beta */
  float shampoo_beta;   /* factor EMA (0.9 in the records the pages describe) */
  float eps;            /* Adam epsilon, outside the square root */
  int bias_correction;  /* 1: V / (1 - b2^t) */
  int ns_steps; float a, b, c, ns_eps;
  int adjust_lr;        /* 0: 0.2 sqrt(max(m, n)); 1: sqrt(max(1, m / n)) */
  float damping;        /* as in mo_soap_cfg: 0 = qr(L Q) (default), or the
                           damped option in (0, 1e-2] */
  int32_t* nonfinite;   /* optional device int32[n] */
  int skip_refresh;     /* 1: keep the bases (factors still update) */
} mo_soap_muon_cfg;

MO_API mo_status soap_muon_step(mo_ctx* ctx, const mo_soap_muon_mat* mats /* host array */, int n,
                                const mo_soap_muon_cfg* cfg, int64_t step, void* stream);

/* Exact workspace of soap_muon_step for these matrices (sides as given). */
MO_API mo_status mo_soap_muon_workspace_bytes(mo_ctx* ctx, const mo_soap_muon_mat* mats, int n,
                                              size_t* bytes);

/* ------------------------------------------------------------------ building block
 * The batched tensor-core GEMM the steps are built from, exposed for tests
 * and for callers composing their own variants:
 *   D_b = alpha s_b^alpha_pow (A_b B_b) + beta s_b^beta_pow C_b,  b < batch
 * A is M x K stored K-major ([M][K]) or, with a_mn, MN-major ([K][M]); B is
 * K x N stored K-major ([N][K]) or, with b_mn, MN-major ([K][N]).  A and B
 * are bf16 (uint16 storage) with row strides that are multiples of 8
 * elements and 16-byte aligned bases.  C and D are bf16 or fp32 (c_f32,
 * d_f32); C may be NULL or alias D.  With sym set the product must be
 * symmetric (M == N): only tiles that touch the upper triangle are computed
 * and each upper element is also written to its mirror position.  band sets
 * the order in which the persistent CTAs take tiles: 0 lets the library
 * choose (column order, or bands of row tiles when A overflows L2); n > 0
 * forces bands of n row tiles, each band taken column by column.  The order
 * changes no result.  band < 0 is MO_ERR_INVALID_ARG. */
typedef struct {
  const void* A; int64_t lda, strideA; int a_mn;
  const void* B; int64_t ldb, strideB; int b_mn;
  int M, N, K, batch, sym;
  float alpha, beta;
  const float* scale; int alpha_pow, beta_pow;   /* scale may be NULL */
  const void* C; int64_t ldc, strideC; int c_f32;
  void* D; int64_t ldd, strideD; int d_f32;
  int band;
} mo_gemm_desc;

MO_API mo_status mo_gemm_bf16(mo_ctx* ctx, const mo_gemm_desc* desc, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MO_H_ */
