/*
 * muon_b200.h -- C ABI of the Muon optimizer step for NVIDIA B200 (sm_100a).
 *
 * What the library computes (sources are the pages the method is described on):
 *
 *  - Muon step, "Muon优化器" (Muon optimizer, linsight.cn/f25d614e.html), section
 *    "Muon 算法伪代码与 PyTorch 实现": for every 2-D weight W (rows = d_out, cols = d_in)
 *      M <- beta*M + G                       (heavy-ball momentum, fp32 buffer)
 *      U <- nesterov ? beta*M + G : M
 *      X0 <- bf16(U), X <- X0 / (||X0||_F + eps)            ("zeropower_via_newtonschulz")
 *      T times: A = X X^T, B = b A + c A A, X = a X + B X   (X^T X form when rows > cols)
 *      W <- (1 - lr*wd) W - lr * scale(rows, cols) * X      (decoupled weight decay)
 *    with per-iteration (a, b, c): the fixed schedule (3.4445, -4.7750, 2.0315) x 5 of the
 *    section "Newton-Schulz 迭代", or the hybrid 8 fast + 2 stabilising iterations of
 *    prism.simon-ai.net/article/8795 (DeepSeek V4 section); the scale is one of the four
 *    of the section "缩放因子" (Moonlight 0.2*sqrt(max), KellerJordan, muP, naive).
 *  - Stiefel variant, "Muon 在 Stiefel 流形上的精确闭式更新" (mlqm.cn/news/1339166):
 *      V = G - W sym(W^T G)                                  (§1.3 / §3.2 tangent projection)
 *      W <- (I + c A)^-1 (I - c A) W, A = V W^T - W V^T, c = lr/2   (§3.2 Cayley)
 *    evaluated in the rank-2k Woodbury form of §6.2 (a 2k x 2k solve plus n x k GEMMs).
 *
 * Conventions shared by every entry point:
 *  - All matrices are dense row-major.  Matrix pointers are DEVICE pointers (except the
 *    gradients of muon_step_batched_host_grad, which sit in pinned host memory); descriptor
 *    arrays, schedules and coefficient tables are HOST pointers read during the call only.
 *  - The caller owns every buffer, including the workspace; the library never allocates
 *    device memory.  The workspace holds the library's tables between calls: a call with
 *    the same arguments and workspace as the previous call on that workspace reuses them
 *    (it then issues kernel launches only).  Do not write to a workspace between calls.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every entry point is
 *    asynchronous on `stream` and never synchronises it, except
 *    muon_workspace_device_status(), which does.
 *  - Host-side argument checks run before any launch; on error nothing is launched and
 *    buffers are untouched.  Launch failures return MUON_ERR_CUDA (muon_last_error() then
 *    names the failing call).  Device-side conditions (a non-finite Frobenius norm, a zero
 *    or non-finite pivot in the Cayley solve, a kernel wait that ran out of time) are
 *    recorded in the workspace and read back by muon_workspace_device_status().
 *  - bf16 matrices handled on the tensor-core path need rows % 8 == 0, cols % 8 == 0 and
 *    16-byte aligned pointers (TMA and 128-bit accesses); fp32 mode has no shape limit
 *    beyond 16-byte aligned pointers.  Workspaces must be 256-byte aligned (they hold TMA
 *    tensor maps); torch and cudaMalloc allocations are.
 */
#ifndef MUON_B200_H
#define MUON_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MUON_OK = 0,
    MUON_ERR_INVALID_ARG = 1,          /* null pointer, count <= 0, bad enum, bad schedule   */
    MUON_ERR_UNSUPPORTED_SHAPE = 2,    /* rows/cols not a multiple of 8 on the bf16 path;
                                          n < k for Stiefel; a dimension above the limits */
    MUON_ERR_ALIGNMENT = 3,            /* a device pointer not 16-byte aligned            */
    MUON_ERR_WORKSPACE_TOO_SMALL = 4,  /* ws_bytes below the *_workspace_size() minimum    */
    MUON_ERR_CUDA = 5,                 /* a CUDA runtime/driver call failed               */
    MUON_ERR_NONFINITE = 6,            /* device status: a NaN/Inf Frobenius norm          */
    MUON_ERR_DEVICE_TIMEOUT = 7,       /* device status: a kernel wait gave up (bounded); the
                                          kernel drained its copies and MMAs in flight before
                                          it released its memory, so the context stays usable */
    MUON_ERR_DEVICE_UNDRAINED = 8      /* device status: a wait gave up AND copies or MMAs
                                          already in flight did not finish within the drain
                                          limit (100 ms) before the kernel released its shared
                                          and tensor memory.  Results are undefined and the
                                          CUDA context should not be trusted: end the process */
} muon_status;

typedef enum { MUON_BF16 = 0, MUON_F32 = 1 } muon_dtype;

/* Update scale for W in R^{d_out x d_in} (Muon optimizer page, section "缩放因子"). */
typedef enum {
    MUON_SCALE_MOONLIGHT = 0,   /* 0.2 * sqrt(max(d_out, d_in))  */
    MUON_SCALE_KJ = 1,          /* sqrt(max(1, d_out / d_in))    */
    MUON_SCALE_MUP = 2,         /* sqrt(d_out / d_in)            */
    MUON_SCALE_NAIVE = 3        /* 1                             */
} muon_scale_mode;

#define MUON_MAX_NS_ITERS 32

/* Newton-Schulz schedule.  Iteration t (0-based) uses a = coeffs[3t], b = coeffs[3t+1],
 * c = coeffs[3t+2].  The first n_split_iters iterations run in split-bf16 (every operand
 * and intermediate kept as a bf16 hi + lo pair, three tensor-core products per GEMM:
 * hi*hi + hi*lo + lo*hi); later ones in plain bf16.  fp32_mode = 1 skips the bf16 cast and
 * runs every product in fp32 FMA arithmetic (no TF32).  eps is added to the Frobenius norm
 * (the page uses 1e-7). */
typedef struct {
    int n_iters;              /* 0 .. MUON_MAX_NS_ITERS (0: X = X0 / (||X0|| + eps)) */
    const float* coeffs;      /* host, 3 * n_iters floats                                */
    int n_split_iters;        /* 0 .. n_iters; ignored when fp32_mode                     */
    int fp32_mode;            /* 0 or 1                                                  */
    float eps;                /* > 0                                                     */
} muon_ns_schedule;

/* One Muon matrix.  W is updated in place (w_dtype), M (fp32) is updated in place, G is
 * read (g_dtype).  O_out, if not NULL, receives the orthogonalised update X of Newton-
 * Schulz (before the shape scale) as rows x cols bf16 (fp32 in fp32 mode). */
typedef struct {
    void* W;
    const void* G;
    float* M;
    void* O_out;
    int rows;
    int cols;
    int w_dtype;              /* muon_dtype */
    int g_dtype;              /* muon_dtype */
} muon_matrix_desc;

typedef struct {
    float lr;
    float beta;               /* momentum coefficient (page default 0.95)                 */
    float weight_decay;       /* decoupled: W <- (1 - lr*wd) W before the step             */
    int nesterov;             /* 0: NS input is M; 1: beta*M + G                          */
    int scale_mode;           /* muon_scale_mode                                          */
    muon_ns_schedule ns;
} muon_hyper;

/* Bytes of workspace muon_step_batched needs for this set (0 if the arguments are
 * invalid).  The step runs the set in consecutive groups whose Newton-Schulz buffers share
 * one region of at most 5 GiB (one group if the whole set fits; a single larger matrix
 * forms its own group); this size covers that region.  A smaller workspace of at least
 * muon_step_workspace_min() is processed in smaller groups.  Grouping does not change any
 * result: every matrix goes through the same arithmetic. */
MUON_API size_t muon_step_workspace_size(const muon_matrix_desc* descs, int count, const muon_hyper* hp);
MUON_API size_t muon_step_workspace_min(const muon_matrix_desc* descs, int count, const muon_hyper* hp);

/* One full Muon step (momentum, bf16 cast, Frobenius pre-scale, Newton-Schulz, shape
 * scale, decoupled weight decay, update) for `count` matrices of any shapes.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, ALIGNMENT, WORKSPACE_TOO_SMALL, CUDA. */
MUON_API muon_status muon_step_batched(const muon_matrix_desc* descs, int count, const muon_hyper* hp,
                              void* workspace, size_t ws_bytes, void* stream);

/* The same step with every G in pinned (page-locked) host memory; W, M and O_out stay on
 * the device.  The set is cut, in descriptor order, into up to MUON_HOST_GRAD_CHUNKS
 * chunks whose gradient bytes grow by a factor of 1.5 from one to the next (the first, whose
 * copy nothing can hide, holds 2% of the bytes for 8 chunks; the staging slots hold the
 * largest, 35%).  The chunks' gradients are copied into two staging
 * slots of the workspace on a library-owned copy stream, one cudaMemcpyAsync per matrix,
 * while the previous chunk's step runs on `stream`, so the host-to-device transfer
 * overlaps the computation of earlier chunks.  Results equal those of muon_step_batched on
 * device copies of the gradients.  `stream` orders the whole call (the copy stream joins it
 * through events), so it can be captured in a CUDA graph.  The workspace's device status
 * word gathers the status of every chunk.  There is no counterpart of this entry point on
 * the source pages: it serves callers whose gradients arrive in host memory.
 * Errors: those of muon_step_batched; INVALID_ARG if a G is not page-locked host memory.
 * Query the workspace size with muon_step_host_grad_workspace_size (0 if invalid). */
#define MUON_HOST_GRAD_CHUNKS 8
MUON_API size_t muon_step_host_grad_workspace_size(const muon_matrix_desc* descs, int count, const muon_hyper* hp);
MUON_API muon_status muon_step_batched_host_grad(const muon_matrix_desc* descs, int count, const muon_hyper* hp,
                                                 void* workspace, size_t ws_bytes, void* stream);

/* Newton-Schulz orthogonalisation (Muon optimizer page, zeropower_via_newtonschulz) of a
 * contiguous batch of rows x cols matrices: X_out[i] ~ msign(X_in[i]).  X_in is read as
 * in_dtype; in bf16 mode an fp32 input is first rounded to bf16 (the page's cast).
 * X_out is written as out_dtype.  X_in and X_out may not overlap. */
MUON_API size_t ns_workspace_size(int batch, int rows, int cols, const muon_ns_schedule* sch);
MUON_API muon_status ns_orthogonalize(const void* X_in, int in_dtype, void* X_out, int out_dtype,
                             int batch, int rows, int cols, const muon_ns_schedule* sch,
                             void* workspace, size_t ws_bytes, void* stream);

/* Stiefel-manifold step for a contiguous batch of column-orthonormal W (n x k fp32,
 * n >= k): tangent projection of G (n x k fp32), then the Cayley retraction with
 * c = lr/2 in Woodbury form (§6.2), evaluated through (I + cA)^-1 (I - cA) = 2 (I + cA)^-1 - I
 * as W - 2 U C^-1 (c B W) with U = [V, W], B = [W^T; -V^T], C = I + c B U: the same map as the
 * page's b / y = B b steps with two n x k products fewer.  The direction's two products
 * (W^T G and W sym(.)) run on the tensor cores as three bf16 planes (fp32-exact operands,
 * fp32 accumulation); every product that enters the retraction runs in fp32 FMA arithmetic
 * (no TF32); the 2k x 2k system is solved by fp64 Gaussian elimination with partial
 * pivoting.
 * W is updated in place; G is read.  n < k returns MUON_ERR_UNSUPPORTED_SHAPE (transpose
 * the problem, as the page advises).  k <= 4096. */
MUON_API size_t stiefel_workspace_size(int batch, int n, int k);
MUON_API muon_status stiefel_cayley_step(float* W, const float* G, int batch, int n, int k, float lr,
                                void* workspace, size_t ws_bytes, void* stream);

/* Frobenius pre-scaling without a workspace: X_out[i] = X0[i] / (||X0[i]||_F + eps) for a
 * contiguous batch of rows x cols matrices, X0 = bf16(X_in) (fp32 X_in when fp32_mode = 1),
 * written as out_dtype; the same values ns_orthogonalize gives with zero iterations.  If
 * scale_out (device, batch floats) is not NULL it receives the per-matrix 1/(||X0|| + eps).
 * There is no counterpart of this entry point on the source pages: it exists for callers
 * that cannot allocate device memory when they call it -- code running under a framework
 * whose allocator owns all device memory and cannot hand out a workspace at that point,
 * or paths where a cudaMalloc is not allowed because it would synchronise the device.
 * It allocates nothing: its scratch (fp64 block sums and per-matrix scales, 528 KiB) is a
 * fixed array inside the library, which every GPU that loads the library holds until the
 * process exits.  The first call on each device looks up that array's device address
 * (with the device current) and caches it; make that first call before any stream
 * capture.  Every call shares the array and overwrites it; nothing in it needs to start
 * at zero (each slot is written before it is read within a call).  Calls that overlap on
 * the GPU (e.g. on two streams) race on the array and must be ordered by the caller.
 * Limits: batch <= MUON_STATIC_MAX_BATCH and batch * ceil(rows*cols / 8192) <=
 * MUON_STATIC_MAX_BLOCKS, else MUON_ERR_UNSUPPORTED_SHAPE.  Pointers need no alignment.
 * X_out may equal X_in when in_dtype == out_dtype (each element is read before it is
 * written, by the same thread); other overlaps are not allowed.
 * A non-finite input is not reported (there is no status word): a matrix with an infinite
 * element gets scale 0 and NaN at that element, one with a NaN gets a NaN scale and NaN
 * everywhere.  Callers that need the check pass scale_out and test it for 0 or NaN. */
#define MUON_STATIC_MAX_BLOCKS 65536
#define MUON_STATIC_MAX_BATCH 4096
MUON_API muon_status muon_frobenius_prescale_static(const void* X_in, int in_dtype, void* X_out, int out_dtype,
                                                    int batch, int rows, int cols, int fp32_mode, float eps,
                                                    float* scale_out, void* stream);

/* MuonCayley update ("Muon 在 Stiefel 流形上的精确闭式更新" page, §3.3 and §4.3) for a
 * contiguous batch of column-orthonormal W (n x k fp32, n >= k, row-major):
 *   M <- beta*M + (1 - beta)*G                       (EMA momentum, M fp32, in place)
 *   D = M - (column means of M over the n rows)      (center = 1; D = M when center = 0)
 *   W <- Cayley retraction of W along the tangent projection of D, c = lr/2
 * The centering follows the page's printed code (mean over dim 0, i.e. each column's mean);
 * the projection and retraction are those of stiefel_cayley_step.
 * A wide batch (n < k: W row-orthonormal) is updated as its transpose, as the page's §4.4
 * and §6.1 advise: W, G and M keep the caller's n x k layout, the library transposes W and
 * the momentum into the workspace, runs the step on the k x n transposes (so the centring
 * removes each row's mean of the caller's M) and writes W back transposed; M is updated in
 * place as above.  The workspace then also holds the two transposes.
 * Errors: INVALID_ARG for null pointers, batch or sizes <= 0, a non-finite lr or beta, or
 * center not in {0, 1}; UNSUPPORTED_SHAPE when min(n, k) > 4096; ALIGNMENT for W, G or M
 * not 16-byte aligned or a workspace not 256-byte aligned; WORKSPACE_TOO_SMALL below
 * muon_cayley_workspace_size (which returns 0 for unsupported arguments). */
MUON_API size_t muon_cayley_workspace_size(int batch, int n, int k);
MUON_API muon_status muon_cayley_step(float* W, const float* G, float* M, int batch, int n, int k, float lr,
                                      float beta, int center, void* workspace, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then reads the device-side status word of `workspace` into
 * *status_out and clears it: MUON_ERR_DEVICE_UNDRAINED if any kernel gave up a wait and
 * could not drain, else MUON_ERR_DEVICE_TIMEOUT if a wait gave up, else MUON_ERR_NONFINITE
 * if a norm or pivot was not finite, else MUON_OK. */
MUON_API muon_status muon_workspace_device_status(void* workspace, size_t ws_bytes, int* status_out,
                                         void* stream);

/* Per-kernel-kind device timing, for measurement.  While enabled, every launch is
 * bracketed by CUDA events on its stream (this adds a little host overhead).
 * muon_timing_read() synchronises the recorded events and returns, for `kind`, the summed
 * milliseconds, the launch count and the summed algorithmic work (FLOP for GEMM kinds,
 * bytes for elementwise kinds) since the last reset. */
typedef enum {
    MUON_KERNEL_MOMENTUM = 0,     /* momentum + bf16 cast + Frobenius partial sums        */
    MUON_KERNEL_SCALE = 1,        /* per-matrix 1 / (||X0|| + eps)                        */
    MUON_KERNEL_NS_GEMM = 2,      /* tcgen05 Gram / polynomial / apply (bf16, fp32 acc)   */
    MUON_KERNEL_UPDATE = 3,       /* scale + decoupled weight decay + update              */
    MUON_KERNEL_SIMT_GEMM = 4,    /* fp32 FMA GEMMs (fp32 NS mode, Stiefel)               */
    MUON_KERNEL_LU = 5,           /* 2k x 2k LU and triangular solves                     */
    MUON_KERNEL_MISC = 6,         /* casts, copies, block assembly, plane splits          */
    MUON_KERNEL_TC_F32 = 7,       /* tcgen05 fp32 products from three bf16 planes (Stiefel) */
    MUON_KERNEL_SIMT_GEMM_F64 = 8,  /* fp64 GEMMs (Stiefel LU updates and back substitution),
                                       on the fp64 tensor cores where the layout allows  */
    MUON_KERNEL_KINDS = 9
} muon_kernel_kind;
MUON_API muon_status muon_timing_enable(int enable);
MUON_API muon_status muon_timing_reset(void);
MUON_API muon_status muon_timing_read(int kind, double* ms, long long* launches, double* work);

MUON_API const char* muon_status_string(muon_status s);
/* Description of the last MUON_ERR_CUDA failure on the calling thread: the library call
 * that failed (a launch names its index and kernel kind) and the CUDA error name and text;
 * "" if none.  The string stays valid until the thread's next failing call. */
MUON_API const char* muon_last_error(void);

/* Self-test of the bounded device waits (failure detection): launches one CTA that waits,
 * through the pipeline's own wait routine, on an mbarrier that nothing completes.  The wait
 * gives up after its limit (4 s), the kernel records MUON_ERR_DEVICE_TIMEOUT in the
 * workspace status word and ends; read it with muon_workspace_device_status().  The
 * context stays usable.  No counterpart on the source pages.
 * Errors: INVALID_ARG (null workspace or ws_bytes < 256), ALIGNMENT (workspace not
 * 256-byte aligned), CUDA. */
MUON_API muon_status muon_selftest_wait_timeout(void* workspace, size_t ws_bytes, void* stream);
MUON_API const char* muon_build_info(void);

#ifdef __cplusplus
}
#endif
#endif /* MUON_B200_H */
