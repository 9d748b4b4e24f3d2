/*
 * mao.h — C ABI of libmao: one optimizer step of the matrix-aware optimizers
 * Muon (with the optional Muon+ normalisation), two-sided SOAP with a per-step
 * power-iteration/QR eigenbasis refresh, and one-sided factored FOAM, applied
 * to a batch of weight matrices on one B200 GPU (sm_100a).
 *
 * Sources of the operations (page title, section):
 *   "SOAP, Muon and Beyond" review: 1-1 Problem definition (Shampoo factors
 *     L = b2 L + (1-b2) G G^T, R = b2 R + (1-b2) G^T G), 2-1 Main contribution
 *     (Muon approximates the polar factor U V^T by Newton-Schulz), 3-2 Module
 *     breakdown (Muon recipe epsilon 1e-7; SOAP rotation Q_L^T M Q_R, Adam in the
 *     eigenbasis, rotation back; real-time eigenbasis update: factors first,
 *     then refresh, then QR, then preconditioning).
 *   "SOAP, Muon, and Beyond" summary: eq. (1) u = Q_L Adam(Q_L^T m Q_R) Q_R^T.
 *   "Factored One-sided Adam-Moment for Practical and Scalable SOAP" review:
 *     1 Key Terms (input-only rotation G Q_R; row/column mean EMAs r, c; trace
 *     normalisation tau = tr(R)/(|r|_1 |c|_1)), 3 Method (adaptive refresh with
 *     pf = 10, tol = 0.1; bias-corrected Adam step in the rotated space).
 *   "Muon+: Towards Better Muon via One Additional Normalization Step":
 *     2 Methodology (M = mu M + (1-mu) G; O = Norm^(d)(Ortho(M));
 *     W = W - lr sqrt(m/n) O; d = row, column, Col-Row, Row-Col).
 *
 * Conventions for every call:
 *   - A matrix is row-major m x n (m rows, n columns), leading dimension n,
 *     rows contiguous.  Every device pointer is 16-byte aligned, and
 *     n * sizeof(element) is a multiple of 16 (n % 4 == 0 for fp32 buffers,
 *     n % 8 == 0 when G is bf16), so rows stay 16-byte aligned.
 *   - The caller owns every buffer: W, G, the optimizer state, the workspace
 *     and the optional stats.  The library never allocates device memory and
 *     never synchronises the stream inside a step.  Descriptor arrays and
 *     parameter structs are host memory, read only during the call.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) of the current device.  State updates happen in place in stream
 *     order.  G is read-only.  No two buffers may alias.
 *   - Errors: arguments, shapes, dtypes, alignment and workspace size are
 *     validated before anything is enqueued; on failure nothing is modified and
 *     the status says why.  A failed launch returns MAO_ERR_CUDA.  Conditions
 *     found on the device never trap: a bounded wait that gave up, and (when
 *     stats are requested) a non-finite weight written by the step, are recorded
 *     in a status word at the start of the workspace, which mao_workspace_status()
 *     reads.  A non-finite gradient propagates: the step writes non-finite
 *     weights and states, and the caller restores them from its own copy.
 *   - Initial state is the caller's job: L = R = 1e-6 I, Q = I,
 *     M = V = r = c = 0, t = 1 for the first step.
 */
#ifndef MAO_H_
#define MAO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MAO_VERSION 4

#if defined(__GNUC__)
#define MAO_API __attribute__((visibility("default")))
#else
#define MAO_API
#endif

/* cudaStream_t without including the CUDA headers. */
typedef struct CUstream_st* mao_stream_t;

typedef enum {
  MAO_OK = 0,
  MAO_ERR_INVALID_ARG = 1, /* NULL pointer, count < 0, bad enum or parameter value */
  MAO_ERR_SHAPE = 2,       /* m or n < 1, or a row length that breaks 16-byte rows */
  MAO_ERR_DTYPE = 3,       /* g_dtype not MAO_F32 / MAO_BF16 */
  MAO_ERR_ALIGN = 4,       /* a device pointer not 16-byte aligned */
  MAO_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than the *_workspace_size() answer */
  MAO_ERR_CUDA = 6,        /* a CUDA runtime call or kernel launch failed */
  MAO_ERR_NONFINITE = 7,   /* device status only: the step wrote a non-finite weight (stats requested) */
  MAO_ERR_TIMEOUT = 8,     /* a bounded device-side wait gave up (a defect, never expected) */
  MAO_ERR_UNSUPPORTED = 9, /* a valid request this build does not implement (e.g. no sm_100 device) */
  MAO_ERR_NOT_INITIALIZED = 10 /* a call that needs one-time set-up ran before it */
} mao_status;

typedef enum { MAO_F32 = 0, MAO_BF16 = 1 } mao_dtype;

/* Muon+ normalisation direction applied after orthogonalisation. */
typedef enum {
  MAO_NORM_NONE = 0,
  MAO_NORM_ROW = 1,     /* O_ij / (||O_i,:||_2 + 1e-7) */
  MAO_NORM_COL = 2,     /* O_ij / (||O_:,j||_2 + 1e-7) */
  MAO_NORM_COL_ROW = 3, /* column normalisation, then row normalisation */
  MAO_NORM_ROW_COL = 4  /* row normalisation, then column normalisation */
} mao_norm_mode;

typedef enum {
  MAO_REFRESH_EVERY_K = 0, /* refresh iff (t-1) % k == 0; k = 1 refreshes every step */
  MAO_REFRESH_ADAPTIVE = 1,/* on steps with (t-1) % pf == 0: D = Q^T F Q, refresh iff
                              ||offdiag D||_F / ||D||_F > tol */
  MAO_REFRESH_NEVER = 2
} mao_refresh_kind;

typedef struct {
  int32_t kind; /* mao_refresh_kind */
  int32_t k;    /* EVERY_K period (>= 1) */
  int32_t pf;   /* ADAPTIVE check period (>= 1) */
  float tol;    /* ADAPTIVE threshold on the off-diagonal ratio */
  int32_t sort; /* 1: before the power step, order the basis by diag(Q^T F Q) descending
                   (stable) and permute the moment state with it; 0: keep the order */
  int32_t lag;  /* 0: the current gradient enters the factors before the refresh (the
                   real-time order of "SOAP, Muon and Beyond" review 3-2 (4));
                   1: the refresh runs on the factors as they were before this step's
                   gradient entered them, the order of the standard implementation
                   that the summary's "SOAP Instability Diagnosis" names as a cause of
                   the slingshot instability (kept to reproduce the stale basis) */
} mao_refresh;

/* Optional per-matrix diagnostics, written on the device (array of `count`). */
typedef struct {
  float update_rms;    /* ||W_new - W_old||_F / sqrt(m n) */
  float offdiag_ratio; /* FOAM/SOAP adaptive check ratio of this step, -1 if none ran */
  int32_t refreshed;   /* bit 0: right basis refreshed, bit 1: left basis refreshed */
  int32_t nonfinite;   /* number of non-finite entries in W_new (also recorded in the status word) */
} mao_stats;

/* ------------------------------------------------------------------ Muon */

typedef struct {
  int32_t m, n;    /* rows, columns */
  float* W;        /* device fp32 m x n, updated in place */
  const void* G;   /* device m x n gradient, fp32 or bf16 (g_dtype) */
  int32_t g_dtype; /* mao_dtype */
  float* M;        /* device fp32 m x n momentum, updated in place */
  int32_t split_rows, split_cols; /* 0 or 1: one matrix.  Otherwise the stored matrix
                   holds split_rows x split_cols logical matrices of (m / split_rows) x
                   (n / split_cols), each stepped as a matrix of its own (a fused QKV
                   projection stored as [q | k | v] is split_cols = 3): its own
                   pre-normalisation, orthogonalisation, Muon+ norms and
                   sqrt(m_b / n_b) scale ("SOAP, Muon and Beyond" review 3-2 (2),
                   4-4 (2)).  Each block width keeps the row rule above (n / split_cols
                   a multiple of 4, of 8 for a bf16 G), else MAO_ERR_SHAPE */
} mao_muon_mat;

typedef enum {
  MAO_POLAR_NS = 0,    /* Newton-Schulz with the given coefficients, bf16 operands */
  MAO_POLAR_EXACT = 1  /* MOP ("SOAP, Muon, and Beyond" summary, "Muon vs SOAP Comparison"):
                          the polar factor U V^T of each (logical) matrix to fp32 accuracy.
                          ns_steps and ns_coef are ignored: the library runs 16 Newton-Schulz
                          iterations in fp32-faithful arithmetic (three bf16 planes per fp32
                          operand), 11 with (3.4445, -4.7750, 2.0315) that lift every singular
                          value at least ~2e-7 ||M||_F into [0.23, 1.21], then 5 of
                          (15/8, -10/8, 3/8), which converge cubically to 1.  Singular values
                          below ~2e-7 ||M||_F are not resolved (they are fp32 noise there). */
} mao_polar;

typedef struct {
  float mu;             /* momentum EMA coefficient */
  float lr;             /* learning rate eta */
  float wd;             /* decoupled weight decay: W <- W (1 - lr wd) - ... */
  float eps;            /* Frobenius pre-normalisation epsilon (1e-7 in the recipe) */
  int32_t ns_steps;     /* Newton-Schulz iterations, 0..16 */
  const float* ns_coef; /* host, ns_steps x 3 (a, b, c) per iteration, or NULL for
                           (3.4445, -4.7750, 2.0315) every iteration */
  int32_t norm;         /* mao_norm_mode */
  int32_t polar;        /* mao_polar */
} mao_muon_params;

/*
 * mao_muon_step — one Muon / Muon+ step on `count` matrices ("Muon+" page,
 * 2 Methodology; "SOAP, Muon and Beyond" review 2-1 and 3-2):
 *   M <- mu M + (1 - mu) G
 *   X0 = M / (||M||_F + eps), transposed when m > n (so X is min(m,n) x max(m,n))
 *   ns_steps times: A = X X^T ; B = b A + c A A ; X <- a X + B X
 *   O = Norm^(d)(X in W's orientation)
 *   W <- W (1 - lr wd) - lr sqrt(m/n) O
 * Newton-Schulz runs in bf16 operands with fp32 accumulation.
 * workspace: device, >= mao_muon_workspace_size() bytes, 256-byte aligned;
 * its contents need no initialisation and are scratch after the call.
 * stats: device array of `count` mao_stats, or NULL.
 */
MAO_API mao_status mao_muon_workspace_size(const mao_muon_mat* mats, int32_t count, const mao_muon_params* p,
                                   size_t* bytes);
MAO_API mao_status mao_muon_step(const mao_muon_mat* mats, int32_t count, const mao_muon_params* p, void* workspace,
                         size_t ws_bytes, mao_stats* stats, mao_stream_t stream);

/* Size of the static device scratch behind mao_muon_step_noalloc. */
#define MAO_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

/*
 * mao_muon_step_noalloc — an addition of this library with no counterpart in
 * the source pages.  Some callers cannot allocate device memory for the step's
 * scratch workspace: a host program that runs under a device-memory budget fixed
 * at start-up, or a caller inside a framework whose own caching allocator owns
 * the device memory, has no allocator at hand for a raw scratch buffer.  This
 * entry point runs the same step as mao_muon_step but takes its scratch from one
 * static device array of MAO_NOALLOC_SCRATCH_BYTES (64 MiB) built into the
 * library, which every GPU that loads the library holds until the process exits.
 *   - The caller still passes the matrices (W, G, M) and optional stats.
 *   - A batch whose mao_muon_workspace_size() exceeds MAO_NOALLOC_SCRATCH_BYTES is
 *     rejected with MAO_ERR_WORKSPACE before anything is enqueued.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make that
 *     first call before any stream capture on that device.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Every call shares the one array, and the array keeps the last call's
 *     contents; each call clears what must start at zero (the status word).
 *     Calls whose work overlaps on the GPU (different streams, or different
 *     threads without ordering) race on the array: serialise them.
 */
MAO_API mao_status mao_muon_step_noalloc(const mao_muon_mat* mats, int32_t count, const mao_muon_params* p,
                                         mao_stats* stats, mao_stream_t stream);

/*
 * mao_muon_noalloc_status — an addition of this library with no counterpart in the
 * source pages.  mao_muon_step_noalloc keeps its device status word at the start of
 * its static scratch, whose address the caller never sees, so mao_workspace_status
 * cannot reach it; this call reads it instead.  It synchronises `stream` and returns
 * MAO_OK if the last mao_muon_step_noalloc on the current device recorded no
 * device-side condition, otherwise that condition (MAO_ERR_TIMEOUT: a bounded wait
 * gave up and W may be partly updated; MAO_ERR_NONFINITE: with stats requested, a
 * non-finite weight was written).  `where` (nullable) receives the site identifier.
 * The first call on a device does the same address look-up as the step.
 */
MAO_API mao_status mao_muon_noalloc_status(mao_stream_t stream, int32_t* where);

/* ------------------------------------------------------------------ SOAP */

typedef struct {
  int32_t m, n;
  float* W;         /* device fp32 m x n, updated in place */
  const void* G;    /* device m x n, fp32 or bf16 */
  int32_t g_dtype;
  float* M;         /* m x n first moment (original space) */
  float* V;         /* m x n second moment (eigenbasis) */
  float* L;         /* m x m left factor */
  float* R;         /* n x n right factor */
  float* QL;        /* m x m left basis (orthonormal columns) */
  float* QR;        /* n x n right basis */
  int32_t* perm_L;  /* device, m entries, or NULL: the permutation applied to Q_L this step */
  int32_t* perm_R;  /* device, n entries, or NULL */
} mao_soap_mat;

typedef struct {
  float beta1, beta2, eps, lr, wd;
  int64_t t; /* 1-based step number shared by the batch (bias correction, schedules) */
  mao_refresh refresh;
} mao_soap_params;

/*
 * mao_soap_step — one two-sided SOAP step with the real-time eigenbasis
 * refresh ("SOAP, Muon and Beyond" review 1-1, 3-2 (3)(4); summary eq. (1)):
 *   L <- b2 L + (1-b2) G G^T ; R <- b2 R + (1-b2) G^T G
 *   on refresh steps, per side: [sort Q by diag(Q^T F Q)], P = F Q, Q <- qr(P)
 *     (positive diagonal); V's rows (left) / columns (right) follow the sort
 *   M <- b1 M + (1-b1) G
 *   Gh = Q_L^T G Q_R ; Mh = Q_L^T M Q_R
 *   V <- b2 V + (1-b2) Gh^2 ; N = (Mh / (1-b1^t)) / (sqrt(V / (1-b2^t)) + eps)
 *   U = Q_L N Q_R^T ; W <- W (1 - lr wd) - lr U
 * Contractions use fp32-faithful tensor-core arithmetic: every fp32 operand is
 * held as three bf16 planes and the six significant cross products accumulate
 * in fp32 (a bf16 G is exact in one plane: G G^T is one product, Q_L^T G three).
 * The workspace size depends on the descriptors and on the refresh policy but
 * not on t: one workspace serves every step of the descriptor set.
 */
MAO_API mao_status mao_soap_workspace_size(const mao_soap_mat* mats, int32_t count, const mao_soap_params* p,
                                   size_t* bytes);
MAO_API mao_status mao_soap_step(const mao_soap_mat* mats, int32_t count, const mao_soap_params* p, void* workspace,
                         size_t ws_bytes, mao_stats* stats, mao_stream_t stream);

/* ------------------------------------------------------------------ FOAM */

typedef struct {
  int32_t m, n;
  float* W;
  const void* G;
  int32_t g_dtype;
  float* M;        /* m x n first moment (original space) */
  float* r;        /* m row second-moment EMA */
  float* c;        /* n column second-moment EMA (follows Q_R's column order) */
  float* R;        /* n x n input-side factor */
  float* QR;       /* n x n input-side basis */
  int32_t* perm_R; /* device, n entries, or NULL */
} mao_foam_mat;

typedef struct {
  float beta1, beta2, eps, lr, wd;
  int64_t t;
  mao_refresh refresh;
  int32_t tau_raw_trace; /* 0: tau uses tr(R/(1-b2^t)) (default); 1: the literal tr(R) */
} mao_foam_params;

/*
 * mao_foam_step — one FOAM step ("Factored One-sided Adam-Moment" review,
 * 1 Key Terms, 3 Method):
 *   R <- b2 R + (1-b2) G^T G
 *   refresh decision (ADAPTIVE: pf, tol) ; on refresh: [sort], P = R Q_R, Q_R <- qr(P);
 *     c follows the sort
 *   M <- b1 M + (1-b1) G ; Gr = G Q_R ; Mr = M Q_R
 *   r <- b2 r + (1-b2) rowmean(Gr^2) ; c <- b2 c + (1-b2) colmean(Gr^2)
 *   tau = tr(R^) / (|r^|_1 |c^|_1) ; v_ij = tau r^_i c^_j (never materialised)
 *   N = (Mr / (1-b1^t)) / (sqrt(v) + eps) ; U = N Q_R^T ; W <- W (1 - lr wd) - lr U
 * Arithmetic and workspace as for mao_soap_step.
 */
MAO_API mao_status mao_foam_workspace_size(const mao_foam_mat* mats, int32_t count, const mao_foam_params* p,
                                   size_t* bytes);
MAO_API mao_status mao_foam_step(const mao_foam_mat* mats, int32_t count, const mao_foam_params* p, void* workspace,
                         size_t ws_bytes, mao_stats* stats, mao_stream_t stream);

/* ------------------------------------------------------------------ misc */

/* Optimizer-state element counts per matrix ("Factored One-sided Adam-Moment"
 * review, 1 Key Terms and 3 Method): SOAP 2mn + 2m^2 + 2n^2, FOAM mn + 2n^2 + m + n,
 * Muon mn.  Pure host functions; 0 for m or n < 1. */
MAO_API uint64_t mao_muon_state_elems(int32_t m, int32_t n);
MAO_API uint64_t mao_soap_state_elems(int32_t m, int32_t n);
MAO_API uint64_t mao_foam_state_elems(int32_t m, int32_t n);

/* Static string for a status code (never NULL). */
MAO_API const char* mao_status_string(int32_t status);

/* Reads the device status word kept at the start of a step's workspace
 * (synchronises `stream`).  MAO_OK if the last step that used this workspace
 * recorded no device-side error; otherwise that error (e.g. MAO_ERR_TIMEOUT).
 * `where` (nullable) receives the site identifier of the error. */
MAO_API mao_status mao_workspace_status(const void* workspace, mao_stream_t stream, int32_t* where);

/* ------------------------------------------------------------------ profiling */

/* Kernel identifiers reported by the launch profiler. */
typedef enum {
  MAO_K_MUON_PREP = 1,     /* momentum EMA + norm partials + bf16 operands (HBM) */
  MAO_K_MUON_SCALE = 2,    /* per-matrix pre-normalisation scale */
  MAO_K_NS_GRAM = 3,       /* A = X X^T (tensor cores) */
  MAO_K_NS_POLY = 4,       /* B = b A + c A A (tensor cores) */
  MAO_K_NS_AXPY = 5,       /* X = a X + B X (tensor cores) */
  MAO_K_MUON_COLSQ = 6,    /* Muon+ column sums of squares */
  MAO_K_MUON_COLSCALE = 7,
  MAO_K_MUON_ROWSCALE = 8,
  MAO_K_MUON_UPDATE = 9,   /* weight update (HBM) */
  MAO_K_MUON_STATS = 10,
  MAO_K_SPLIT3 = 11,         /* fp32 -> three bf16 planes (GEMM verification entry) */
  MAO_K_GEMM_TEST = 12,
  MAO_K_PC_ELEMENTWISE = 13, /* SOAP/FOAM momentum, splits, Adam, r/c/tau, N (HBM) */
  MAO_K_PC_FACTOR = 14,      /* L / R EMA products (tensor cores, fp32-faithful SPLIT3) */
  MAO_K_PC_CHECK = 15,       /* adaptive check D = Q^T F Q and its ratio */
  MAO_K_PC_POWER = 16,       /* power step P = F Q */
  MAO_K_PC_SORT = 17,        /* sort keys, argsort, gathers */
  MAO_K_PC_QR = 18,          /* QR panel projections C = Q^T P, W = P - Q C (tensor cores) */
  MAO_K_PC_ROTATE = 19,      /* rotations into the eigenbasis and back (before the update) */
  MAO_K_PC_UPDATE = 20,      /* last rotation fused with the weight update */
  MAO_K_PC_PANEL = 21,       /* QR panel Gram products (tensor cores, K slices) and their reduction */
  MAO_K_PC_CHOL = 22,        /* QR panel Cholesky and R^{-1} (fp64, one block per panel) */
  MAO_K_PC_QR_APPLY = 23,    /* QR panel products W R^{-1} (tensor cores) */
  MAO_K_PC_QR_REDUCE = 24,   /* sum of the K-slice partials of the projection coefficients */
  MAO_K_PC_STATS = 25,       /* per-matrix diagnostics of a SOAP / FOAM step */
  MAO_K_MOP_INIT = 26        /* exact polar factor: fp32 X0 = M / (||M||_F + eps) and its planes (HBM) */
} mao_kernel_id;

/* What one recorded launch was: its kernel and its algorithmic work (useful
 * floating-point operations and the bytes the algorithm must move). */
typedef struct {
  int32_t kernel; /* mao_kernel_id */
  int32_t pad;
  double flops;     /* algorithmic floating-point operations of the launch (2 per multiply-add);
                       launches whose work is decided on the device count none */
  double bytes;     /* algorithmic bytes moved (memory-bound kernels), else 0 */
  double tc_flops;  /* tensor-core operations issued for `flops`: an fp32-faithful product of
                       three-plane operands issues six bf16 products per multiply-add, a
                       three-plane by one-plane product three, a bf16 product one */
  double exec_flops;    /* operations the device executed, filled by mao_profile_stop(): for a
                           table-mode product counted over the tiles it computed, problems that
                           a device flag let run included; for every other launch equal to
                           flops */
  double exec_tc_flops; /* tensor-core operations the device issued for exec_flops */
} mao_launch_info;

/*
 * Launch profiler for timing inside a caller's timed region.  While active,
 * every kernel launch of the library is bracketed by cudaEventRecord of
 * events[2i] and events[2i+1] on the launching stream (no synchronisation) and
 * info[i] describes it, for the first `capacity` launches.  `events` is a host
 * array of 2*capacity cudaEvent_t created by the caller, or NULL to record only
 * `info`; `info` a host array of `capacity`.  mao_profile_stop() ends recording and returns how many launches
 * happened since the start (which may exceed capacity); with an `info` array it
 * synchronises the device and fills the exec_* fields (the table-mode kernels count
 * their executed work in device counters that mao_profile_start allocates once and
 * clears).  Not thread-safe: one profiling session per process at a time.
 */
MAO_API mao_status mao_profile_start(void** events, mao_launch_info* info, int32_t capacity);
MAO_API int32_t mao_profile_stop(void);

/* MAO_VERSION of the built library. */
MAO_API int32_t mao_version(void);

/* MAO_OK if the current device is an sm_100 part this build's kernels run on,
 * MAO_ERR_UNSUPPORTED otherwise, MAO_ERR_CUDA if no device can be queried. */
MAO_API mao_status mao_device_check(void);

#ifdef __cplusplus
}
#endif

#endif /* MAO_H_ */
