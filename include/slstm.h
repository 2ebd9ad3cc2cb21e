/*
 * slstm.h - C ABI of the Newton-solved diag-mix sLSTM library (libslstm.so).
 *
 * The library solves the diag-mix sLSTM recurrence of xLSTM in parallel over
 * the sequence with Newton iterations whose linear solves are associative
 * scans of 4x4 affine maps, on one NVIDIA B200 (sm_100a).
 *
 * Sources (page titles and sections):
 *   "sLSTM in this library" (pararnn-torch docs): "Cell" (state (B,T,4,d_h)
 *     = (c,n,m,h), hidden slot 3; mix='diag' with channelwise R of shape
 *     (4,d_h) and a 4x4 Jacobian per feature), "API notes" (Newton in
 *     training, sequential stepping in evaluation, W_x is a GEMM, out=
 *     buffers), "Backward" (one reverse associative scan of J^T, then a packed
 *     cell VJP for grad R and grad W_x).
 *   "pararnn-torch structure": "Current surface" (fused kernels prepend h0;
 *     residual early stop; divergence when max|F| > 1 after K), "Naming"
 *     (scan_block4 for the (B,T,4,4,d) layout).
 *   "xLSTM - a from-scratch, educational reimplementation": "Exponential
 *     gating + the stabilizer" (the stabilised step).
 *   "xLSTM: Extended Long Short-Term Memory" (summary): "Method", the sLSTM
 *     step (gate order z, i, f, o; h = o * c / n) and the stabilizer
 *     m_t = max(log f_t + m_{t-1}, log i_t).
 *
 * The cell, per batch row b, feature j and step t (gate order z, i, f, o;
 * slot order c, n, m, h):
 *   a_g = P[b,t,g,j] + R[g,j] * h_{t-1}
 *   z = tanh a_z, o = sigmoid a_o, log i = a_i,
 *   log f = log sigmoid a_f (SLSTM_FORGET_SIGMOID) or a_f (SLSTM_FORGET_EXP)
 *   m = max(log f + m_{t-1}, a_i), i' = exp(a_i - m), f' = exp(log f + m_{t-1} - m)
 *   c = f' c_{t-1} + i' z,  n = f' n_{t-1} + i',  h = o c / n
 * with (c,n,m,h)_{-1} = s0.
 *
 * Conventions shared by every call:
 *   - Every tensor pointer is DEVICE memory owned by the caller, contiguous
 *     (row-major in the stated shape) and 16-byte aligned.  Outputs are
 *     written in full; the library keeps no pointer after the call returns.
 *   - The library allocates no device memory.  Calls that need scratch take
 *     a caller-owned workspace (ws, ws_bytes) of at least
 *     slstm_workspace_size(op, ...) bytes, 256-byte aligned.  Calls that
 *     share a workspace must not overlap in time (use one stream).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and the call returns without synchronising.
 *   - Return value: SLSTM_OK, SLSTM_ERR_INVALID_ARG for arguments rejected on
 *     the host before anything is launched (null or misaligned pointers,
 *     non-positive or too-large sizes, workspace too small, unknown enum), or
 *     SLSTM_ERR_CUDA when a launch fails.  Newton outcomes (iterations,
 *     convergence, divergence, bounded-wait timeouts) are written to the
 *     device-side stats record and read by the caller after synchronising.
 *   - No call aborts, traps or throws.
 *   - Tiles hand scan carries to one another through the workspace with
 *     bounded waits.  A wait that expires (it should never happen; it means
 *     a tile was not scheduled within the limit) makes the carry it waited
 *     for NaN, so every output that depends on it is NaN instead of silently
 *     wrong, and sets a nonzero error word in the workspace: the 32-bit word
 *     at byte offset 4 for scan_block4 and slstm_newton_backward(_varlen)
 *     (cleared by every call), the same word of the library's own block for
 *     scan_block4_noalloc (not readable by the caller; the NaN outputs show
 *     it).  slstm_newton_forward also reports it as SLSTM_ERR_TIMEOUT in its
 *     stats (with the bit 4 of the same word at byte offset 4 of its
 *     workspace when the wait was a grid barrier of its device loop).
 *   - Sizes: 1 <= B <= 65535, 1 <= T, 1 <= d_in, d_h, d <= 2^20, B*T < 2^31
 *     and B * ceil(T/32) * ceil(max(d_in, d_h)/32) < 2^31.
 */
#ifndef SLSTM_H
#define SLSTM_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void *slstm_stream_t; /* a cudaStream_t */

typedef enum {
    SLSTM_OK = 0,
    SLSTM_ERR_INVALID_ARG = 1,
    SLSTM_ERR_CUDA = 2,
    SLSTM_ERR_DIVERGED = 3,    /* stats.error only: max|F| > 1 or non-finite */
    SLSTM_ERR_TIMEOUT = 4,     /* stats.error only: a bounded wait ran out   */
    SLSTM_ERR_UNSUPPORTED = 5  /* valid request the library cannot run       */
} slstm_status;

typedef enum { SLSTM_F32 = 0, SLSTM_BF16 = 1 } slstm_dtype;

typedef enum { SLSTM_FORGET_SIGMOID = 0, SLSTM_FORGET_EXP = 1 } slstm_forget;

/* Operation codes for slstm_workspace_size. */
typedef enum {
    SLSTM_OP_PREACT_GEMM = 0,
    SLSTM_OP_NEWTON_FORWARD = 1,
    SLSTM_OP_SCAN_BLOCK4 = 2,
    SLSTM_OP_NEWTON_BACKWARD = 3,
    SLSTM_OP_NEWTON_FORWARD_VARLEN = 4,   /* B = number of sequences, T = total packed length */
    SLSTM_OP_NEWTON_BACKWARD_VARLEN = 5,  /* B = number of sequences, T = total packed length */
    SLSTM_OP_NEWTON_BACKWARD_HEAD = 6,    /* sized for the largest head width, SLSTM_MAX_HEAD_DIM */
    SLSTM_OP_CONTEXT_PARALLEL = 7         /* one rank's time slice: T = the slice's length */
} slstm_op;

#define SLSTM_MAX_ITERS 65536     /* largest accepted max_iters              */
#define SLSTM_MAX_HEAD_DIM 32     /* largest head width of the head-mixing calls */
#define SLSTM_MAX_GUESS_SWEEPS 64 /* largest guess_sweeps                       */
#define SLSTM_STATS_HISTORY 64    /* residual history kept in the stats record */

/* scan_block4 flags */
#define SLSTM_SCAN_REVERSE_T 1
#define SLSTM_SCAN_DEBUG_WITHHOLD 2   /* fault injection, see scan_block4 */

/*
 * Newton solver settings ("pararnn-torch structure", "Current surface":
 * NewtonConfig(max_iters), residual early stop, fixed-K compile-safe preset).
 *   max_iters   1..SLSTM_MAX_ITERS (0 allowed with SLSTM_INIT_DECOUPLED):
 *               iteration cap (tolerance mode) or the exact iteration count
 *               (fixed mode).
 *   fixed_iters 0: stop at the first iteration whose new iterate meets tol;
 *               1: run exactly max_iters iterations.
 *   tol         tolerance of the stopping test (residual_mode), taken over
 *               every (b, t, slot, j) of the new iterate.
 *   forget      slstm_forget.
 *   debug_fault 0 in normal use.  1 makes one tile of the first iteration
 *               withhold its scan carry, so that its successor's bounded
 *               wait expires (the run then reports SLSTM_ERR_TIMEOUT in
 *               stats.error; results are not meaningful).  2: in the
 *               bounds-checked build, each iteration checks its last tile
 *               boundary store against an extent one element short (the
 *               store is skipped and reported; a self-test of the checks);
 *               ignored in the normal build.  3: the device loop (loop_from)
 *               loses one CTA before its first grid barrier, whose wait then
 *               expires in the others (SLSTM_ERR_TIMEOUT in stats.error; a
 *               self-test of the bounded barrier).
 *   wait_limit_us  upper bound of one bounded wait, in microseconds
 *               (0 = the default of 2 seconds).
 *   carry_mode  how a tile gets the scan carry entering it (same results up
 *               to rounding): SLSTM_CARRY_FUSED, one launch per iteration in
 *               which each tile takes its predecessor's published prefix
 *               (decoupled look-back); SLSTM_CARRY_TWO_PASS, a pass that
 *               stores every tile's aggregate map, a scan of the aggregates
 *               of each feature group, and a pass that applies the carries
 *               (no tile waits on another; cheaper with few feature groups);
 *               SLSTM_CARRY_AUTO (0) picks two passes when there are at
 *               most SMs / 4 feature groups (B * ceil(d_h/32)) and at least
 *               256 chunks of 64 steps, and debug_fault is 0.
 *   init        the initial guess (the pages give none beyond prepending
 *               h0; the default is this library's reading):
 *               SLSTM_INIT_DECOUPLED (0): the trajectory of the cell with
 *               its gates blind to h_{t-1} (R taken as 0: z, o, log i, log f
 *               from P alone, c, n, m recurring exactly), computed by an
 *               associative scan that reads P and writes S, then refined
 *               by guess_sweeps fixed-point sweeps (the same scan with the
 *               gates seeing R h_{t-1} of the previous guess).  The guess
 *               and its first three sweeps run tile by tile in one launch
 *               (P read once, S written once); each further sweep is a
 *               launch of its own that reads P and h and writes S.  From this
 *               guess the solve converges in a few iterations on long
 *               sequences where the zero guess overflows.  In tolerance mode
 *               the first iteration records the guess's residual
 *               (stats.init_max_*); max_iters may then be 0, which returns
 *               the guess itself;
 *               SLSTM_INIT_ZERO: S = 0 at every step;
 *               SLSTM_INIT_GIVEN: S holds the guess on entry (warm start).
 *               The stopping test starts with iteration 1 in every case.
 *   guess_sweeps  0..SLSTM_MAX_GUESS_SWEEPS refinement sweeps of the
 *               decoupled guess (ignored by the other inits).
 *   residual_mode  the stopping test: SLSTM_RESIDUAL_SCALED (0),
 *               max |F| / (1 + |s|) <= tol; SLSTM_RESIDUAL_RAW, max|F| <= tol
 *               (the pages' own norm).  Both maxima are recorded either way.
 *   history     what an iteration records of its residual (tolerance mode):
 *               SLSTM_HISTORY_BOUND (0): once any part of the new iterate
 *               fails the test the solve goes on whatever the rest is, so the
 *               rest of that iteration only checks that its states are
 *               finite; the recorded maxima of such an iteration are then
 *               lower bounds of its residual (still above tol).  The
 *               iteration that stops the solve, the last allowed one and
 *               every fixed-K run record exact maxima, and the decisions
 *               (converged, diverged, non-finite) are those of the exact
 *               residual;  SLSTM_HISTORY_EXACT: every iteration evaluates and
 *               records its whole residual.  (Packed sequences and rows that
 *               are not 16-byte aligned always take the exact history.)
 *   n_events, events  optional per-launch timing (0 / NULL: none): events
 *               holds n_events CUDA events (cudaEvent_t handles, created by
 *               the caller); events[i] is recorded on the stream just before
 *               the call's i-th launch of work and events[n] just after its
 *               last, for the indices below n_events.  The launches in order:
 *               the guess launches (one with up to three sweeps, plus one per
 *               further sweep; none for SLSTM_INIT_ZERO, a small copy kernel
 *               for SLSTM_INIT_GIVEN), then one per iteration up to max_iters
 *               (with the two-pass carry an iteration's three kernels count as
 *               one; the device loop below counts as one launch); launches
 *               after the stop return at once but are still bracketed.  The
 *               events past the last launch's are all recorded after it, so
 *               events[n_events - 1] marks the end of the call whatever the
 *               number of launches.  Timing only: results do not depend on
 *               them.
 *               slstm_newton_forward and slstm_newton_forward_varlen only.
 *   loop_from   tolerance mode with the fused carry: the iterations from
 *               this one on (counting from 0) run inside one cooperative
 *               launch that loops on the device, a grid-wide barrier between
 *               two iterations, and ends as soon as the stopping rule does,
 *               so a converged solve does not pay for the rest of its cap.
 *               0: SLSTM_DEFAULT_LOOP_FROM; negative: never (one launch per
 *               iteration).  The earlier iterations, the fixed mode, the
 *               two-pass carry and calls on a stream being captured into a
 *               graph keep one launch per iteration.  Results do not depend
 *               on it.
 */
#define SLSTM_DEFAULT_LOOP_FROM 2
typedef enum { SLSTM_CARRY_AUTO = 0, SLSTM_CARRY_FUSED = 1, SLSTM_CARRY_TWO_PASS = 2 } slstm_carry_mode;

typedef enum { SLSTM_INIT_DECOUPLED = 0, SLSTM_INIT_ZERO = 1, SLSTM_INIT_GIVEN = 2 } slstm_init;

typedef enum { SLSTM_RESIDUAL_SCALED = 0, SLSTM_RESIDUAL_RAW = 1 } slstm_residual_mode;

typedef enum { SLSTM_HISTORY_BOUND = 0, SLSTM_HISTORY_EXACT = 1 } slstm_history;

typedef struct {
    int max_iters;
    int fixed_iters;
    float tol;
    int forget;
    int debug_fault;
    int wait_limit_us;
    int carry_mode;
    int init;
    int residual_mode;
    int guess_sweeps;
    int history;
    int n_events;
    void *const *events;
    int loop_from;
} slstm_newton_config;

/*
 * Newton outcome, in DEVICE memory owned by the caller (zeroing it is not
 * required; slstm_newton_forward initialises it on the stream).
 *   iters        Newton iterations performed (the initial guess is not one).
 *   converged    1 when the last iterate meets the stopping test.
 *   diverged     1 when not converged and max|F| > 1 or non-finite after the
 *                last iteration ("NewtonDivergenceError" of the pages).
 *   error        0, SLSTM_ERR_DIVERGED when diverged, or SLSTM_ERR_TIMEOUT.
 *   max_abs_F[k % 64], max_scaled_F[k % 64]   residual of the iterate
 *                produced by iteration k (max over every element), for the
 *                last min(iters, 64) iterations.  In fixed mode only the final
 *                iteration evaluates its residual; the others hold -1.
 *   init_max_abs_F, init_max_scaled_F   residual of the initial guess,
 *                recorded by the first iteration (SLSTM_INIT_DECOUPLED in
 *                tolerance mode), else -1.
 */
typedef struct {
    int iters;
    int converged;
    int diverged;
    int error;
    float max_abs_F[SLSTM_STATS_HISTORY];
    float max_scaled_F[SLSTM_STATS_HISTORY];
    float init_max_abs_F;
    float init_max_scaled_F;
} slstm_newton_stats;

/* Human-readable name of a status code (static string, never NULL). */
const char *slstm_status_string(int status);

/*
 * Bounds-checked build.  The library can also be built with SLSTM_CHECKED
 * defined (a separate diagnostic library, libslstm_checked.so): there every
 * guarded global-memory access of the kernels tests its element index
 * against the extent of its buffer, skips the access when it is outside,
 * counts it and records the first one.  Nothing traps; the kernels run on.
 *   slstm_check_enabled  1 in the checked build, 0 in the normal one.
 *   slstm_check_status   waits for the device, then writes out[0] = the
 *                        number of out-of-bounds accesses since the last
 *                        clear and, for the first of them (0 when none),
 *                        out[1] = its site (file id * 100000 + source line;
 *                        slstm_check_site_file names the file), out[2] = the
 *                        element index, out[3] = the extent.  All zero in the
 *                        normal build.  SLSTM_ERR_INVALID_ARG for a null out,
 *                        SLSTM_ERR_CUDA when the device cannot be read.
 *   slstm_check_clear    zeroes the records (waits for the device).
 *   slstm_check_site_file  the source file of a site's file id, or NULL.
 */
int slstm_check_enabled(void);
int slstm_check_status(long long *out);
int slstm_check_clear(void);
const char *slstm_check_site_file(int file_id);

/*
 * Bytes of workspace an operation needs for the given sizes (0 when it needs
 * none).  Unused size arguments may be 0.  Returns 0 for invalid input.
 */
size_t slstm_workspace_size(int op, int B, int T, int d_in, int d_h);

/*
 * Input projection ("sLSTM in this library", "API notes": W_x is a GEMM;
 * the summary's sLSTM step: W_* x + b_*):
 *   P[b,t,g,j] = sum_k x[b,t,k] * Wx[g*d_h + j, k] + bias[g,j]
 *   x     (B, T, d_in)  dtype `dtype` (SLSTM_F32 or SLSTM_BF16)
 *   Wx    (4*d_h, d_in) same dtype; rows gate-major (z, i, f, o)
 *   bias  (4, d_h) fp32
 *   P     (B, T, 4, d_h) fp32 output
 * bf16 inputs run on the tcgen05 tensor cores with fp32 accumulation; fp32
 * inputs run an fp32 CUDA-core GEMM.  bf16 requires d_in % 8 == 0.
 */
int slstm_preact_gemm(const void *x, const void *Wx, int dtype, const float *bias, float *P,
                      int B, int T, int d_in, int d_h, void *ws, size_t ws_bytes,
                      slstm_stream_t stream);

/*
 * Tile shape of every tensor-core (bf16) GEMM of the library: the input
 * projection, the gradient GEMMs and the trunk layer's GEMMs.
 *   SLSTM_GEMM_TILES_PAIR: 256 x 256 tiles of C on a pair of SMs (a cluster
 *     of two CTAs, tcgen05 cta_group::2); each SM stages its own 128 rows of
 *     A and 128 rows of B, and the pair's tensor cores read both.
 *   SLSTM_GEMM_TILES_SINGLE: 128 x 256 tiles, one CTA per SM.
 *   SLSTM_GEMM_TILES_AUTO (the default): SM pairs for the products whose
 *     work items span at least 4096 of K and only store C (the gradient
 *     GEMMs), single SMs for the others, whose output stream the pair's
 *     shared accumulator hand-off slows (the input projection, the trunk
 *     layer's forward GEMMs).
 * Where clusters of two cannot run, single-SM tiles are used.  Process-wide
 * setting (not synchronised with calls in flight on other host threads).
 * Both shapes compute the same fp32-accumulated products; the input
 * projection is identical bit for bit, while the gradient GEMMs may round
 * differently (their split-K counts follow the tile shape).  Returns the
 * previous setting, or -1 (and changes nothing) for another value.
 */
typedef enum { SLSTM_GEMM_TILES_AUTO = 0, SLSTM_GEMM_TILES_PAIR = 1, SLSTM_GEMM_TILES_SINGLE = 2 } slstm_gemm_tiles;
int slstm_set_gemm_tiles(int tiles);

/*
 * Newton solve of the whole trajectory ("sLSTM in this library", "Cell";
 * "pararnn-torch structure", "Current surface"):
 *   initial guess as cfg->init selects; s0 enters as the step before t = 0;
 *   each iteration evaluates F_t = S_t - f(S_{t-1}, P_t) and J_t = df/ds_{t-1}
 *   at the guess, solves delta_t = J_t delta_{t-1} - F_t (delta_{-1} = 0) by a
 *   blocked associative scan of 4x4 affine maps, and sets S <- S + delta;
 *   it then evaluates the residual of the new iterate for the stopping test.
 *   P     (B, T, 4, d_h) fp32
 *   R     (4, d_h) fp32
 *   s0    (B, 4, d_h) fp32, or NULL for zeros
 *   S     (B, T, 4, d_h) fp32 output (the last iterate; h is slot 3)
 *   cfg   host pointer, read during the call
 *   stats device pointer to one slstm_newton_stats, written on the stream
 * The call enqueues up to max_iters iterations without synchronising with the
 * host: in tolerance mode the first cfg->loop_from of them as launches of
 * their own and the rest as one launch that loops on the device and ends
 * with the solve (see loop_from); iterations after convergence (or after a
 * timeout or non-finite residual) do no work.  Two calls may run on one
 * workspace only in stream order; the device loop needs every CTA of its
 * cooperative launch resident, which the library's grid size ensures.
 */
int slstm_newton_forward(const float *P, const float *R, const float *s0, float *S,
                         const slstm_newton_config *cfg, slstm_newton_stats *stats, int B, int T,
                         int d_h, void *ws, size_t ws_bytes, slstm_stream_t stream);

/*
 * Associative scan of 4x4 affine maps ("pararnn-torch structure", "Naming":
 * scan_block4 for the (B,T,4,4,d) layout; "sLSTM in this library", "Packed
 * sequences": the Newton inner solve is a scan on the (J, r) monoid):
 *   flags = 0:                    y_t = A_t y_{t-1} + b_t,   y_{-1} = y0
 *   flags = SLSTM_SCAN_REVERSE_T: y_t = A_t^T y_{t+1} + b_t, y_T   = y0
 *   A   (B, T, 4, 4, d) fp32, indexed [b][t][row][col][j]
 *   b   (B, T, 4, d) fp32
 *   y0  (B, 4, d) fp32, or NULL for zeros
 *   y   (B, T, 4, d) fp32 output; may not alias A or b
 * Composition is in fp32.  The reverse mode pairs A_t^T with b_t at the same
 * index t; the map that carries y_{t+1} back to step t is the one stored at
 * t (a deliberate reading: the caller stores, at step t, the transpose it
 * wants applied there).
 * flags may also hold SLSTM_SCAN_DEBUG_WITHHOLD (tests only, needs T > 64):
 * the tile of steps 32..63 (in processing order) of batch row 0, features
 * 0..31 withholds its carry; the next tile's bounded wait (20 ms in this
 * mode) expires, and the outputs of those features from step 64 (in
 * processing order) on are NaN.  The rest is computed as usual.
 */
int scan_block4(const float *A, const float *b, const float *y0, float *y, int B, int T, int d,
                int flags, void *ws, size_t ws_bytes, slstm_stream_t stream);

/*
 * scan_block4 for callers that cannot allocate device memory.  (The pages
 * have no counterpart of this call; it is a service of this library.)
 * Some callers own no workspace to pass: their own allocator has reserved
 * every byte of the GPU, or they may not call cudaMalloc because it can
 * synchronise the device, or they are plugins handed only input and output
 * pointers.  This entry point takes the same arguments as scan_block4
 * minus the workspace, and computes the same result, using scratch from one
 * fixed block of SLSTM_NOALLOC_SCRATCH_BYTES of device memory that the
 * library reserves on every GPU that loads it, held until the process exits.
 *   - It allocates nothing.  The first call on each device looks up the
 *     block's device address (a one-time set-up); make that first call
 *     before any stream capture begins.
 *   - All calls on a device share the block.  Calls that overlap on the same
 *     GPU (other streams, other host threads) race on it: serialise them.
 *     Each call clears the counters and flags it relies on before use.
 *   - Returns SLSTM_ERR_UNSUPPORTED when the problem needs more scratch than
 *     the block holds, that is when slstm_workspace_size(SLSTM_OP_SCAN_BLOCK4,
 *     B, T, 0, d) > SLSTM_NOALLOC_SCRATCH_BYTES (up to 2337 tiles of 32 steps
 *     x 32 features: B * ceil(T/32) * ceil(d/32) <= 2337); other errors as
 *     scan_block4.
 */
#define SLSTM_NOALLOC_SCRATCH_BYTES (8u << 20)
int scan_block4_noalloc(const float *A, const float *b, const float *y0, float *y, int B, int T,
                        int d, int flags, slstm_stream_t stream);

/*
 * Sequential stepping ("sLSTM in this library", "API notes": the evaluation
 * path; T_steps = 1 is one decode step):
 *   S_t = f(S_{t-1}, P_t) for t = 0 .. T_steps-1, S_{-1} = s0.
 *   P (B, T_steps, 4, d_h), R (4, d_h), s0 (B, 4, d_h) or NULL, S (B, T_steps, 4, d_h).
 */
int slstm_sequential_step(const float *P, const float *R, const float *s0, float *S, int B,
                          int T_steps, int d_h, int forget, slstm_stream_t stream);

/*
 * One decode step for B batch rows ("sLSTM in this library", "API notes": at
 * T = 1 evaluation is one recurrent step; "pararnn-torch structure": the T = 1
 * step is replayed under CUDA graphs): the input projection fused with the
 * cell update,
 *   P[b, g, j]     = sum_k Wx[g d_h + j, k] x[b, k] + bias[g, j]
 *   s_next[b, :, j] = f(s_prev[b, :, j], P[b, :, j])      (f as in slstm_newton_forward)
 * x: (B, d_in), Wx: (4 d_h, d_in), both of `dtype` (SLSTM_F32 or SLSTM_BF16),
 * d_in a multiple of 4 (f32) or 8 (bf16).  bias, R: (4, d_h) fp32.  s_prev:
 * (B, 4, d_h) fp32 or NULL (zero state); s_next: (B, 4, d_h) fp32, which may
 * be s_prev itself (in-place step) but must not overlap it otherwise.  All
 * pointers device memory owned by the caller, 16-byte aligned.  W_x is read
 * once per 16 batch rows; accumulation in fp32.  One launch per 16 rows, no
 * workspace, no synchronisation, so a sequence of steps can be captured in a
 * CUDA graph.  Returns SLSTM_ERR_INVALID_ARG for bad sizes, dtype, forget mode
 * or alignment (before touching the GPU), SLSTM_ERR_CUDA for a launch error.
 */
int slstm_decode_step(const void *x, const void *Wx, int dtype, const float *bias, const float *R,
                      const float *s_prev, float *s_next, int forget, int B, int d_in, int d_h,
                      slstm_stream_t stream);

/*
 * Gradients of L = sum_{b,t,j} dH[b,t,j] * h[b,t,j] at the solution S
 * ("sLSTM in this library", "Backward": one reverse associative scan of J^T,
 * then the packed cell VJP):
 *   lambda_t = e_h dH_t + J_{t+1}^T lambda_{t+1}   (reverse scan, fp32)
 *   dP_t = G_t^T lambda_t with G_t = ds_t/da_t, a_t = P_t + R h_{t-1}
 *   dR[g,j] = sum_{b,t} dP[b,t,g,j] h[b,t-1,j]; db[g,j] = sum_{b,t} dP[b,t,g,j]
 *   ds0 = J_0^T lambda_0;  dx = dP Wx;  dWx = dP^T x
 *   x (B,T,d_in) and Wx (4*d_h,d_in) in `dtype`; P, S (B,T,4,d_h); R (4,d_h);
 *   s0 (B,4,d_h) or NULL; dH (B,T,d_h); outputs fp32: dx (B,T,d_in),
 *   dWx (4*d_h,d_in), dR (4,d_h), db (4,d_h), ds0 (B,4,d_h) (may be NULL).
 */
int slstm_newton_backward(const void *x, const void *Wx, int dtype, const float *P,
                          const float *R, const float *s0, const float *S, const float *dH,
                          float *dx, float *dWx, float *dR, float *db, float *ds0, int forget,
                          int B, int T, int d_in, int d_h, void *ws, size_t ws_bytes,
                          slstm_stream_t stream);

/*
 * Packed ragged sequences ("sLSTM in this library", "Packed sequences": time
 * packed as (1, N, ...) with FlashAttention-style exclusive-prefix offsets,
 * one initial state per sequence, the Newton inner solve a segmented scan on
 * the (J, r) monoid with a head flag at each sequence start).
 *   cu_seqlens  device int32 array of n_seq + 1 offsets: cu_seqlens[0] = 0,
 *               nondecreasing, cu_seqlens[n_seq] = total_T; sequence k
 *               occupies packed steps [cu_seqlens[k], cu_seqlens[k+1]) and
 *               may be empty
 *   P, S        (total_T, 4, d_h) fp32;  dH (total_T, d_h);  x (total_T, d_in)
 *   s0, ds0     (n_seq, 4, d_h) fp32, s0 may be NULL (zeros), ds0 may be NULL
 * At a sequence's first step the previous state is its own s0 and the step
 * does not depend on the step before it (a zero Jacobian: the head flag), so
 * every sequence is solved exactly as on its own; the stopping test and the
 * stats are over all sequences together.  The offsets are read on the
 * device: the forward checks them and, when they are malformed, writes
 * SLSTM_ERR_INVALID_ARG to stats->error and leaves S untouched; both calls
 * clamp every offset into [0, total_T], so malformed offsets never lead to an
 * access outside the arrays.  Workspace: slstm_workspace_size with
 * SLSTM_OP_NEWTON_FORWARD_VARLEN / _BACKWARD_VARLEN, B = n_seq, T = total_T.
 * Other arguments and errors as slstm_newton_forward / slstm_newton_backward.
 */
int slstm_newton_forward_varlen(const float *P, const float *R, const float *s0, const int *cu_seqlens,
                                int n_seq, float *S, const slstm_newton_config *cfg, slstm_newton_stats *stats,
                                int total_T, int d_h, void *ws, size_t ws_bytes, slstm_stream_t stream);

int slstm_newton_backward_varlen(const void *x, const void *Wx, int dtype, const float *P, const float *R,
                                 const float *s0, const int *cu_seqlens, int n_seq, const float *S,
                                 const float *dH, float *dx, float *dWx, float *dR, float *db, float *ds0,
                                 int forget, int total_T, int d_in, int d_h, void *ws, size_t ws_bytes,
                                 slstm_stream_t stream);

/*
 * Time context parallel ("sLSTM in this library", section "Tensor parallel":
 * context parallel splits time).  Rank r of n holds the steps of its time
 * slice of every sequence: P and S are (B, T, 4, d_h) with T the slice's
 * length (it may differ between ranks; B and d_h may not).  A solve keeps the
 * single-GPU call's arithmetic, with every scan split into three phases:
 * each rank composes its slice into one map (…_run / …_map), the caller
 * gathers every rank's map on every rank (an all-gather: NCCL over NVLink in
 * the Python layer; nothing here communicates), and each rank enters its
 * slice through the maps of the ranks before it (…_apply).  The solve:
 *   guess:  slstm_cp_guess_run(sweep 0) -> gather runs -> slstm_cp_guess_apply(sweep 0)
 *   each refinement sweep: gather every rank's last state of the current
 *           guess, then slstm_cp_guess_run(sweep 1) -> gather runs ->
 *           slstm_cp_guess_apply(sweep 1)
 *   each Newton iteration: gather last states, slstm_cp_newton_map ->
 *           gather maps -> slstm_cp_newton_apply, whose stats record
 *           (max_abs_F[0], max_scaled_F[0]) holds the slice's residual
 *           maxima of the new iterate; the caller takes the maximum over
 *           ranks for the stopping test.
 * Arguments:
 *   s_before  (B, 4, d_h) the current iterate's (or, for a sweep, the
 *             previous guess's) state just before the slice: the last state
 *             of rank r - 1, or the sequences' s0 on rank 0 (NULL: zero)
 *   s0        (B, 4, d_h) the sequences' initial state (NULL: zero); only its
 *             value on the ranks' apply matters
 *   run       (B, 5, d_h) output: the slice's run of the guess's monoid
 *             (log f sum, stabiliser, u, v, last output gate)
 *   runs      (n, B, 5, d_h) every rank's run in rank order (ranks before
 *             `rank` are read; may be NULL on rank 0)
 *   map       (B, 20, d_h) output: the slice's affine map of the linear
 *             solve (4x4 row-major, then the offset)
 *   maps      (n, B, 20, d_h) every rank's map in rank order
 *   cfg       tol and residual_mode are used (the rest is fixed: one
 *             iteration from the given iterate)
 * slstm_cp_newton_map and slstm_cp_newton_apply of one iteration share the
 * workspace (the apply reuses the tile maps the map call left there).
 * Workspace: slstm_workspace_size(SLSTM_OP_CONTEXT_PARALLEL, B, T, 0, d_h).
 */
int slstm_cp_guess_run(const float *P, const float *R, const float *s_before, const float *S, int sweep,
                       int forget, float *run, int B, int T, int d_h, void *ws, size_t ws_bytes,
                       slstm_stream_t stream);

int slstm_cp_guess_apply(const float *P, const float *R, const float *s0, const float *s_before,
                         const float *runs, int rank, float *S, int sweep, int forget, int B, int T, int d_h,
                         void *ws, size_t ws_bytes, slstm_stream_t stream);

int slstm_cp_newton_map(const float *P, const float *R, const float *s_before, const float *S, int forget,
                        float *map, int B, int T, int d_h, void *ws, size_t ws_bytes, slstm_stream_t stream);

int slstm_cp_newton_apply(const float *P, const float *R, const float *s_before, const float *maps, int rank,
                          float *S, const slstm_newton_config *cfg, slstm_newton_stats *stats, int B, int T,
                          int d_h, void *ws, size_t ws_bytes, slstm_stream_t stream);

/*
 * Head mixing ("sLSTM in this library", section "Cell", row 'head': Beck's
 * block-diagonal R of shape (4, n_heads, d_head, d_head), n_heads d_head =
 * d_h; the factorised Newton, reverse pass and packed VJP that never form
 * the dense (4 d_head)^2 Jacobian, fused for d_head <= 32).  The recurrent
 * input of gate g of feature i of head hd is
 *   sum_k R_head[g][hd][i][k] h_{t-1}[hd d_head + k]
 * in place of diag mixing's R[g][j] h_{t-1}[j]; everything else is the cell
 * of slstm_newton_forward.  R_head is (4, n_heads, d_head, d_head) fp32,
 * 1 <= d_head <= SLSTM_MAX_HEAD_DIM and d_head divides d_h; other tensors and
 * conventions as the diag calls.  One warp serves one (batch row, head):
 * the Jacobian's h column is applied as G (R_head delta_h) (G = ds/da per
 * feature), so the Newton linear solve runs as a recurrence of these
 * matrix-vector products over time, in parallel over batch rows and heads.
 *
 * slstm_sequential_step_head: S_t = f(S_{t-1}, P_t) stepped over T_steps.
 * slstm_newton_forward_head: the Newton solve; cfg as slstm_newton_forward
 *   (debug_fault and guess_sweeps must be 0; carry_mode is ignored).  With
 *   SLSTM_INIT_DECOUPLED the guess is the same decoupled trajectory (it does
 *   not depend on the mixing); its residual is not recorded.  Workspace: slstm_workspace_size(
 *   SLSTM_OP_NEWTON_FORWARD, B, T, 0, d_h).
 * slstm_newton_backward_head: gradients of L = sum dH * h as
 *   slstm_newton_backward, with dR_head (4, n_heads, d_head, d_head) in
 *   place of dR.  Workspace: slstm_workspace_size(
 *   SLSTM_OP_NEWTON_BACKWARD_HEAD, B, T, d_in, d_h).
 * Errors: SLSTM_ERR_INVALID_ARG for a d_head outside 1..32 or not dividing
 * d_h, and as the diag calls otherwise.
 */
int slstm_sequential_step_head(const float *P, const float *R_head, const float *s0, float *S, int B,
                               int T_steps, int d_h, int d_head, int forget, slstm_stream_t stream);

int slstm_newton_forward_head(const float *P, const float *R_head, const float *s0, float *S,
                              const slstm_newton_config *cfg, slstm_newton_stats *stats, int B, int T,
                              int d_h, int d_head, void *ws, size_t ws_bytes, slstm_stream_t stream);

int slstm_newton_backward_head(const void *x, const void *Wx, int dtype, const float *P, const float *R_head,
                               const float *s0, const float *S, const float *dH, float *dx, float *dWx,
                               float *dR_head, float *db, float *ds0, int forget, int B, int T, int d_in,
                               int d_h, int d_head, void *ws, size_t ws_bytes, slstm_stream_t stream);

/*
 * The trunk layer, forward ("sLSTM in this library", section "Stacking":
 * RMSNorm -> ParaRNN(ParaSLSTM) -> residual -> RMSNorm -> SwiGLU -> residual):
 *   z1 = RMSNorm(x) * norm1_w,  P = z1 Wx^T + bias,  S = the cell's solution
 *        on P from the zero state (Newton, as slstm_newton_forward with cfg)
 *   u  = x + h  (h = slot 3 of S),  z2 = RMSNorm(u) * norm2_w
 *   y  = u + W_down (silu(W_gate z2) * (W_up z2))
 * with RMSNorm(v) = v / sqrt(mean over the d_model axis of v^2 + eps).
 *   x, y     (B, T, d_model) fp32; y may be x (in place), must not overlap S
 *   norm1_w, norm2_w  (d_model) fp32;  bias, R (4, d_model) fp32
 *   Wx       (4 d_model, d_model) bf16, gate-major rows g d_model + j
 *   W_gu     (2 d_ff, d_model) bf16: W_gate and W_up interleaved in blocks
 *            of 32 rows (rows 64 k .. 64 k + 31 = W_gate rows 32 k .. 32 k + 31,
 *            rows 64 k + 32 .. 64 k + 63 = W_up rows 32 k .. 32 k + 31)
 *   W_down   (d_model, d_ff) bf16
 *   S        (B, T, 4, d_model) fp32, the cell's states (kept for a backward pass)
 * d_model a multiple of 8, d_ff a multiple of 32.  The GEMM operands z1, z2
 * and the SwiGLU product are rounded to bf16; accumulation and everything
 * else in fp32.  The SwiGLU product and the residual are formed in the GEMM
 * epilogues.  Workspace: slstm_block_workspace_size(B, T, d_model, d_ff) bytes,
 * 256-byte aligned.  Stats and errors as slstm_newton_forward (argument errors
 * before touching the GPU); a bounded wait that expires inside a GEMM sets
 * the first 4-byte word of the workspace nonzero.
 */
size_t slstm_block_workspace_size(int B, int T, int d_model, int d_ff);

int slstm_block_forward(const float *x, const float *norm1_w, const void *Wx, const float *bias, const float *R,
                        const float *norm2_w, const void *W_gu, const void *W_down, float *y, float *S,
                        const slstm_newton_config *cfg, slstm_newton_stats *stats, int B, int T, int d_model,
                        int d_ff, float eps, void *ws, size_t ws_bytes, slstm_stream_t stream);

/*
 * Gradients of L = sum(dY * y) for y = slstm_block_forward(...), given x, the
 * weights and the forward's S (the layer's activations are recomputed):
 *   dx (B, T, d_model), dnorm1_w, dnorm2_w (d_model), dWx (4 d_model,
 *   d_model), dbias, dR (4, d_model), dW_gu (2 d_ff, d_model; the interleaved
 *   row order of W_gu), dW_down (d_model, d_ff), all fp32, caller-owned,
 *   16-byte aligned, none overlapping an input.
 * Read as the gradient of the layer with unrounded operands (the bf16
 * rounding of z1, z2 and the SwiGLU product is piecewise constant): the
 * recomputed z1 and z2 are the forward's bf16 values, every gradient is
 * formed in fp32.  The cell's part is slstm_newton_backward's (dH = dL/du,
 * zero initial state, its tensor-core GEMMs); the FFN gradient GEMMs run on
 * the tensor cores with the fp32 upstream gradients as bf16 hi + lo pairs.
 * Sizes as slstm_block_forward and B * T <= 16 776 960 (65535 chunks of 256
 * rows for the norm weights' column sums); workspace:
 * slstm_block_backward_workspace_size(B, T, d_model, d_ff) bytes, 256-byte
 * aligned.  Returns SLSTM_ERR_INVALID_ARG before touching the GPU for bad
 * sizes, forget mode, eps, alignment or workspace.
 */
size_t slstm_block_backward_workspace_size(int B, int T, int d_model, int d_ff);

int slstm_block_backward(const float *x, const float *norm1_w, const void *Wx, const float *bias, const float *R,
                         const float *norm2_w, const void *W_gu, const void *W_down, const float *S, const float *dY,
                         float *dx, float *dnorm1_w, float *dWx, float *dbias, float *dR, float *dnorm2_w,
                         float *dW_gu, float *dW_down, int forget, int B, int T, int d_model, int d_ff, float eps,
                         void *ws, size_t ws_bytes, slstm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SLSTM_H */
