// Internal launchers behind the C ABI in slstm_api.cu.  Arguments have been
// validated by the caller; every launcher only enqueues work on `st`.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/slstm.h"

namespace slstm {

// Per-iteration counters; iteration k uses slot k & 1 and its finalizer
// clears the other slot for iteration k + 1.
struct NewtonSlot {
    unsigned ticket;
    unsigned finished;
    unsigned maxF_raw;     // float bits of a non-negative max
    unsigned maxF_scaled;
    unsigned failed;       // nonzero once a residual of this iteration failed the stopping test
};

// Device-side control block of one slstm_newton_forward call.
struct NewtonCtrl {
    unsigned done;
    unsigned error;
    unsigned init_raw;      // residual of the initial guess (float bits), recorded by the first iteration
    unsigned init_scaled;
    unsigned gbar;          // grid-barrier arrivals of the device loop over iterations
    unsigned pad[11];
    NewtonSlot slot[2];
};

// Packed ragged sequences: the head flags of the packed time axis, built on
// the device from cu_seqlens.  mask[c] bit i: step 32 c + i is the first step
// of a nonempty sequence, whose index is seq[32 c + i].  err: nonzero when
// the offsets are malformed.
struct Varlen {
    const int *cu;     // the caller's offsets (n_seq + 1)
    int n_seq;
    unsigned *mask;    // [ceil(total_T / 32)]
    int *seq;          // [total_T]
    unsigned *err;
};
size_t varlen_table_bytes(int total_T);
// Carve the table out of `ws` (varlen_table_bytes(total_T) bytes, 256-aligned).
Varlen varlen_layout(const int *cu, int n_seq, int total_T, void *ws);
// Build the table on `st`.  On malformed offsets: *err = 1 and, when given,
// stats->error = SLSTM_ERR_INVALID_ARG and *done = 1.  Offsets are clamped to
// [0, total_T] either way.
cudaError_t varlen_build(const Varlen &v, int total_T, slstm_newton_stats *stats, unsigned *done,
                         cudaStream_t st);

size_t newton_workspace_bytes(int B, int T, int d);
// vl: packed ragged sequences (B = 1, T = total_T), or null for B sequences of T.
cudaError_t newton_forward(const float *P, const float *R, const float *s0, float *S,
                           const slstm_newton_config &cfg, slstm_newton_stats *stats, int B, int T,
                           int d, void *ws, cudaStream_t st, const Varlen *vl = nullptr);

// The head-mixing solve's set-up in a Newton workspace (newton_workspace_bytes):
// clears the control block and the stats record and, for SLSTM_INIT_DECOUPLED,
// enqueues the decoupled guess into S (its residual is not tested).  *ctrl
// receives the call's control block.
cudaError_t newton_guess_prepare(const float *P, const float *s0, float *S, const slstm_newton_config &cfg,
                                 slstm_newton_stats *stats, int B, int T, int d, void *ws, cudaStream_t st,
                                 NewtonCtrl **ctrl);

// Head mixing (head.cu): R_head (4, d / dh, dh, dh), 1 <= dh <= 32, dh | d.
cudaError_t head_sequential_launch(const float *P, const float *Rh, const float *s0, float *S, int B, int T, int d,
                                   int dh, int forget, cudaStream_t st);
// Workspace: newton_workspace_bytes(B, T, d).
cudaError_t head_newton_forward(const float *P, const float *Rh, const float *s0, float *S,
                                const slstm_newton_config &cfg, slstm_newton_stats *stats, int B, int T, int d,
                                int dh, void *ws, cudaStream_t st);
size_t head_backward_workspace_bytes(int B, int T, int d_in, int d, int dh);
cudaError_t head_backward_launch(const void *x, const void *Wx, int dtype, const float *P, const float *Rh,
                                 const float *s0, const float *S, const float *dH, float *dx, float *dWx, float *dRh,
                                 float *db, float *ds0, int forget, int B, int T, int d_in, int d, int dh, void *ws,
                                 cudaStream_t st);

// Time context parallel (newton.cu): the phases of a solve split over time
// slices; the caller exchanges the slice results between the phases.
size_t cp_workspace_bytes(int B, int T, int d);
cudaError_t cp_guess_run(const float *P, const float *R, const float *s_before, const float *S, bool sweep, int forget,
                         float *run_out, int B, int T, int d, void *ws, cudaStream_t st);
cudaError_t cp_guess_apply(const float *P, const float *R, const float *s0, const float *s_before,
                           const float *runs, int rank, float *S, bool sweep, int forget, int B, int T, int d,
                           void *ws, cudaStream_t st);
cudaError_t cp_newton_map(const float *P, const float *R, const float *s_before, const float *S, int forget,
                          float *map_out, int B, int T, int d, void *ws, cudaStream_t st);
cudaError_t cp_newton_apply(const float *P, const float *R, const float *s_before, const float *maps, int rank,
                            float *S, const slstm_newton_config &cfg, slstm_newton_stats *stats, int B, int T, int d,
                            void *ws, cudaStream_t st);

size_t scan_workspace_bytes(int B, int T, int d);
// debug_withhold: host-requested fault injection (one tile withholds its
// carry; its successor's bounded wait expires and the outputs after it are NaN).
cudaError_t scan_block4_launch(const float *A, const float *b, const float *y0, float *y, int B,
                               int T, int d, bool reverse, void *ws, cudaStream_t st, bool debug_withhold = false);

cudaError_t decode_launch(const void *x, const void *Wx, int dtype, const float *bias, const float *R,
                          const float *s_prev, float *s_next, int forget, int B, int d_in, int d, cudaStream_t st);
cudaError_t sequential_launch(const float *P, const float *R, const float *s0, float *S, int B,
                              int T, int d, int forget, cudaStream_t st);

size_t backward_workspace_bytes(int B, int T, int d_in, int d_h);
// vl: packed ragged sequences (B = 1, T = total_T; s0 and ds0 per sequence).
cudaError_t backward_launch(const void *x, const void *Wx, int dtype, const float *P, const float *R,
                            const float *s0, const float *S, const float *dH, float *dx, float *dWx,
                            float *dR, float *db, float *ds0, int forget, int B, int T, int d_in,
                            int d_h, void *ws, cudaStream_t st, const Varlen *vl = nullptr);

// C[M][N] = sum_k A(m,k) B(k,n) (+ bias[n]) with fp32 accumulation.
// A(m,k) = A[m*sam + k*sak], B(k,n) = B[k*sbk + n*sbn]; element types as
// `dtype` (SLSTM_F32 / SLSTM_BF16) per operand.
struct GemmDesc {
    int M, N, K;
    const void *A;
    int a_dtype;
    long long sam, sak;
    const void *B;
    int b_dtype;
    long long sbk, sbn;
    const float *bias;  // [N] or null
    float *C;           // [M][N], row-major
};
cudaError_t gemm_simt(const GemmDesc &g, cudaStream_t st);

// C[M][N] = A[M][K] B[N][K]^T + bias[N] on the tcgen05 tensor cores; A and B
// bf16, K-major, K % 8 == 0, 16-byte aligned.  `error` (device word) is set
// nonzero if a bounded wait inside the kernel expires.
cudaError_t gemm_tc_bf16(const void *A, const void *Bm, const float *bias, float *C, int M, int N, int K,
                         unsigned *error, cudaStream_t st);
// General form: C = (A0 [+ A1]) B^T (+ bias).  A0, A1: [M][K] (a_mn false)
// or [K][M] (a_mn true) with row stride lda; B: [N][K] (b_mn false) or
// [K][N] (b_mn true) with row stride ldb (elements, multiples of 8); split-K
// into `splits` fp32 slices of C (C + z*M*N) when splits > 1.
cudaError_t gemm_tc_bf16_ex(const void *A0, const void *A1, int lda, bool a_mn, const void *Bm, int ldb, bool b_mn,
                            const float *bias, float *C, int M, int N, int K, int splits, unsigned *error,
                            cudaStream_t st);
// The split count gemm_tc_bf16_ex will actually use for a request of `want`.
int gemm_tc_splits(int M, int N, int K, int a_parts, int want);
// The tile shape of the tensor-core GEMMs (SLSTM_GEMM_TILES_*); returns the
// previous one, or -1 for an unknown value.
int gemm_tc_set_tiles(int tiles);
// Rows of C per work item of a split-K product (256 on SM pairs, 128 on
// single SMs; 256 columns either way) and the work items that run at once
// (clusters, or SMs).
void gemm_tc_waves(int *tile_rows, int *units);
// out[i] = sum over z in order of part[z * n + i] (split-K partial sums).
cudaError_t sum_splits(const float *part, float *out, long long n, int splits, cudaStream_t st);

// Input projection P = x Wx^T + bias (tcgen05 for bf16, CUDA cores for fp32).
size_t preact_workspace_bytes(int B, int T, int d_in, int d_h, int dtype);
cudaError_t preact_launch(const void *x, const void *Wx, int dtype, const float *bias, float *P,
                          int B, int T, int d_in, int d_h, void *ws, cudaStream_t st);

}  // namespace slstm
