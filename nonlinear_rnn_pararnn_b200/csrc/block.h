// The trunk layer (csrc/block.cu) and the GEMM epilogue variants it uses
// (csrc/gemm_tc.cu).  Arguments validated by the caller, as in launchers.h.
#pragma once

#include <cuda_bf16.h>

#include "launchers.h"

namespace slstm {

// Epilogue variants of the K-major tcgen05 GEMM (no split-K, no bias):
//   GEMM_EPI_SWIGLU    B's rows come in blocks of 64: 32 gate rows, then the
//                      32 up rows of the same features; Cb[M][N/2] (bf16) =
//                      silu(gate) * up.  N % 64 == 0.
//   GEMM_EPI_RESIDUAL  C[M][N] = A B^T + res[M][N] (res may be C).
constexpr int GEMM_EPI_STORE = 0;
constexpr int GEMM_EPI_SWIGLU = 1;
constexpr int GEMM_EPI_RESIDUAL = 2;
cudaError_t gemm_tc_bf16_epi(const void *A, const void *Bm, float *C, __nv_bfloat16 *Cb, const float *res, int M,
                             int N, int K, int epi, unsigned *error, cudaStream_t st);

// RMSNorm -> cell -> residual -> RMSNorm -> SwiGLU -> residual, forward.
size_t block_workspace_bytes(int B, int T, int D, int F);
cudaError_t block_forward_launch(const float *x, const float *norm1_w, const void *Wx, const float *bias,
                                 const float *R, const float *norm2_w, const void *W_gu, const void *W_down, float *y,
                                 float *S, const slstm_newton_config &cfg, slstm_newton_stats *stats, int B, int T,
                                 int D, int F, float eps, void *ws, cudaStream_t st);

// Gradients of sum(dY * y) for the forward above (recomputes its activations
// from x and the forward's S).
size_t block_backward_workspace_bytes(int B, int T, int D, int F);
cudaError_t block_backward_launch(const float *x, const float *norm1_w, const void *Wx, const float *bias,
                                  const float *R, const float *norm2_w, const void *W_gu, const void *W_down,
                                  const float *S, const float *dY, float *dx, float *dnorm1_w, float *dWx,
                                  float *dbias, float *dR, float *dnorm2_w, float *dW_gu, float *dW_down, int forget,
                                  int B, int T, int D, int F, float eps, void *ws, cudaStream_t st);

}  // namespace slstm
