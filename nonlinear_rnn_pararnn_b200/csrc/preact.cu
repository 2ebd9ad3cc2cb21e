// Input projection P[b,t,g,j] = sum_k x[b,t,k] Wx[g*d_h+j, k] + bias[g,j]
// ("sLSTM in this library", section "API notes": W_x is a GEMM; summary of
// "xLSTM: Extended Long Short-Term Memory", sLSTM step: W_* x + b_*).
// bf16 operands run on the tcgen05 tensor cores (gemm_tc.cu); fp32 operands
// run the exact fp32 CUDA-core GEMM (tf32 tensor cores would round the
// operands to 10 mantissa bits).
#include "launchers.h"

namespace slstm {

size_t preact_workspace_bytes(int B, int T, int d_in, int d_h, int dtype)
{
    (void)B;
    (void)T;
    (void)d_in;
    (void)d_h;
    return dtype == SLSTM_BF16 ? 256 : 0;   // the tensor-core GEMM's error word
}

cudaError_t preact_launch(const void *x, const void *Wx, int dtype, const float *bias, float *P,
                          int B, int T, int d_in, int d_h, void *ws, cudaStream_t st)
{
    if (dtype == SLSTM_BF16) {
        unsigned *err = static_cast<unsigned *>(ws);
        const cudaError_t e = cudaMemsetAsync(err, 0, sizeof(unsigned), st);
        if (e != cudaSuccess) return e;
        return gemm_tc_bf16(x, Wx, bias, P, B * T, 4 * d_h, d_in, err, st);
    }
    GemmDesc g;
    g.M = B * T;
    g.N = 4 * d_h;
    g.K = d_in;
    g.A = x;
    g.a_dtype = dtype;
    g.sam = d_in;
    g.sak = 1;
    g.B = Wx;
    g.b_dtype = dtype;
    g.sbk = 1;
    g.sbn = d_in;
    g.bias = bias;
    g.C = P;
    return gemm_simt(g, st);
}

}  // namespace slstm
