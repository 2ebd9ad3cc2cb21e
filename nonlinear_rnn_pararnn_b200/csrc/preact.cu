// Input projection P[b,t,g,j] = sum_k x[b,t,k] Wx[g*d_h+j, k] + bias[g,j]
// ("sLSTM in this library", section "API notes": W_x is a GEMM; summary of
// "xLSTM: Extended Long Short-Term Memory", sLSTM step: W_* x + b_*).
#include "launchers.h"

namespace slstm {

size_t preact_workspace_bytes(int B, int T, int d_in, int d_h, int dtype)
{
    (void)B;
    (void)T;
    (void)d_in;
    (void)d_h;
    (void)dtype;
    return 0;
}

cudaError_t preact_launch(const void *x, const void *Wx, int dtype, const float *bias, float *P,
                          int B, int T, int d_in, int d_h, void *ws, cudaStream_t st)
{
    (void)ws;
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
