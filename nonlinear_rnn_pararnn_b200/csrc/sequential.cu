// Sequential stepping of the diag-mix sLSTM: S_t = f(S_{t-1}, P_t), one
// thread per (batch row, feature) walking time ("sLSTM in this library",
// section "API notes": evaluation runs the sequential step; at T = 1 it is
// one recurrent-step launch while W_x stays a GEMM).
#define SLSTM_FILE_ID 4
#include "checked.cuh"
#include "common.cuh"
#include "launchers.h"

namespace slstm {
namespace {

template <int FORGET>
__global__ void __launch_bounds__(128) sequential_kernel(const float *__restrict__ P,
                                                         const float *__restrict__ R,
                                                         const float *__restrict__ s0,
                                                         float *__restrict__ S, int T, int d)
{
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    const int b = blockIdx.y;
    if (j >= d) return;
    const size_t dd = (size_t)d;
    // extents (checked build): P and S (B, T, 4, d), s0 (B, 4, d), R (4, d)
    [[maybe_unused]] const long long n_ps = (long long)gridDim.y * T * 4 * d;
    [[maybe_unused]] const long long n_s0 = (long long)gridDim.y * 4 * d;
    if (!SLSTM_IN(3 * dd + j, 4LL * d)) return;
    const float rz = R[j], ri = R[dd + j], rf = R[2 * dd + j], ro = R[3 * dd + j];
    float c = 0.f, n = 0.f, m = 0.f, h = 0.f;
    if (s0 && SLSTM_IN((size_t)b * 4 * dd + 3 * dd + j, n_s0)) {
        const float *p = s0 + (size_t)b * 4 * dd + j;
        c = p[0];
        n = p[dd];
        m = p[2 * dd];
        h = p[3 * dd];
    }
    const float *pp = P + (size_t)b * T * 4 * dd + j;
    float *ps = S + (size_t)b * T * 4 * dd + j;
    // one step ahead prefetch of P keeps a load in flight while the step computes
    float nz = 0.f, ni = 0.f, nf = 0.f, no = 0.f;
    if (SLSTM_PIN(pp + 3 * dd, P, n_ps)) {
        nz = __ldg(pp);
        ni = __ldg(pp + dd);
        nf = __ldg(pp + 2 * dd);
        no = __ldg(pp + 3 * dd);
    }
    for (int t = 0; t < T; ++t) {
        const float pz = nz, pi = ni, pf = nf, po = no;
        if (t + 1 < T && SLSTM_PIN(pp + (size_t)(t + 1) * 4 * dd + 3 * dd, P, n_ps)) {
            const float *q = pp + (size_t)(t + 1) * 4 * dd;
            nz = __ldg(q);
            ni = __ldg(q + dd);
            nf = __ldg(q + 2 * dd);
            no = __ldg(q + 3 * dd);
        }
        Cell o;
        cell_eval<FORGET, false>(c, n, m, h, pz, pi, pf, po, rz, ri, rf, ro, o);
        c = o.c;
        n = o.n;
        m = o.m;
        h = o.h;
        float *q = ps + (size_t)t * 4 * dd;
        if (!SLSTM_PIN(q + 3 * dd, S, n_ps)) continue;
        q[0] = c;
        q[dd] = n;
        q[2 * dd] = m;
        q[3 * dd] = h;
    }
}

}  // namespace

cudaError_t sequential_launch(const float *P, const float *R, const float *s0, float *S, int B,
                              int T, int d, int forget, cudaStream_t st)
{
    const dim3 block(128);
    const dim3 grid((d + 127) / 128, B);
    if (forget == SLSTM_FORGET_EXP)
        sequential_kernel<SLSTM_FORGET_EXP><<<grid, block, 0, st>>>(P, R, s0, S, T, d);
    else
        sequential_kernel<SLSTM_FORGET_SIGMOID><<<grid, block, 0, st>>>(P, R, s0, S, T, d);
    return cudaGetLastError();
}

}  // namespace slstm
