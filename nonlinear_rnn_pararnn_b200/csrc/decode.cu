// Decode: one step of the diag-mix sLSTM for a batch of B rows, the input
// projection fused with the cell update ("sLSTM in this library", section
// "API notes": at T = 1 evaluation is one recurrent step; "pararnn-torch
// structure": the T = 1 decode step is replayed under CUDA graphs).
//
//   P_t[b, g, j] = sum_k W_x[g d + j, k] x_t[b, k] + bias[g, j]
//   s_t[b, :, j] = f(s_{t-1}[b, :, j], P_t[b, :, j])
//
// Four warps per feature j: its four W_x rows (gates z, i, f, o) stream once
// through 16-byte loads split over the warps' lanes and are used for every
// batch row (up to DEC_BMAX per launch), the sums are reduced across the
// lanes and warps, and lane b applies the cell to batch row b.  The step reads W_x once, so at
// decode batch sizes it is bound by the bandwidth that W_x streams from.
// s_next may be s_prev: each (row, feature) is read and then written by the
// same lane.
#include <cuda_bf16.h>

#define SLSTM_FILE_ID 6
#include "checked.cuh"
#include "common.cuh"
#include "launchers.h"

namespace slstm {
namespace {

constexpr int DEC_WPF = 4;                   // warps per feature (d_in split four ways)
constexpr int DEC_FPB = 2;                   // features per block
constexpr int DEC_WARPS = DEC_WPF * DEC_FPB;
constexpr int DEC_BMAX = 16;

SLSTM_DEVINL void load_vec(const float *p, float v[4])
{
    const float4 q = __ldg(reinterpret_cast<const float4 *>(p));
    v[0] = q.x;
    v[1] = q.y;
    v[2] = q.z;
    v[3] = q.w;
}

SLSTM_DEVINL void load_vec(const __nv_bfloat16 *p, float v[8])
{
    const uint4 q = __ldg(reinterpret_cast<const uint4 *>(p));
    const unsigned w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// Block: DEC_FPB features, DEC_WPF warps each; warp q of a feature takes the
// 16-byte pieces q, q + DEC_WPF, ... of every W_x row (interleaved over the
// lanes), the four warps' sums meet in shared memory, and lane b of the
// feature's first warp applies the cell to batch row b.
template <typename T, int FORGET, int BM>
__global__ void __launch_bounds__(DEC_WARPS * 32) decode_kernel(const T *__restrict__ x, const T *__restrict__ Wx,
                                                               const float *__restrict__ bias,
                                                               const float *__restrict__ R,
                                                               const float *s_prev, float *s_next, int B, int d_in,
                                                               int d)
{
    constexpr int VEC = 16 / (int)sizeof(T);   // elements per 16-byte load
    __shared__ float red[DEC_FPB][DEC_WPF][4][BM];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int fl = warp / DEC_WPF, q = warp % DEC_WPF;
    const int j = blockIdx.x * DEC_FPB + fl;
    const bool jv = j < d;
    const size_t dd = (size_t)d;
    float acc[4][BM];
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int b = 0; b < BM; ++b) acc[g][b] = 0.0f;
    if (jv) {
        for (int k = (q * 32 + lane) * VEC; k < d_in; k += DEC_WPF * 32 * VEC) {
            float w[4][VEC];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                if (SLSTM_IN(((size_t)g * dd + j) * d_in + k + VEC - 1, 4LL * d * d_in))
                    load_vec(Wx + ((size_t)g * dd + j) * d_in + k, w[g]);
                else
                    for (int i = 0; i < VEC; ++i) w[g][i] = 0.0f;
            }
#pragma unroll
            for (int b = 0; b < BM; ++b) {
                if (b < B && SLSTM_IN((size_t)b * d_in + k + VEC - 1, (long long)B * d_in)) {
                    float xv[VEC];
                    load_vec(x + (size_t)b * d_in + k, xv);
#pragma unroll
                    for (int g = 0; g < 4; ++g)
#pragma unroll
                        for (int i = 0; i < VEC; ++i) acc[g][b] = fmaf(w[g][i], xv[i], acc[g][b]);
                }
            }
        }
    }
    // sum over the lanes, then over the feature's warps
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int b = 0; b < BM; ++b) acc[g][b] += __shfl_xor_sync(0xffffffffu, acc[g][b], o);
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int b = 0; b < BM; ++b) red[fl][q][g][b] = acc[g][b];
    }
    __syncthreads();
    if (!jv || q != 0 || lane >= B) return;
    float p[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        float t = 0.0f;
#pragma unroll
        for (int w = 0; w < DEC_WPF; ++w) t += red[fl][w][g][lane];
        p[g] = t + __ldg(bias + g * dd + j);
    }
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    if (s_prev && SLSTM_IN(((size_t)lane * 4 + 3) * dd + j, (long long)B * 4 * d)) {
#pragma unroll
        for (int e = 0; e < 4; ++e) s[e] = s_prev[((size_t)lane * 4 + e) * dd + j];
    }
    Cell o;
    cell_eval<FORGET, false>(s[0], s[1], s[2], s[3], p[0], p[1], p[2], p[3], __ldg(R + j), __ldg(R + dd + j),
                             __ldg(R + 2 * dd + j), __ldg(R + 3 * dd + j), o);
    float *qo = s_next + (size_t)lane * 4 * dd + j;
    if (!SLSTM_PIN(qo + 3 * dd, s_next, (long long)B * 4 * d)) return;
    qo[0] = o.c;
    qo[dd] = o.n;
    qo[2 * dd] = o.m;
    qo[3 * dd] = o.h;
}

template <typename T, int FORGET>
cudaError_t decode_rows(const T *x, const T *Wx, const float *bias, const float *R, const float *s_prev,
                        float *s_next, int B, int d_in, int d, cudaStream_t st)
{
    const dim3 grid((d + DEC_FPB - 1) / DEC_FPB);
    // batch rows in slices of up to DEC_BMAX (W_x streams once per slice)
    for (int b0 = 0; b0 < B; b0 += DEC_BMAX) {
        const int nb = min(DEC_BMAX, B - b0);
        const T *xs = x + (size_t)b0 * d_in;
        const float *sp = s_prev ? s_prev + (size_t)b0 * 4 * d : nullptr;
        float *sn = s_next + (size_t)b0 * 4 * d;
        if (nb <= 4)
            decode_kernel<T, FORGET, 4><<<grid, DEC_WARPS * 32, 0, st>>>(xs, Wx, bias, R, sp, sn, nb, d_in, d);
        else if (nb <= 8)
            decode_kernel<T, FORGET, 8><<<grid, DEC_WARPS * 32, 0, st>>>(xs, Wx, bias, R, sp, sn, nb, d_in, d);
        else
            decode_kernel<T, FORGET, 16><<<grid, DEC_WARPS * 32, 0, st>>>(xs, Wx, bias, R, sp, sn, nb, d_in, d);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t decode_launch(const void *x, const void *Wx, int dtype, const float *bias, const float *R,
                          const float *s_prev, float *s_next, int forget, int B, int d_in, int d, cudaStream_t st)
{
    if (dtype == SLSTM_BF16) {
        const auto *xb = static_cast<const __nv_bfloat16 *>(x);
        const auto *wb = static_cast<const __nv_bfloat16 *>(Wx);
        return forget == SLSTM_FORGET_EXP
                   ? decode_rows<__nv_bfloat16, SLSTM_FORGET_EXP>(xb, wb, bias, R, s_prev, s_next, B, d_in, d, st)
                   : decode_rows<__nv_bfloat16, SLSTM_FORGET_SIGMOID>(xb, wb, bias, R, s_prev, s_next, B, d_in, d,
                                                                     st);
    }
    const auto *xf = static_cast<const float *>(x);
    const auto *wf = static_cast<const float *>(Wx);
    return forget == SLSTM_FORGET_EXP
               ? decode_rows<float, SLSTM_FORGET_EXP>(xf, wf, bias, R, s_prev, s_next, B, d_in, d, st)
               : decode_rows<float, SLSTM_FORGET_SIGMOID>(xf, wf, bias, R, s_prev, s_next, B, d_in, d, st);
}

}  // namespace slstm
