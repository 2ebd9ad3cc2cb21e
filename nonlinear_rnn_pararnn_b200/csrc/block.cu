// The trunk layer, forward ("sLSTM in this library", section "Stacking":
// RMSNorm -> ParaRNN(ParaSLSTM) -> residual -> RMSNorm -> SwiGLU -> residual),
// for x (B, T, D) in fp32 with bf16 weights:
//
//   z1 = RMSNorm(x) w1                       block_norm_kernel<false>   -> bf16
//   P  = z1 W_x^T + b                        tcgen05 GEMM (bias epilogue)
//   S  = Newton solve of the cell on P       newton_iter launches
//   u  = x + h,  z2 = RMSNorm(u) w2          block_norm_kernel<true>    -> u fp32 (in y), z2 bf16
//   a  = silu(z2 W_gate^T) * (z2 W_up^T)     tcgen05 GEMM, SwiGLU epilogue -> bf16
//   y  = u + a W_down^T                      tcgen05 GEMM, residual epilogue (in place on y)
//
// RMSNorm(v) = v / sqrt(mean(v^2) + eps) over the model axis (the plain form;
// the section names the norm only).  The gate and up projections are one
// GEMM whose weight rows come in blocks of 64 (32 gate rows, then the 32 up
// rows of the same features), so that the epilogue holds both halves of a
// feature in one thread and the (M, 2F) product never reaches memory; the
// down projection adds the residual in its epilogue.  The cell starts from the
// zero state (d_in = d_h = D).
#include <cuda_bf16.h>

#include "common.cuh"
#include "block.h"
#include "launchers.h"

namespace slstm {
namespace {

size_t al256(size_t v) { return (v + 255) & ~(size_t)255; }

constexpr int NORM_ROWS = 8;   // rows (warps) per block

// One warp per row.  RESID: v = x + h (h = slot 3 of S), stored to u; else v = x.
// z = bf16(v / sqrt(mean(v^2) + eps) * w).  D % 4 == 0, 16-byte aligned rows.
template <bool RESID>
__global__ void __launch_bounds__(NORM_ROWS * 32) block_norm_kernel(const float *x, const float *S,
                                                                    const float *__restrict__ w, float *u,
                                                                    __nv_bfloat16 *__restrict__ z, int M, int D,
                                                                    float eps)
{
    const int r = blockIdx.x * NORM_ROWS + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= M) return;
    const int n4 = D >> 2;
    const float4 *xr = reinterpret_cast<const float4 *>(x + (size_t)r * D);
    float4 *ur = RESID ? reinterpret_cast<float4 *>(u + (size_t)r * D) : nullptr;
    const float4 *hr = RESID ? reinterpret_cast<const float4 *>(S + ((size_t)r * 4 + 3) * D) : nullptr;
    float ss = 0.0f;
    for (int i = lane; i < n4; i += 32) {
        // u may be x (in place): plain loads, each element read before this lane writes it
        float4 v = RESID ? xr[i] : __ldg(xr + i);
        if (RESID) {
            const float4 h = hr[i];
            v.x += h.x;
            v.y += h.y;
            v.z += h.z;
            v.w += h.w;
            ur[i] = v;
        }
        ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rs = rsqrtf(ss / (float)D + eps);
    const float4 *w4 = reinterpret_cast<const float4 *>(w);
    uint2 *zr = reinterpret_cast<uint2 *>(z + (size_t)r * D);
    for (int i = lane; i < n4; i += 32) {
        const float4 v = RESID ? ur[i] : __ldg(xr + i);   // u[i] was written by this lane
        const float4 wv = __ldg(w4 + i);
        const __nv_bfloat162 p0 = __floats2bfloat162_rn(v.x * rs * wv.x, v.y * rs * wv.y);
        const __nv_bfloat162 p1 = __floats2bfloat162_rn(v.z * rs * wv.z, v.w * rs * wv.w);
        zr[i] = make_uint2(*reinterpret_cast<const unsigned *>(&p0), *reinterpret_cast<const unsigned *>(&p1));
    }
}

struct BlockLayout {
    unsigned *err;          // the GEMMs' bounded-wait flag
    __nv_bfloat16 *z;       // (M, D): z1, later z2
    float *P;               // (M, 4D) pre-activations; its space later holds a (M, F) bf16
    void *newton_ws;
};

BlockLayout block_layout(void *ws, int B, int T, int D, int F)
{
    const size_t M = (size_t)B * T;
    const size_t p_bytes = al256(M * 4 * D * 4) > al256(M * F * 2) ? al256(M * 4 * D * 4) : al256(M * F * 2);
    char *base = static_cast<char *>(ws);
    BlockLayout l;
    l.err = reinterpret_cast<unsigned *>(base);
    l.z = reinterpret_cast<__nv_bfloat16 *>(base + 256);
    l.P = reinterpret_cast<float *>(base + 256 + al256(M * D * 2));
    l.newton_ws = base + 256 + al256(M * D * 2) + p_bytes;
    return l;
}

}  // namespace

size_t block_workspace_bytes(int B, int T, int D, int F)
{
    const size_t M = (size_t)B * T;
    const size_t p_bytes = al256(M * 4 * D * 4) > al256(M * F * 2) ? al256(M * 4 * D * 4) : al256(M * F * 2);
    return 256 + al256(M * D * 2) + p_bytes + newton_workspace_bytes(B, T, D);
}

cudaError_t block_forward_launch(const float *x, const float *norm1_w, const void *Wx, const float *bias,
                                 const float *R, const float *norm2_w, const void *W_gu, const void *W_down, float *y,
                                 float *S, const slstm_newton_config &cfg, slstm_newton_stats *stats, int B, int T,
                                 int D, int F, float eps, void *ws, cudaStream_t st)
{
    const BlockLayout l = block_layout(ws, B, T, D, F);
    const int M = B * T;
    const dim3 grid((M + NORM_ROWS - 1) / NORM_ROWS);
    cudaError_t e = cudaMemsetAsync(l.err, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return e;
    block_norm_kernel<false><<<grid, NORM_ROWS * 32, 0, st>>>(x, nullptr, norm1_w, nullptr, l.z, M, D, eps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = gemm_tc_bf16(l.z, Wx, bias, l.P, M, 4 * D, D, l.err, st)) != cudaSuccess) return e;
    if ((e = newton_forward(l.P, R, nullptr, S, cfg, stats, B, T, D, l.newton_ws, st)) != cudaSuccess) return e;
    block_norm_kernel<true><<<grid, NORM_ROWS * 32, 0, st>>>(x, S, norm2_w, y, l.z, M, D, eps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    __nv_bfloat16 *a = reinterpret_cast<__nv_bfloat16 *>(l.P);
    if ((e = gemm_tc_bf16_epi(l.z, W_gu, nullptr, a, nullptr, M, 2 * F, D, GEMM_EPI_SWIGLU, l.err, st)) !=
        cudaSuccess)
        return e;
    return gemm_tc_bf16_epi(a, W_down, y, nullptr, y, M, D, F, GEMM_EPI_RESIDUAL, l.err, st);
}

}  // namespace slstm
