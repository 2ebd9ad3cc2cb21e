// CUDA-core fp32 GEMM with strided operands (fp32 or bf16 elements):
//   C[m][n] = sum_k A(m,k) B(k,n) (+ bias[n]),  fp32 accumulation.
// It serves the fp32 input projection (where tensor-core tf32 would not meet
// fp32 accuracy) and any operand layout the tensor-core path does not take.
// 128x128 output tile per CTA, 8x8 per thread, K staged through shared
// memory in slices of 16.
#include <cuda_bf16.h>

#define SLSTM_FILE_ID 9
#include "checked.cuh"
#include "common.cuh"
#include "launchers.h"

namespace slstm {
namespace {

constexpr int BM = 128, BN = 128, BK = 16;

SLSTM_DEVINL float load_elem(const void *p, int dt, long long idx)
{
    if (dt == SLSTM_BF16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[idx]);
    return static_cast<const float *>(p)[idx];
}

__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmDesc g)
{
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * BM;
    const int n0 = blockIdx.x * BN;
    const int tm = (tid / 16) * 8;  // 16 x 16 threads, 8 x 8 outputs each
    const int tn = (tid % 16) * 8;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int jn = 0; jn < 8; ++jn) acc[i][jn] = 0.f;

    const bool a_m_contig = (g.sam == 1);
    const bool b_n_contig = (g.sbn == 1);
    // extents the strides span (checked build)
    [[maybe_unused]] const long long n_a = (long long)(g.M - 1) * g.sam + (long long)(g.K - 1) * g.sak + 1;
    [[maybe_unused]] const long long n_b = (long long)(g.K - 1) * g.sbk + (long long)(g.N - 1) * g.sbn + 1;
    for (int k0 = 0; k0 < g.K; k0 += BK) {
        // A tile: BM x BK = 2048 elements, 8 per thread; walk the contiguous
        // dimension across consecutive threads.
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int e = r * 256 + tid;
            int mm, kk;
            if (a_m_contig) {
                mm = e % BM;
                kk = e / BM;
            } else {
                kk = e % BK;
                mm = e / BK;
            }
            const int m = m0 + mm, k = k0 + kk;
            float v = 0.f;
            if (m < g.M && k < g.K && SLSTM_IN((long long)m * g.sam + (long long)k * g.sak, n_a))
                v = load_elem(g.A, g.a_dtype, (long long)m * g.sam + (long long)k * g.sak);
            As[kk][mm] = v;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int e = r * 256 + tid;
            int nn, kk;
            if (b_n_contig) {
                nn = e % BN;
                kk = e / BN;
            } else {
                kk = e % BK;
                nn = e / BK;
            }
            const int n = n0 + nn, k = k0 + kk;
            float v = 0.f;
            if (n < g.N && k < g.K && SLSTM_IN((long long)k * g.sbk + (long long)n * g.sbn, n_b))
                v = load_elem(g.B, g.b_dtype, (long long)k * g.sbk + (long long)n * g.sbn);
            Bs[kk][nn] = v;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float av[8], bv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) av[i] = As[kk][tm + i];
#pragma unroll
            for (int i = 0; i < 8; ++i) bv[i] = Bs[kk][tn + i];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int jn = 0; jn < 8; ++jn) acc[i][jn] = fmaf(av[i], bv[jn], acc[i][jn]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int m = m0 + tm + i;
        if (m >= g.M) continue;
#pragma unroll
        for (int jn = 0; jn < 8; ++jn) {
            const int n = n0 + tn + jn;
            if (n >= g.N) continue;
            float v = acc[i][jn];
            if (g.bias) v += g.bias[n];
            if (SLSTM_IN((size_t)m * g.N + n, (long long)g.M * g.N)) g.C[(size_t)m * g.N + n] = v;
        }
    }
}

}  // namespace

cudaError_t gemm_simt(const GemmDesc &g, cudaStream_t st)
{
    const dim3 grid((g.N + BN - 1) / BN, (g.M + BM - 1) / BM);
    if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
    gemm_simt_kernel<<<grid, 256, 0, st>>>(g);
    return cudaGetLastError();
}

}  // namespace slstm
