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

#define SLSTM_FILE_ID 8
#include "checked.cuh"
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
    // the row's last element in x, u, z and (RESID) h's slot of S
    if (!SLSTM_IN((size_t)r * D + 4 * n4 - 1, (long long)M * D)) return;
    if (RESID && !SLSTM_IN(((size_t)r * 4 + 3) * D + 4 * n4 - 1, 4LL * M * D)) return;
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

// ---------------------------------------------------------------------------
// backward
// ---------------------------------------------------------------------------

// RMSNorm backward, one warp per row, for z = w v r with r = (mean(v^2) + eps)^(-1/2):
//   out = base + r w dz - r^3 v (sum_i dz_i w_i v_i) / D
// and dz is overwritten with the row's weight-gradient terms dz v r.  out may
// be base and each element of dz_c is read, then written, by the same lane.
__global__ void __launch_bounds__(NORM_ROWS * 32) norm_bwd_kernel(const float *v, const float *__restrict__ w,
                                                                  float *dz_c, const float *base, float *out, int M,
                                                                  int D, float eps)
{
    const int r = blockIdx.x * NORM_ROWS + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= M) return;
    const int n4 = D >> 2;
    if (!SLSTM_IN((size_t)r * D + 4 * n4 - 1, (long long)M * D)) return;   // the row's last element
    const float4 *vr = reinterpret_cast<const float4 *>(v + (size_t)r * D);
    float4 *dr = reinterpret_cast<float4 *>(dz_c + (size_t)r * D);
    const float4 *br = reinterpret_cast<const float4 *>(base + (size_t)r * D);
    float4 *orow = reinterpret_cast<float4 *>(out + (size_t)r * D);
    const float4 *w4 = reinterpret_cast<const float4 *>(w);
    float ss = 0.0f, sd = 0.0f;
    for (int i = lane; i < n4; i += 32) {
        const float4 a = vr[i], g = dr[i], wv = __ldg(w4 + i);
        ss = fmaf(a.x, a.x, fmaf(a.y, a.y, fmaf(a.z, a.z, fmaf(a.w, a.w, ss))));
        sd = fmaf(g.x * wv.x, a.x, fmaf(g.y * wv.y, a.y, fmaf(g.z * wv.z, a.z, fmaf(g.w * wv.w, a.w, sd))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
        sd += __shfl_xor_sync(0xffffffffu, sd, o);
    }
    const float rs = rsqrtf(ss / (float)D + eps);
    const float k3 = rs * rs * rs * sd / (float)D;
    for (int i = lane; i < n4; i += 32) {
        const float4 a = vr[i], g = dr[i], wv = __ldg(w4 + i), b = br[i];
        orow[i] = make_float4(b.x + rs * wv.x * g.x - k3 * a.x, b.y + rs * wv.y * g.y - k3 * a.y,
                              b.z + rs * wv.z * g.z - k3 * a.z, b.w + rs * wv.w * g.w - k3 * a.w);
        dr[i] = make_float4(g.x * a.x * rs, g.y * a.y * rs, g.z * a.z * rs, g.w * a.w * rs);
    }
}

// fp32 -> a pair of bf16 with v ~ hi + lo (|v - hi - lo| <= 2^-16 |v|), the
// tensor-core operand form of an fp32 matrix.
__global__ void __launch_bounds__(256) split_pair_kernel(const float *__restrict__ v, __nv_bfloat16 *__restrict__ hi,
                                                         __nv_bfloat16 *__restrict__ lo, long long n)
{
    const long long q = (long long)blockIdx.x * 256 + threadIdx.x;
    if (q >= n) return;
    const float x = v[q];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[q] = h;
    lo[q] = __float2bfloat16_rn(x - __bfloat162float(h));
}

// SwiGLU backward, one thread per (row m, hidden feature f): gv holds the
// gate/up projections in the interleaved column order (gate of f at column
// 64 (f / 32) + f % 32, up 32 columns later); da[m][f] = dL/da.  The
// gradients of the gate and up projections go out as a bf16 pair in the same
// column order (tensor-core A operands), the product a = silu(gate) up as
// bf16, the forward's own rounding of that GEMM operand.
__global__ void __launch_bounds__(256) swiglu_bwd_pair_kernel(const float *__restrict__ gv, const float *__restrict__ da,
                                                              __nv_bfloat16 *__restrict__ dgv_hi,
                                                              __nv_bfloat16 *__restrict__ dgv_lo,
                                                              __nv_bfloat16 *__restrict__ a, long long total, int F)
{
    const long long q = (long long)blockIdx.x * 256 + threadIdx.x;
    if (q >= total) return;
    const long long m = q / F;
    const int f = (int)(q - m * F);
    const long long cg = m * 2 * F + (f >> 5) * 64 + (f & 31);
    if (!SLSTM_IN(cg + 32, 2 * total)) return;   // the up column of the pair (F a multiple of 32)
    const float g = gv[cg], u = gv[cg + 32], d = da[q];
    const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
    const float silu = g * sg;
    const float dg = d * u * sg * fmaf(g, 1.0f - sg, 1.0f);
    const float du = d * silu;
    const __nv_bfloat16 hg = __float2bfloat16_rn(dg), hu = __float2bfloat16_rn(du);
    dgv_hi[cg] = hg;
    dgv_lo[cg] = __float2bfloat16_rn(dg - __bfloat162float(hg));
    dgv_hi[cg + 32] = hu;
    dgv_lo[cg + 32] = __float2bfloat16_rn(du - __bfloat162float(hu));
    a[q] = __float2bfloat16_rn(silu * u);
}

// Column sums of c (M x D) in a fixed order: chunk k of rows_per_chunk rows
// into partial[k][:], then the chunks in order.
__global__ void __launch_bounds__(256) colsum_partial_kernel(const float *__restrict__ c, int M, int D,
                                                             int rows_per_chunk, float *__restrict__ partial)
{
    const int i = blockIdx.x * 256 + threadIdx.x;
    if (i >= D) return;
    const int r0 = blockIdx.y * rows_per_chunk;
    const int r1 = min(M, r0 + rows_per_chunk);
    float acc = 0.0f;
    for (int r = r0; r < r1; ++r)
        if (SLSTM_IN((size_t)r * D + i, (long long)M * D)) acc += c[(size_t)r * D + i];
    if (SLSTM_IN((size_t)blockIdx.y * D + i, ((long long)(M + rows_per_chunk - 1) / rows_per_chunk) * D))
        partial[(size_t)blockIdx.y * D + i] = acc;
}

__global__ void __launch_bounds__(256) colsum_final_kernel(const float *__restrict__ partial, int n_chunks, int D,
                                                           float *__restrict__ out)
{
    const int i = blockIdx.x * 256 + threadIdx.x;
    if (i >= D) return;
    float acc = 0.0f;
    for (int k = 0; k < n_chunks; ++k) acc += partial[(size_t)k * D + i];
    out[i] = acc;
}

constexpr int COLSUM_ROWS = 256;

struct BlockBwdLayout {
    unsigned *err;
    __nv_bfloat16 *z1, *z2;   // (M, D) each
    float *P;                 // (M, 4D)
    float *u;                 // (M, D)
    float *gv;                // (M, 2F): gate/up
    float *da;                // (M, F): dL/da
    __nv_bfloat16 *dy_hi, *dy_lo;     // (M, D): dY as a bf16 pair
    __nv_bfloat16 *dgv_hi, *dgv_lo;   // (M, 2F): gate/up gradients as a bf16 pair
    __nv_bfloat16 *a;                 // (M, F): silu(gate) up in bf16
    float *wpart;             // split-K partial sums of the weight gradients
    float *dz2, *dz1;         // (M, D) each
    float *partial;           // (M / COLSUM_ROWS + 1, D)
    void *cell_ws;
    int splits_down, splits_gu;
};

// split-K count of a weight-gradient GEMM (M x N output, K = B*T rows, two A
// parts): the count (up to 16) whose work items fill whole waves of the
// persistent CTAs or CTA pairs (128 x 256 or 256 x 256 output tiles) best.
int block_wgrad_splits(int M, int N, int K)
{
    int rows = 128, sms = 148;
    gemm_tc_waves(&rows, &sms);
    const long long tiles = ((long long)(M + rows - 1) / rows) * ((N + 255) / 256);
    int best = 1;
    double best_eff = 0.0;
    for (int want = 1; want <= 16; ++want) {
        const int s = gemm_tc_splits(M, N, K, 2, want);
        const long long work = tiles * s;
        const double eff = (double)work / (double)(((work + sms - 1) / sms) * sms);
        if (eff > best_eff + 0.02) {
            best_eff = eff;
            best = s;
        }
    }
    return best;
}

// Byte offsets of the backward's buffers inside its workspace; `total` is
// where the cell backward's own workspace starts.
struct BlockBwdOffsets {
    size_t err, z1, z2, P, u, gv, da, dy_hi, dy_lo, dgv_hi, dgv_lo, a, wpart, dz2, dz1, partial, total;
    int splits_down, splits_gu;
};

BlockBwdOffsets block_bwd_offsets(int B, int T, int D, int F)
{
    const size_t M = (size_t)B * T;
    const size_t chunks = (M + COLSUM_ROWS - 1) / COLSUM_ROWS;
    BlockBwdOffsets o;
    o.splits_down = block_wgrad_splits(D, F, (int)M);
    o.splits_gu = block_wgrad_splits(2 * F, D, (int)M);
    const size_t wpart = (size_t)(o.splits_down > o.splits_gu ? o.splits_down : o.splits_gu) * 2 * F * D;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += al256(bytes);
        return at;
    };
    o.err = take(256);
    o.z1 = take(M * D * 2);
    o.z2 = take(M * D * 2);
    o.P = take(M * 4 * D * 4);
    o.u = take(M * D * 4);
    o.gv = take(M * 2 * F * 4);
    o.da = take(M * F * 4);
    o.dy_hi = take(M * D * 2);
    o.dy_lo = take(M * D * 2);
    o.dgv_hi = take(M * 2 * F * 2);
    o.dgv_lo = take(M * 2 * F * 2);
    o.a = take(M * F * 2);
    o.wpart = take(wpart * 4);
    o.dz2 = take(M * D * 4);
    o.dz1 = take(M * D * 4);
    o.partial = take(chunks * D * 4);
    o.total = off;
    return o;
}

BlockBwdLayout block_bwd_layout(void *ws, int B, int T, int D, int F)
{
    const BlockBwdOffsets o = block_bwd_offsets(B, T, D, F);
    char *p = static_cast<char *>(ws);
    BlockBwdLayout l;
    l.splits_down = o.splits_down;
    l.splits_gu = o.splits_gu;
    l.err = reinterpret_cast<unsigned *>(p + o.err);
    l.z1 = reinterpret_cast<__nv_bfloat16 *>(p + o.z1);
    l.z2 = reinterpret_cast<__nv_bfloat16 *>(p + o.z2);
    l.P = reinterpret_cast<float *>(p + o.P);
    l.u = reinterpret_cast<float *>(p + o.u);
    l.gv = reinterpret_cast<float *>(p + o.gv);
    l.da = reinterpret_cast<float *>(p + o.da);
    l.dy_hi = reinterpret_cast<__nv_bfloat16 *>(p + o.dy_hi);
    l.dy_lo = reinterpret_cast<__nv_bfloat16 *>(p + o.dy_lo);
    l.dgv_hi = reinterpret_cast<__nv_bfloat16 *>(p + o.dgv_hi);
    l.dgv_lo = reinterpret_cast<__nv_bfloat16 *>(p + o.dgv_lo);
    l.a = reinterpret_cast<__nv_bfloat16 *>(p + o.a);
    l.wpart = reinterpret_cast<float *>(p + o.wpart);
    l.dz2 = reinterpret_cast<float *>(p + o.dz2);
    l.dz1 = reinterpret_cast<float *>(p + o.dz1);
    l.partial = reinterpret_cast<float *>(p + o.partial);
    l.cell_ws = p + o.total;
    return l;
}

cudaError_t colsum(const float *c, int M, int D, float *partial, float *out, cudaStream_t st)
{
    const int chunks = (M + COLSUM_ROWS - 1) / COLSUM_ROWS;
    colsum_partial_kernel<<<dim3((D + 255) / 256, chunks), 256, 0, st>>>(c, M, D, COLSUM_ROWS, partial);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    colsum_final_kernel<<<(D + 255) / 256, 256, 0, st>>>(partial, chunks, D, out);
    return cudaGetLastError();
}

}  // namespace

size_t block_backward_workspace_bytes(int B, int T, int D, int F)
{
    return block_bwd_offsets(B, T, D, F).total + backward_workspace_bytes(B, T, D, D);
}

cudaError_t block_backward_launch(const float *x, const float *norm1_w, const void *Wx, const float *bias,
                                  const float *R, const float *norm2_w, const void *W_gu, const void *W_down,
                                  const float *S, const float *dY, float *dx, float *dnorm1_w, float *dWx,
                                  float *dbias, float *dR, float *dnorm2_w, float *dW_gu, float *dW_down, int forget,
                                  int B, int T, int D, int F, float eps, void *ws, cudaStream_t st)
{
    const BlockBwdLayout l = block_bwd_layout(ws, B, T, D, F);
    const int M = B * T;
    const dim3 rows((M + NORM_ROWS - 1) / NORM_ROWS);
    cudaError_t e = cudaMemsetAsync(l.err, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return e;
    // the forward's activations: z1, P = z1 W_x^T + b, u = x + h, z2
    block_norm_kernel<false><<<rows, NORM_ROWS * 32, 0, st>>>(x, nullptr, norm1_w, nullptr, l.z1, M, D, eps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = gemm_tc_bf16(l.z1, Wx, bias, l.P, M, 4 * D, D, l.err, st)) != cudaSuccess) return e;
    block_norm_kernel<true><<<rows, NORM_ROWS * 32, 0, st>>>(x, S, norm2_w, l.u, l.z2, M, D, eps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // every GEMM below runs on the tcgen05 tensor cores; fp32 operands enter
    // as a bf16 pair (hi + lo) on the A side
    // gate/up projections (interleaved columns): gv = z2 W_gu^T
    if ((e = gemm_tc_bf16(l.z2, W_gu, nullptr, l.gv, M, 2 * F, D, l.err, st)) != cudaSuccess) return e;
    // dL/da = dY W_down (W_down (D, F) is an MN-major B operand)
    const long long nmd = (long long)M * D;
    split_pair_kernel<<<(unsigned)((nmd + 255) / 256), 256, 0, st>>>(dY, l.dy_hi, l.dy_lo, nmd);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = gemm_tc_bf16_ex(l.dy_hi, l.dy_lo, D, false, W_down, F, true, nullptr, l.da, M, F, D, 1, l.err, st)) !=
        cudaSuccess)
        return e;
    const long long total = (long long)M * F;
    swiglu_bwd_pair_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(l.gv, l.da, l.dgv_hi, l.dgv_lo, l.a,
                                                                             total, F);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // dW_down = dY^T a: A = the dY pair read MN-major (B*T, D), B = a (B*T, F)
    // MN-major; split over B*T, partial sums added in order
    if ((e = gemm_tc_bf16_ex(l.dy_hi, l.dy_lo, D, true, l.a, F, true, nullptr, l.wpart, D, F, M, l.splits_down,
                             l.err, st)) != cudaSuccess)
        return e;
    if ((e = sum_splits(l.wpart, dW_down, (long long)D * F, gemm_tc_splits(D, F, M, 2, l.splits_down), st)) !=
        cudaSuccess)
        return e;
    // dz2 = dgv W_gu: A = the dgv pair (B*T, 2F) K-major, W_gu (2F, D) MN-major
    if ((e = gemm_tc_bf16_ex(l.dgv_hi, l.dgv_lo, 2 * F, false, W_gu, D, true, nullptr, l.dz2, M, D, 2 * F, 1, l.err,
                             st)) != cudaSuccess)
        return e;
    // dW_gu = dgv^T z2: A = the dgv pair read MN-major, z2 (B*T, D) MN-major
    if ((e = gemm_tc_bf16_ex(l.dgv_hi, l.dgv_lo, 2 * F, true, l.z2, D, true, nullptr, l.wpart, 2 * F, D, M,
                             l.splits_gu, l.err, st)) != cudaSuccess)
        return e;
    if ((e = sum_splits(l.wpart, dW_gu, 2LL * F * D, gemm_tc_splits(2 * F, D, M, 2, l.splits_gu), st)) !=
        cudaSuccess)
        return e;
    // du = dY + RMSNorm2 backward (into dx), dnorm2_w
    norm_bwd_kernel<<<rows, NORM_ROWS * 32, 0, st>>>(l.u, norm2_w, l.dz2, dY, dx, M, D, eps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = colsum(l.dz2, M, D, l.partial, dnorm2_w, st)) != cudaSuccess) return e;
    // the cell: dH = du; its input gradient is dz1
    if ((e = backward_launch(l.z1, Wx, SLSTM_BF16, l.P, R, nullptr, S, dx, l.dz1, dWx, dR, dbias, nullptr, forget, B,
                             T, D, D, l.cell_ws, st)) != cudaSuccess)
        return e;
    // dx = du + RMSNorm1 backward, dnorm1_w
    norm_bwd_kernel<<<rows, NORM_ROWS * 32, 0, st>>>(x, norm1_w, l.dz1, dx, dx, M, D, eps);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return colsum(l.dz1, M, D, l.partial, dnorm1_w, st);
}

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
