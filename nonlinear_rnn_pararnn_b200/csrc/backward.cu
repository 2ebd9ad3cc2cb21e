// Backward pass of the Newton-solved diag-mix sLSTM ("sLSTM in this
// library", section "Backward": one reverse associative scan of J^T, then a
// packed cell VJP for the gradients of R and W_x).
//
// Fused adjoint + VJP kernel, tiles in reverse time order:
//   lambda_t = e_h dH_t + J_{t+1}^T lambda_{t+1}   (J recomputed from S_t, P_{t+1})
//   dP_t     = G_t^T lambda_t,  G_t = d s_t / d a_t (recomputed from S_{t-1}, P_t)
//   dR      += dP_t * h_{t-1},  db += dP_t   (per-tile partials, reduced after)
//   ds0      = J_0^T lambda_0
// then dx = dP W_x and dW_x = dP^T x.
#include <cuda_bf16.h>

#include "launchers.h"
#include "lookback.cuh"

namespace slstm {
namespace {

constexpr int NW = 8;
constexpr int L = 4;
constexpr int TT = NW * L;

struct BwdArgs {
    const float *P;
    const float *R;
    const float *s0;
    const float *S;
    const float *dH;
    float *dP;        // (B, T, 4, d) fp32, when the GEMMs run on CUDA cores
    // bf16 pair dP ~ hi + lo (|dP - hi - lo| <= 2^-18 |dP|) for the tensor-core
    // GEMMs, stored transposed: (4d, ldT) with ldT = B*T rounded up to 8
    __nv_bfloat16 *dpt_hi, *dpt_lo;
    long long ldT;
    float *partial;   // [n_tiles][8][32]  dR (4) then db (4)
    float *ds0;       // (B, 4, d) or null
    unsigned *ticket;
    CarryArgs ca;
    int T, d, groups_per_row, n_tiles, vec16;
};

// Shared memory of one CTA.  A tile covers steps t in [t_lo, t_hi] with
// t_hi = T-1-32c and t_lo = t_hi-31 (chunk c in reverse time order); it
// needs S at t_lo-1 .. t_hi, P at t_lo .. t_hi+1 and dH at t_lo .. t_hi.
struct BwdSmem {
    float S[2][TT + 1][4][32];   // row r <-> t = t_lo - 1 + r
    float P[2][TT + 1][4][32];   // row r <-> t = t_lo + r
    float dH[2][TT][32];         // row r <-> t = t_lo + r
    union {
        float agg[NW][20][32];
        __nv_bfloat16 dpt[2][4][32][TT + 2];   // transposed staging of the dP pair
    } u;
    float cin[NW][4][32];
    float part[NW][8][32];
    unsigned tick[2];
};

SLSTM_DEVINL void split_bf16(float v, __nv_bfloat16 &hi, __nv_bfloat16 &lo)
{
    hi = __float2bfloat16_rn(v);
    lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

// Copies of one tile's S, P and dH rows into stage `st`; rows outside [0, T)
// and features past d arrive as zeros.
SLSTM_DEVINL void bwd_prefetch(const BwdArgs &a, BwdSmem &sm, int st, unsigned ticket)
{
    if (ticket >= (unsigned)a.n_tiles) return;
    const int G = a.ca.n_groups;
    const int chunk = (int)(ticket / (unsigned)G);
    const int grp = (int)(ticket % (unsigned)G);
    const int b = grp / a.groups_per_row;
    const int j0 = (grp % a.groups_per_row) * 32;
    const int t_lo = a.T - (chunk + 1) * TT;
    const size_t d = (size_t)a.d;
    const size_t row0 = (size_t)b * a.T;
    const int T = a.T;
    constexpr int RS = (TT + 1) * 4;           // (row, slot) pairs of S and of P
    if (a.vec16) {
        // thread (q, c) copies 16-byte chunk c of (row, slot) pairs q, q+32, ...
        const int c = threadIdx.x & 7, q = threadIdx.x >> 3;
        const int jj = j0 + 4 * c;
        const int fbytes = jj < a.d ? 4 * min(4, a.d - jj) : 0;
#pragma unroll
        for (int k = 0; k < (RS + 31) / 32; ++k) {
            const int rs = q + 32 * k;
            if (rs < RS) {
                const int r = rs >> 2, slot = rs & 3;
                const int tS = t_lo - 1 + r, tP = t_lo + r;   // S row r <-> t_lo-1+r, P row r <-> t_lo+r
                const int bS = (tS >= 0 && tS < T) ? fbytes : 0;
                const int bP = (tP >= 0 && tP < T) ? fbytes : 0;
                cp_async16(&sm.S[st][r][slot][4 * c], bS ? a.S + ((row0 + tS) * 4 + slot) * d + jj : a.S, bS);
                cp_async16(&sm.P[st][r][slot][4 * c], bP ? a.P + ((row0 + tP) * 4 + slot) * d + jj : a.P, bP);
            }
        }
        const int t = t_lo + q;   // dH row q
        const int bH = (t >= 0 && t < T) ? fbytes : 0;
        cp_async16(&sm.dH[st][q][4 * c], bH ? a.dH + (row0 + t) * d + jj : a.dH, bH);
    } else {
        // 4-byte copies, lane = feature, warp w takes every 8th row
        const int jl = threadIdx.x & 31, w = threadIdx.x >> 5;
        const bool fj = j0 + jl < a.d;
        const size_t jj = (size_t)j0 + jl;
        for (int rs = w; rs < RS; rs += NW) {
            const int r = rs >> 2, slot = rs & 3;
            const int tS = t_lo - 1 + r, tP = t_lo + r;
            const int bS = (fj && tS >= 0 && tS < T) ? 4 : 0;
            const int bP = (fj && tP >= 0 && tP < T) ? 4 : 0;
            cp_async4(&sm.S[st][r][slot][jl], bS ? a.S + ((row0 + tS) * 4 + slot) * d + jj : a.S, bS);
            cp_async4(&sm.P[st][r][slot][jl], bP ? a.P + ((row0 + tP) * 4 + slot) * d + jj : a.P, bP);
        }
        for (int r = w; r < TT; r += NW) {
            const int t = t_lo + r;
            const int bH = (fj && t >= 0 && t < T) ? 4 : 0;
            cp_async4(&sm.dH[st][r][jl], bH ? a.dH + (row0 + t) * d + jj : a.dH, bH);
        }
    }
}

template <int FORGET, bool BF16OUT>
__global__ void __launch_bounds__(NW * 32, 2) adjoint_vjp_kernel(BwdArgs a)
{
    extern __shared__ float4 smem_f4[];
    BwdSmem &sm = *reinterpret_cast<BwdSmem *>(smem_f4);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int G = a.ca.n_groups;
    const int T = a.T;
    const size_t d = (size_t)a.d;

    if (threadIdx.x == 0) {
        sm.tick[0] = atomicAdd(a.ticket, 1u);
        sm.tick[1] = atomicAdd(a.ticket, 1u);
    }
    __syncthreads();
    unsigned cur = sm.tick[0];
    unsigned nxt = sm.tick[1];
    int st = 0;
    bwd_prefetch(a, sm, 0, cur);
    cp_async_commit();

    while (cur < (unsigned)a.n_tiles) {
        unsigned after = 0;
        if (threadIdx.x == 0) after = atomicAdd(a.ticket, 1u);
        bwd_prefetch(a, sm, st ^ 1, nxt);
        cp_async_commit();
        cp_async_wait_prev();
        __syncthreads();

        const unsigned ticket = cur;
        const int chunk = (int)(ticket / (unsigned)G);
        const int grp = (int)(ticket % (unsigned)G);
        const int b = grp / a.groups_per_row;
        const int j = (grp % a.groups_per_row) * 32 + lane;
        const bool jv = j < a.d;
        const size_t jj = jv ? (size_t)j : 0;
        const size_t row0 = (size_t)b * T;
        const int t_lo = T - (chunk + 1) * TT;

        float rz = 0.f, ri = 0.f, rf = 0.f, ro = 0.f;
        if (jv) {
            rz = __ldg(a.R + jj);
            ri = __ldg(a.R + d + jj);
            rf = __ldg(a.R + 2 * d + jj);
            ro = __ldg(a.R + 3 * d + jj);
        }

        // ---- walk A: fold lambda -> J_{t+1}^T lambda + e_h dH_t, t descending ----
        Cell Jn[L];   // J_{t+1} of each step
        Aff agg;
        aff_identity(agg);
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int rl = TT - 1 - (warp * L + i);   // t - t_lo
            const int t = t_lo + rl;
            cell_identity(Jn[i]);
            float r[4] = {0.f, 0.f, 0.f, 0.f};
            if (t >= 0) {
                r[3] = sm.dH[st][rl][lane];
                if (t + 1 < T)
                    cell_eval<FORGET, true>(sm.S[st][rl + 1][0][lane], sm.S[st][rl + 1][1][lane],
                                            sm.S[st][rl + 1][2][lane], sm.S[st][rl + 1][3][lane],
                                            sm.P[st][rl + 1][0][lane], sm.P[st][rl + 1][1][lane],
                                            sm.P[st][rl + 1][2][lane], sm.P[st][rl + 1][3][lane], rz, ri, rf, ro, Jn[i]);
            }
            fold_jacT(agg, Jn[i], r);
        }
        store_aff_smem(sm.u.agg, warp, lane, agg);
        __syncthreads();
        if (warp == 0) {
            const float zero[4] = {0.f, 0.f, 0.f, 0.f};
            tile_carry_serial<NW>(a.ca, sm.u.agg, sm.cin, ticket, chunk, grp, zero, false);
        }
        __syncthreads();   // sm.u.agg is dead from here on; sm.u.dpt takes its place

        // ---- walk B: lambda_t, then dP_t = G_t^T lambda_t ----
        float lam[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) lam[e] = sm.cin[warp][e][lane];
        float dr[4] = {0.f, 0.f, 0.f, 0.f}, dbs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int rl = TT - 1 - (warp * L + i);
            const int t = t_lo + rl;
            if (t >= 0) {
                jacT_mul(Jn[i], lam[0], lam[1], lam[2], lam[3]);
                lam[3] += sm.dH[st][rl][lane];
                float prev[4];
                if (t == 0) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) prev[e] = (a.s0 && jv) ? __ldg(a.s0 + ((size_t)b * 4 + e) * d + jj) : 0.f;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) prev[e] = sm.S[st][rl][e][lane];
                }
                Cell c;
                CellG g;
                cell_eval<FORGET, true, true>(prev[0], prev[1], prev[2], prev[3], sm.P[st][rl][0][lane],
                                              sm.P[st][rl][1][lane], sm.P[st][rl][2][lane], sm.P[st][rl][3][lane], rz,
                                              ri, rf, ro, c, &g);
                const float dz = fmaf(g.gcz, lam[0], g.ghz * lam[3]);
                const float di = fmaf(g.gci, lam[0], fmaf(g.gni, lam[1], fmaf(g.gmi, lam[2], g.ghi * lam[3])));
                const float df = fmaf(g.gcf, lam[0], fmaf(g.gnf, lam[1], fmaf(g.gmf, lam[2], g.ghf * lam[3])));
                const float dq = g.gho * lam[3];
                if (BF16OUT) {
                    const float dv[4] = {dz, di, df, dq};
#pragma unroll
                    for (int gi = 0; gi < 4; ++gi) {
                        __nv_bfloat16 hi, lo;
                        split_bf16(dv[gi], hi, lo);
                        sm.u.dpt[0][gi][lane][rl] = hi;
                        sm.u.dpt[1][gi][lane][rl] = lo;
                    }
                } else if (jv) {
                    float *pd = a.dP + (row0 + t) * 4 * d + jj;
                    pd[0] = dz;
                    pd[d] = di;
                    pd[2 * d] = df;
                    pd[3 * d] = dq;
                }
                const float hp = prev[3];
                dr[0] = fmaf(dz, hp, dr[0]);
                dr[1] = fmaf(di, hp, dr[1]);
                dr[2] = fmaf(df, hp, dr[2]);
                dr[3] = fmaf(dq, hp, dr[3]);
                dbs[0] += dz;
                dbs[1] += di;
                dbs[2] += df;
                dbs[3] += dq;
                if (t == 0 && a.ds0 && jv) {
                    float v0 = lam[0], v1 = lam[1], v2 = lam[2], v3 = lam[3];
                    jacT_mul(c, v0, v1, v2, v3);
                    float *q = a.ds0 + (size_t)b * 4 * d + jj;
                    q[0] = v0;
                    q[d] = v1;
                    q[2 * d] = v2;
                    q[3 * d] = v3;
                }
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sm.part[warp][e][lane] = jv ? dr[e] : 0.f;
            sm.part[warp][4 + e][lane] = jv ? dbs[e] : 0.f;
        }
        __syncthreads();
        {
            // 256 threads: thread (e, lane) sums entry e over the warps
            const int e = threadIdx.x >> 5;   // 0..7
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) acc += sm.part[w][e][lane];
            a.partial[((size_t)ticket * 8 + e) * 32 + lane] = acc;
        }
        if (BF16OUT) {
            // rows (g, j) of the transposed pair: up to 32 consecutive steps each
            const int tl = threadIdx.x & 31;
            const int t = t_lo + tl;
            const int j0 = (grp % a.groups_per_row) * 32;
            for (int r = threadIdx.x >> 5; r < 2 * 4 * 32; r += NW) {
                const int part = r >> 7;
                const int gi = (r >> 5) & 3;
                const int jl = r & 31;
                if (t >= 0 && j0 + jl < a.d) {
                    __nv_bfloat16 *dst = part ? a.dpt_lo : a.dpt_hi;
                    dst[((size_t)gi * d + j0 + jl) * a.ldT + row0 + t] = sm.u.dpt[part][gi][jl][tl];
                }
            }
        }
        if (threadIdx.x == 0) sm.tick[0] = after;
        __syncthreads();
        cur = nxt;
        nxt = sm.tick[0];
        st ^= 1;
    }
    cp_async_wait_all();
}

// out[i] = sum_z part[z][i], z in order (split-K partial sums).
__global__ void sum_splits_kernel(const float *__restrict__ part, float *__restrict__ out, long long n, int splits)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float acc = 0.0f;
    for (int z = 0; z < splits; ++z) acc += part[(size_t)z * n + i];
    out[i] = acc;
}

// dR[g][j] and db[g][j]: sum of the per-tile partials over chunks and batch
// rows, in a fixed order, accumulated in fp64.
// One block per (entry e, group of 32 features); warp w sums the (chunk, b)
// terms w, w+8, ... for its lane, then the 8 warp sums are added in order.
__global__ void __launch_bounds__(256) reduce_partials_kernel(const float *__restrict__ partial, float *__restrict__ dR,
                                                              float *__restrict__ db, int B, int n_chunks,
                                                              int groups_per_row, int d)
{
    __shared__ double s_sum[8][32];
    const int e = blockIdx.y;              // 0..7
    const int jb = blockIdx.x;             // feature group
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int G = B * groups_per_row;
    const int terms = n_chunks * B;
    double acc = 0.0;
    for (int q = warp; q < terms; q += 8) {
        const int c = q / B, b = q % B;
        const size_t ticket = (size_t)c * G + (size_t)b * groups_per_row + jb;
        acc += partial[(ticket * 8 + e) * 32 + lane];
    }
    s_sum[warp][lane] = acc;
    __syncthreads();
    if (warp == 0) {
        double t = 0.0;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += s_sum[w][lane];
        const int j = jb * 32 + lane;
        if (j < d) {
            if (e < 4)
                dR[(size_t)e * d + j] = (float)t;
            else
                db[(size_t)(e - 4) * d + j] = (float)t;
        }
    }
}

int sm_count_bwd()
{
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 148;
    }
    return n;
}

template <int FORGET, bool BF16OUT>
cudaError_t launch_adjoint(const BwdArgs &a, cudaStream_t st)
{
    auto kern = adjoint_vjp_kernel<FORGET, BF16OUT>;
    static int blocks_per_sm = 0;
    if (blocks_per_sm == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(BwdSmem));
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, kern, NW * 32, sizeof(BwdSmem));
        if (e != cudaSuccess) return e;
        if (blocks_per_sm < 1) blocks_per_sm = 1;
    }
    const int grid = min(a.n_tiles, sm_count_bwd() * blocks_per_sm);
    kern<<<grid, NW * 32, sizeof(BwdSmem), st>>>(a);
    return cudaGetLastError();
}

struct Layout {
    size_t ticket, flags, incw, agg, partial, dP, dpt, wpart, err, total;
    int groups_per_row, n_groups, n_chunks, n_tiles, splits;
    long long n, ldT, ld4;
};

long long round8(long long v) { return (v + 7) & ~7LL; }

// split-K count of the W_x-gradient GEMM: enough CTAs for two per SM
int wgrad_splits(int B, int T, int d_in, int d_h)
{
    const long long tiles = ((4LL * d_h + 127) / 128) * ((d_in + 255) / 256);
    int want = (int)((296 + tiles - 1) / tiles);
    if (want > 16) want = 16;
    return gemm_tc_splits(4 * d_h, d_in, B * T, 2, want);
}

Layout layout(int B, int T, int d_in, int d_h)
{
    Layout l;
    l.groups_per_row = (d_h + 31) / 32;
    l.n_groups = B * l.groups_per_row;
    l.n_chunks = (T + TT - 1) / TT;
    l.n_tiles = l.n_groups * l.n_chunks;
    l.n = (long long)B * T * 4 * d_h;
    l.ldT = round8((long long)B * T);
    l.ld4 = round8(4LL * d_h);
    l.splits = wgrad_splits(B, T, d_in, d_h);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~(size_t)255;
        return at;
    };
    l.ticket = take(256);
    l.flags = take(sizeof(unsigned) * (size_t)l.n_tiles);
    l.incw = take(sizeof(unsigned long long) * 4 * 32 * (size_t)l.n_tiles);
    l.agg = take(sizeof(float) * 20 * 32 * (size_t)l.n_tiles);
    l.partial = take(sizeof(float) * 8 * 32 * (size_t)l.n_tiles);
    // fp32 dP for the CUDA-core GEMMs; the transposed bf16 pair for the
    // tensor-core GEMMs
    l.dP = take(sizeof(float) * (size_t)l.n);
    l.dpt = take(2 * sizeof(__nv_bfloat16) * (size_t)(4LL * d_h) * (size_t)l.ldT);
    l.wpart = take(sizeof(float) * (size_t)l.splits * 4 * d_h * d_in);
    l.err = take(256);
    l.total = off;
    return l;
}

}  // namespace

size_t backward_workspace_bytes(int B, int T, int d_in, int d_h) { return layout(B, T, d_in, d_h).total; }

cudaError_t backward_launch(const void *x, const void *Wx, int dtype, const float *P, const float *R,
                            const float *s0, const float *S, const float *dH, float *dx, float *dWx,
                            float *dR, float *db, float *ds0, int forget, int B, int T, int d_in,
                            int d_h, void *ws, cudaStream_t st)
{
    const Layout l = layout(B, T, d_in, d_h);
    char *base = static_cast<char *>(ws);
    // tensor-core GEMMs need 16-byte TMA strides: (4 d_h) bf16 rows and d_in % 8
    const bool tc = (dtype == SLSTM_BF16) && (d_in % 8 == 0);
    BwdArgs a;
    a.P = P;
    a.R = R;
    a.s0 = s0;
    a.S = S;
    a.dH = dH;
    a.dP = reinterpret_cast<float *>(base + l.dP);
    a.dpt_hi = reinterpret_cast<__nv_bfloat16 *>(base + l.dpt);
    a.dpt_lo = a.dpt_hi + 4LL * d_h * l.ldT;
    a.ldT = l.ldT;
    a.partial = reinterpret_cast<float *>(base + l.partial);
    a.ds0 = ds0;
    a.ticket = reinterpret_cast<unsigned *>(base + l.ticket);
    a.ca.flags = reinterpret_cast<unsigned *>(base + l.flags);
    a.ca.agg = reinterpret_cast<float *>(base + l.agg);
    a.ca.incw = reinterpret_cast<unsigned long long *>(base + l.incw);
    a.ca.error = a.ticket + 1;
    a.ca.epoch = 1;
    a.ca.wait_ns = 2000000000ull;
    a.ca.n_groups = l.n_groups;
    a.T = T;
    a.d = d_h;
    a.groups_per_row = l.groups_per_row;
    a.n_tiles = l.n_tiles;
    a.vec16 = ((d_h & 3) == 0 && (reinterpret_cast<uintptr_t>(S) & 15) == 0 &&
               (reinterpret_cast<uintptr_t>(P) & 15) == 0 && (reinterpret_cast<uintptr_t>(dH) & 15) == 0) ? 1 : 0;
    // ticket, error word, flags and the epoch tags of the inclusive prefixes
    // start cleared
    cudaError_t e = cudaMemsetAsync(base, 0, l.agg, st);
    if (e != cudaSuccess) return e;
    if (forget == SLSTM_FORGET_EXP) {
        e = tc ? launch_adjoint<SLSTM_FORGET_EXP, true>(a, st) : launch_adjoint<SLSTM_FORGET_EXP, false>(a, st);
    } else {
        e = tc ? launch_adjoint<SLSTM_FORGET_SIGMOID, true>(a, st) : launch_adjoint<SLSTM_FORGET_SIGMOID, false>(a, st);
    }
    if (e != cudaSuccess) return e;
    reduce_partials_kernel<<<dim3(l.groups_per_row, 8), 256, 0, st>>>(a.partial, dR, db, B, l.n_chunks,
                                                                   l.groups_per_row, d_h);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const long long N4 = 4LL * d_h;
    const int BT = B * T;
    if (tc) {
        unsigned *err = reinterpret_cast<unsigned *>(base + l.err);
        float *wpart = reinterpret_cast<float *>(base + l.wpart);
        if ((e = cudaMemsetAsync(err, 0, sizeof(unsigned), st)) != cudaSuccess) return e;
        // dx = (dP_hi + dP_lo) W_x: the pair is stored (4 d_h, B*T), i.e. an
        // MN-major A operand; W_x (4 d_h, d_in) is an MN-major B operand
        if ((e = gemm_tc_bf16_ex(a.dpt_hi, a.dpt_lo, (int)l.ldT, true, Wx, d_in, true, nullptr, dx, BT, d_in,
                                 (int)N4, 1, err, st)) != cudaSuccess)
            return e;
        // dW_x = (dP_hi + dP_lo)^T x: K-major A, x (B*T, d_in) an MN-major B
        // operand; split over B*T, partial sums added in order
        if ((e = gemm_tc_bf16_ex(a.dpt_hi, a.dpt_lo, (int)l.ldT, false, x, d_in, true, nullptr, wpart, (int)N4, d_in,
                                 BT, l.splits, err, st)) != cudaSuccess)
            return e;
        const long long nw = N4 * d_in;
        sum_splits_kernel<<<(unsigned)((nw + 255) / 256), 256, 0, st>>>(wpart, dWx, nw, l.splits);
        return cudaGetLastError();
    }

    // dx[(b,t), k] = sum_{g,j} dP[(b,t), (g,j)] Wx[(g,j), k]
    GemmDesc gx;
    gx.M = BT;
    gx.N = d_in;
    gx.K = (int)N4;
    gx.A = a.dP;
    gx.a_dtype = SLSTM_F32;
    gx.sam = N4;
    gx.sak = 1;
    gx.B = Wx;
    gx.b_dtype = dtype;
    gx.sbk = d_in;
    gx.sbn = 1;
    gx.bias = nullptr;
    gx.C = dx;
    if ((e = gemm_simt(gx, st)) != cudaSuccess) return e;
    // dWx[(g,j), k] = sum_{(b,t)} dP[(b,t), (g,j)] x[(b,t), k]
    GemmDesc gw;
    gw.M = (int)N4;
    gw.N = d_in;
    gw.K = BT;
    gw.A = a.dP;
    gw.a_dtype = SLSTM_F32;
    gw.sam = 1;
    gw.sak = N4;
    gw.B = x;
    gw.b_dtype = dtype;
    gw.sbk = d_in;
    gw.sbn = 1;
    gw.bias = nullptr;
    gw.C = dWx;
    return gemm_simt(gw, st);
}

}  // namespace slstm
