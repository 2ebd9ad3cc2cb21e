// Head mixing ("sLSTM in this library", section "Cell", row 'head': Beck's
// block-diagonal R of shape (4, n_heads, d_head, d_head), a factorised
// Newton, reverse pass and packed VJP that never form the dense (4 d_head)^2
// Jacobian, fused for d_head <= 32).
//
// With head mixing the pre-activation of gate g of feature i of head hd is
//   a_g[i] = P_g[i] + sum_k R[g][hd][i][k] h_{t-1}[k]        (k over the head)
// so the step's Jacobian is the feature-diagonal part Jl (the cell with no
// recurrent input) plus G R routed into the h column, G = ds_t/da_t per
// feature.  Every kernel here keeps that factorisation: one warp per (batch
// row, head), lane i = feature i of the head, the warp's R rows (or columns)
// in registers, and the product with R formed as 32 broadcasts and fused
// multiply-adds per gate.  The Newton linear solve
//   delta_t = Jl_t delta_{t-1} + G_t (R delta_h,{t-1}) - F_t
// is applied step by step with these matrix-vector products (composing the
// maps would form the dense (4 d_head)^2 products the factorisation avoids),
// in parallel over batch rows and heads; the nonlinear evaluation of each
// step (gates, stabiliser, Jl, G) sits off that recurrence's critical path.
#include <cuda_bf16.h>
#include <string.h>

#define SLSTM_FILE_ID 7
#include "checked.cuh"
#include "common.cuh"
#include "launchers.h"
#include "stop_rule.cuh"

namespace slstm {
namespace {

constexpr int HW = 4;      // warps per CTA, one (batch row, head) each
constexpr int MAXDH = 32;  // head width handled by one warp

struct HeadArgs {
    const float *P;     // (B, T, 4, d) pre-activations without the recurrent term
    const float *Rh;    // (4, H, dh, dh)
    const float *s0;    // (B, 4, d) or null
    float *S;           // (B, T, 4, d)
    int B, T, d, dh, H;
    long long n_ps, n_s0;   // elements of P (and S), of s0 (checked build)
    StopRule rule;
};

// This lane's R rows: r[g][k] = Rh[g][hd][lane][k], zero past d_head.
SLSTM_DEVINL void load_rows(const float *Rh, int H, int dh, int hd, int lane, float r[4][MAXDH])
{
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int k = 0; k < MAXDH; ++k)
            r[g][k] = (lane < dh && k < dh && SLSTM_IN((((size_t)g * H + hd) * dh + lane) * dh + k, 4LL * H * dh * dh))
                          ? __ldg(Rh + (((size_t)g * H + hd) * dh + lane) * dh + k) : 0.0f;
}

// This lane's R columns: c[g][i] = Rh[g][hd][i][lane], zero past d_head.
SLSTM_DEVINL void load_cols(const float *Rh, int H, int dh, int hd, int lane, float c[4][MAXDH])
{
#pragma unroll
    for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int i = 0; i < MAXDH; ++i)
            c[g][i] = (lane < dh && i < dh && SLSTM_IN((((size_t)g * H + hd) * dh + i) * dh + lane, 4LL * H * dh * dh))
                          ? __ldg(Rh + (((size_t)g * H + hd) * dh + i) * dh + lane) : 0.0f;
}

// out[g] = sum_k r[g][k] v_k, v_k = lane k's v (lanes past d_head hold 0).
SLSTM_DEVINL void mix(const float r[4][MAXDH], float v, float out[4])
{
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int k = 0; k < MAXDH; ++k) {
        const float vk = __shfl_sync(0xffffffffu, v, k);
        a0 = fmaf(r[0][k], vk, a0);
        a1 = fmaf(r[1][k], vk, a1);
        a2 = fmaf(r[2][k], vk, a2);
        a3 = fmaf(r[3][k], vk, a3);
    }
    out[0] = a0;
    out[1] = a1;
    out[2] = a2;
    out[3] = a3;
}

// (G u) for the sparse gate-space derivative (rows c, n, m, h; columns z, i, f, o).
SLSTM_DEVINL void g_mul(const CellG &g, const float u[4], float out[4])
{
    out[0] = fmaf(g.gcz, u[0], fmaf(g.gci, u[1], g.gcf * u[2]));
    out[1] = fmaf(g.gni, u[1], g.gnf * u[2]);
    out[2] = fmaf(g.gmi, u[1], g.gmf * u[2]);
    out[3] = fmaf(g.ghz, u[0], fmaf(g.ghi, u[1], fmaf(g.ghf, u[2], g.gho * u[3])));
}

// G^T l (the packed VJP of one step: dP = G^T lambda).
SLSTM_DEVINL void gT_mul(const CellG &g, const float l[4], float out[4])
{
    out[0] = fmaf(g.gcz, l[0], g.ghz * l[3]);
    out[1] = fmaf(g.gci, l[0], fmaf(g.gni, l[1], fmaf(g.gmi, l[2], g.ghi * l[3])));
    out[2] = fmaf(g.gcf, l[0], fmaf(g.gnf, l[1], fmaf(g.gmf, l[2], g.ghf * l[3])));
    out[3] = g.gho * l[3];
}

// base, n: the buffer p points into and its element count (checked build).
SLSTM_DEVINL void load4(const float *p, size_t stride, bool ok, float v[4], const float *base, long long n)
{
    ok = ok && SLSTM_PIN(p + 3 * stride, base, n);
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = ok ? __ldg(p + e * stride) : 0.0f;
}

// The same through the coherent path, for an array this kernel also writes.
SLSTM_DEVINL void load4_rw(const float *p, size_t stride, bool ok, float v[4], const float *base, long long n)
{
    ok = ok && SLSTM_PIN(p + 3 * stride, base, n);
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = ok ? p[e * stride] : 0.0f;
}

// ---- sequential stepping ----------------------------------------------------
template <int FORGET>
__global__ void __launch_bounds__(HW * 32) head_seq_kernel(HeadArgs a)
{
    const int lane = threadIdx.x & 31;
    const int wg = blockIdx.x * HW + (threadIdx.x >> 5);
    if (wg >= a.B * a.H) return;
    const int b = wg / a.H, hd = wg - b * a.H;
    const bool jv = lane < a.dh;
    const size_t j = (size_t)hd * a.dh + (jv ? lane : 0);
    const size_t d = (size_t)a.d;
    float r[4][MAXDH];
    load_rows(a.Rh, a.H, a.dh, hd, lane, r);
    float s[4];
    load4(a.s0 + (size_t)b * 4 * d + j, d, a.s0 && jv, s, a.s0, a.n_s0);
    const float *pp = a.P + (size_t)b * a.T * 4 * d + j;
    float *sp = a.S + (size_t)b * a.T * 4 * d + j;
    float p[4];
    load4(pp, d, jv, p, a.P, a.n_ps);
    for (int t = 0; t < a.T; ++t) {
        float pn[4];
        load4(pp + (size_t)(t + 1) * 4 * d, d, jv && t + 1 < a.T, pn, a.P, a.n_ps);   // next step's inputs, ahead
        float m4[4];
        mix(r, jv ? s[3] : 0.0f, m4);
        Cell c;
        cell_eval<FORGET, false>(s[0], s[1], s[2], s[3], p[0] + m4[0], p[1] + m4[1], p[2] + m4[2], p[3] + m4[3], 0.f,
                                 0.f, 0.f, 0.f, c);
        s[0] = c.c;
        s[1] = c.n;
        s[2] = c.m;
        s[3] = c.h;
        if (jv && SLSTM_PIN(sp + (size_t)t * 4 * d + 3 * d, a.S, a.n_ps)) {
#pragma unroll
            for (int e = 0; e < 4; ++e) sp[(size_t)t * 4 * d + e * d] = s[e];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) p[e] = pn[e];
    }
}

// ---- one Newton iteration ---------------------------------------------------
// FIRST: the zero initial guess (S is not read).  RESID: evaluate the
// residual of the new iterate for the stopping test.
template <int FORGET, bool FIRST, bool RESID>
__global__ void __launch_bounds__(HW * 32) head_newton_kernel(HeadArgs a, int k)
{
    __shared__ float red[2][HW];
    NewtonCtrl *ctrl = a.rule.ctrl;
    if (*(volatile unsigned *)&ctrl->done) return;   // converged (or stopped) before this launch
    NewtonSlot &slot = ctrl->slot[k & 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wg = blockIdx.x * HW + warp;
    float mx_raw = 0.f, mx_sc = 0.f;
    if (wg < a.B * a.H) {
        const int b = wg / a.H, hd = wg - b * a.H;
        const bool jv = lane < a.dh;
        const size_t j = (size_t)hd * a.dh + (jv ? lane : 0);
        const size_t d = (size_t)a.d;
        float r[4][MAXDH];
        load_rows(a.Rh, a.H, a.dh, hd, lane, r);
        float so_p[4], sn_p[4], dl[4] = {0.f, 0.f, 0.f, 0.f};
        load4(a.s0 + (size_t)b * 4 * d + j, d, a.s0 && jv, so_p, a.s0, a.n_s0);
#pragma unroll
        for (int e = 0; e < 4; ++e) sn_p[e] = so_p[e];
        const float *pp = a.P + (size_t)b * a.T * 4 * d + j;
        float *sp = a.S + (size_t)b * a.T * 4 * d + j;
        float p[4], so[4];
        load4(pp, d, jv, p, a.P, a.n_ps);
        load4_rw(sp, d, jv && !FIRST, so, a.S, a.n_ps);
        for (int t = 0; t < a.T; ++t) {
            // next step's inputs, ahead (S at t + 1 is not written before it is read here)
            float pn[4], son[4];
            load4(pp + (size_t)(t + 1) * 4 * d, d, jv && t + 1 < a.T, pn, a.P, a.n_ps);
            load4_rw(sp + (size_t)(t + 1) * 4 * d, d, jv && !FIRST && t + 1 < a.T, son, a.S, a.n_ps);
            // f, Jl and G at the old iterate
            float mo[4];
            mix(r, jv ? so_p[3] : 0.0f, mo);
            Cell c;
            CellG gg;
            cell_eval<FORGET, true, true>(so_p[0], so_p[1], so_p[2], so_p[3], p[0] + mo[0], p[1] + mo[1],
                                          p[2] + mo[2], p[3] + mo[3], 0.f, 0.f, 0.f, 0.f, c, &gg);
            // S_new = f + Jl delta_{t-1} + G (R delta_h,{t-1});  delta_t = S_new - S_old
            float u[4], gu[4];
            mix(r, jv ? dl[3] : 0.0f, u);
            g_mul(gg, u, gu);
            const float f4[4] = {c.c + gu[0], c.n + gu[1], c.m + gu[2], c.h + gu[3]};
            float sn[4];
            jac_mul_add(c, dl, f4, sn);
#pragma unroll
            for (int e = 0; e < 4; ++e) dl[e] = sn[e] - so[e];
            if (jv && SLSTM_PIN(sp + (size_t)t * 4 * d + 3 * d, a.S, a.n_ps)) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sp[(size_t)t * 4 * d + e * d] = sn[e];
            }
            if (RESID) {
                float mn[4];
                mix(r, jv ? sn_p[3] : 0.0f, mn);
                Cell fnew;
                cell_eval<FORGET, false>(sn_p[0], sn_p[1], sn_p[2], sn_p[3], p[0] + mn[0], p[1] + mn[1],
                                         p[2] + mn[2], p[3] + mn[3], 0.f, 0.f, 0.f, 0.f, fnew);
                const float F[4] = {sn[0] - fnew.c, sn[1] - fnew.n, sn[2] - fnew.m, sn[3] - fnew.h};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float af = jv ? fabsf(F[e]) : 0.0f;
                    mx_raw = fmax_nan(mx_raw, af);
                    mx_sc = fmax_nan(mx_sc, __fdividef(af, 1.0f + fabsf(sn[e])));
                }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                so_p[e] = so[e];
                sn_p[e] = sn[e];
                p[e] = pn[e];
                so[e] = son[e];
            }
        }
    }
    if (RESID) {
        mx_raw = warp_max(mx_raw);
        mx_sc = warp_max(mx_sc);
        if (lane == 0) {
            red[0][warp] = mx_raw;
            red[1][warp] = mx_sc;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (RESID) {
            float r0 = red[0][0], r1 = red[1][0];
            for (int w = 1; w < HW; ++w) {
                r0 = (__float_as_uint(red[0][w]) > __float_as_uint(r0)) ? red[0][w] : r0;
                r1 = (__float_as_uint(red[1][w]) > __float_as_uint(r1)) ? red[1][w] : r1;
            }
            atomic_max_nonneg(&slot.maxF_raw, r0);
            atomic_max_nonneg(&slot.maxF_scaled, r1);
        }
        __threadfence();
        if (atomicAdd(&slot.finished, 1u) == gridDim.x - 1u) {
            __threadfence();
            finalize_iteration(a.rule, k, RESID);
        }
    }
}

// ---- backward ---------------------------------------------------------------
// Pre-activations with the recurrent term, for every step at once:
// A_t = P_t + R h_{t-1} (h_{-1} = s0's h).  One warp per (batch row, head,
// chunk of HCH steps).
constexpr int HCH = 64;

__global__ void __launch_bounds__(HW * 32) head_preact_kernel(HeadArgs a, float *A)
{
    const int lane = threadIdx.x & 31;
    const long long wg = (long long)blockIdx.x * HW + (threadIdx.x >> 5);
    const int n_ch = (a.T + HCH - 1) / HCH;
    if (wg >= (long long)a.B * a.H * n_ch) return;
    const int ch = (int)(wg % n_ch);
    const int bh = (int)(wg / n_ch);
    const int b = bh / a.H, hd = bh - b * a.H;
    const bool jv = lane < a.dh;
    const size_t j = (size_t)hd * a.dh + (jv ? lane : 0);
    const size_t d = (size_t)a.d;
    float r[4][MAXDH];
    load_rows(a.Rh, a.H, a.dh, hd, lane, r);
    const int t0 = ch * HCH, t1 = min(a.T, t0 + HCH);
    const size_t row0 = (size_t)b * a.T;
    for (int t = t0; t < t1; ++t) {
        float hp;
        if (t == 0) hp = (a.s0 && jv && SLSTM_IN(((size_t)b * 4 + 3) * d + j, a.n_s0))
                             ? __ldg(a.s0 + ((size_t)b * 4 + 3) * d + j) : 0.0f;
        else hp = (jv && SLSTM_IN(((row0 + t - 1) * 4 + 3) * d + j, a.n_ps))
                      ? __ldg(a.S + ((row0 + t - 1) * 4 + 3) * d + j) : 0.0f;
        float m4[4];
        mix(r, hp, m4);
        if (jv && SLSTM_IN(((row0 + t) * 4 + 3) * d + j, a.n_ps)) {
#pragma unroll
            for (int e = 0; e < 4; ++e) A[((row0 + t) * 4 + e) * d + j] = __ldg(a.P + ((row0 + t) * 4 + e) * d + j) + m4[e];
        }
    }
}

// The adjoint walked backwards in time with the packed VJP, one warp per
// (batch row, head):
//   lambda_t = e_h dH_t + Jl_{t+1}^T lambda_{t+1} + e_h (R^T dP_{t+1})
//   dP_t = G_t^T lambda_t,   ds0 = Jl_0^T lambda_0 + e_h (R^T dP_0)
// (the h-column part of J^T lambda is R^T G^T lambda = R^T dP).  Writes dP
// (B, T, 4, d) fp32 and ds0.
template <int FORGET>
__global__ void __launch_bounds__(HW * 32) head_adjoint_kernel(HeadArgs a, const float *A, const float *dH, float *dP,
                                                               float *ds0)
{
    const int lane = threadIdx.x & 31;
    const int wg = blockIdx.x * HW + (threadIdx.x >> 5);
    if (wg >= a.B * a.H) return;
    const int b = wg / a.H, hd = wg - b * a.H;
    const bool jv = lane < a.dh;
    const size_t j = (size_t)hd * a.dh + (jv ? lane : 0);
    const size_t d = (size_t)a.d;
    float rc[4][MAXDH];
    load_cols(a.Rh, a.H, a.dh, hd, lane, rc);
    const size_t row0 = (size_t)b * a.T;
    float lam[4] = {0.f, 0.f, 0.f, 0.f};
    float dp1[4] = {0.f, 0.f, 0.f, 0.f};   // dP_{t+1}
    Cell j1;                                // Jl_{t+1}
    cell_zero_jac(j1);
    for (int t = a.T - 1; t >= 0; --t) {
        // e_h (R^T dP_{t+1}): lane k sums R[g][i][k] dP_{t+1}[g][i] over g and i
        float rt = 0.f;
#pragma unroll
        for (int i = 0; i < MAXDH; ++i) {
#pragma unroll
            for (int g = 0; g < 4; ++g) rt = fmaf(rc[g][i], __shfl_sync(0xffffffffu, dp1[g], i), rt);
        }
        jacT_mul(j1, lam[0], lam[1], lam[2], lam[3]);
        lam[3] += rt + ((jv && SLSTM_IN((row0 + t) * d + j, a.n_ps / 4)) ? __ldg(dH + (row0 + t) * d + j) : 0.0f);
        float sp[4], av[4];
        if (t == 0) load4(a.s0 + (size_t)b * 4 * d + j, d, a.s0 && jv, sp, a.s0, a.n_s0);
        else load4(a.S + (row0 + t - 1) * 4 * d + j, d, jv, sp, a.S, a.n_ps);
        load4(A + (row0 + t) * 4 * d + j, d, jv, av, A, a.n_ps);
        Cell c;
        CellG gg;
        cell_eval<FORGET, true, true>(sp[0], sp[1], sp[2], sp[3], av[0], av[1], av[2], av[3], 0.f, 0.f, 0.f, 0.f, c,
                                      &gg);
        float dp[4];
        gT_mul(gg, lam, dp);
        if (!jv) {
#pragma unroll
            for (int e = 0; e < 4; ++e) dp[e] = 0.0f;
        }
        if (jv && SLSTM_IN((row0 + t) * 4 * d + 3 * d + j, a.n_ps)) {
#pragma unroll
            for (int e = 0; e < 4; ++e) dP[(row0 + t) * 4 * d + e * d + j] = dp[e];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) dp1[e] = dp[e];
        j1 = c;
    }
    if (ds0) {
        float rt = 0.f;
#pragma unroll
        for (int i = 0; i < MAXDH; ++i) {
#pragma unroll
            for (int g = 0; g < 4; ++g) rt = fmaf(rc[g][i], __shfl_sync(0xffffffffu, dp1[g], i), rt);
        }
        jacT_mul(j1, lam[0], lam[1], lam[2], lam[3]);
        lam[3] += rt;
        if (jv && SLSTM_IN(((size_t)b * 4 + 3) * d + j, a.n_s0)) {
#pragma unroll
            for (int e = 0; e < 4; ++e) ds0[((size_t)b * 4 + e) * d + j] = lam[e];
        }
    }
}

// dR and db partial sums over one chunk of RCH rows (b, t) for one head:
//   dR[g][i][k] += dP[row][g][i] h_{t-1}[k],  db[g][i] += dP[row][g][i]
// 256 threads, thread (g, i-block, k-block) keeps a 4 x 4 block of dR.
constexpr int RCH = 2048;   // rows per partial
constexpr int RSUB = 32;    // rows staged in shared memory at a time

__global__ void __launch_bounds__(256) head_dr_partial_kernel(HeadArgs a, const float *dP, float *part_r,
                                                              float *part_b)
{
    __shared__ float s_dp[RSUB][4][MAXDH];
    __shared__ float s_h[RSUB][MAXDH];
    const int hd = blockIdx.x, ch = blockIdx.y;
    const long long BT = (long long)a.B * a.T;
    const long long r0 = (long long)ch * RCH, r1 = min(BT, r0 + RCH);
    const int tid = threadIdx.x;
    const int g = tid >> 6, ib = (tid >> 3) & 7, kb = tid & 7;
    const size_t d = (size_t)a.d;
    const int dh = a.dh;
    float acc[4][4];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = 0.0f;
    float bsum = 0.0f;   // threads 0 .. 4 dh - 1: db of (g, i) = (tid / dh, tid % dh)
    for (long long rs = r0; rs < r1; rs += RSUB) {
        __syncthreads();
        // stage RSUB rows of dP (4 x dh) and of h_{t-1} (dh)
        for (int q = tid; q < RSUB * 5 * MAXDH; q += 256) {
            const int rr = q / (5 * MAXDH), e = (q / MAXDH) % 5, i = q % MAXDH;
            const long long row = rs + rr;
            float v = 0.0f;
            if (row < r1 && i < dh) {
                const size_t jj = (size_t)hd * dh + i;
                if (e < 4) {
                    if (SLSTM_IN(((size_t)row * 4 + e) * d + jj, a.n_ps)) v = __ldg(dP + ((size_t)row * 4 + e) * d + jj);
                } else {
                    const long long b = row / a.T, t = row - b * a.T;
                    if (t > 0 && SLSTM_IN((((size_t)row - 1) * 4 + 3) * d + jj, a.n_ps))
                        v = __ldg(a.S + (((size_t)row - 1) * 4 + 3) * d + jj);
                    else if (t == 0 && a.s0 && SLSTM_IN(((size_t)b * 4 + 3) * d + jj, a.n_s0))
                        v = __ldg(a.s0 + ((size_t)b * 4 + 3) * d + jj);
                }
            }
            if (e < 4) s_dp[rr][e][i] = v;
            else s_h[rr][i] = v;
        }
        __syncthreads();
        const int nr = (int)min((long long)RSUB, r1 - rs);
        for (int rr = 0; rr < nr; ++rr) {
            float pv[4], hv[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) pv[x] = s_dp[rr][g][ib * 4 + x];
#pragma unroll
            for (int y = 0; y < 4; ++y) hv[y] = s_h[rr][kb * 4 + y];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(pv[x], hv[y], acc[x][y]);
            if (tid < 4 * dh) bsum += s_dp[rr][tid / dh][tid % dh];
        }
    }
    // part_r[ch][g][hd][i][k], part_b[ch][g][hd * dh + i]
    const size_t base = ((size_t)ch * 4 + g) * a.H + hd;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const int i = ib * 4 + x;
        if (i >= dh) continue;
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int kk = kb * 4 + y;
            if (kk < dh) part_r[(base * dh + i) * dh + kk] = acc[x][y];
        }
    }
    if (tid < 4 * dh) part_b[((size_t)ch * 4 + tid / dh) * d + (size_t)hd * dh + tid % dh] = bsum;
}

// Sums of the partials over the chunks, in chunk order.
__global__ void __launch_bounds__(256) head_dr_final_kernel(const float *part_r, const float *part_b, int n_ch,
                                                            long long n_r, long long n_b, float *dR, float *db)
{
    const long long q = (long long)blockIdx.x * 256 + threadIdx.x;
    if (q < n_r) {
        float acc = 0.0f;
        for (int c = 0; c < n_ch; ++c) acc += part_r[(size_t)c * n_r + q];
        dR[q] = acc;
    } else if (q < n_r + n_b) {
        const long long qb = q - n_r;
        float acc = 0.0f;
        for (int c = 0; c < n_ch; ++c) acc += part_b[(size_t)c * n_b + qb];
        db[qb] = acc;
    }
}

__global__ void __launch_bounds__(256) split_pair_rows_kernel(const float *__restrict__ v, __nv_bfloat16 *__restrict__ hi,
                                                              __nv_bfloat16 *__restrict__ lo, long long n)
{
    const long long q = (long long)blockIdx.x * 256 + threadIdx.x;
    if (q >= n) return;
    const float x = v[q];
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi[q] = h;
    lo[q] = __float2bfloat16_rn(x - __bfloat162float(h));
}

size_t al256(size_t v) { return (v + 255) & ~(size_t)255; }

HeadArgs head_args(const float *P, const float *Rh, const float *s0, float *S, int B, int T, int d, int dh)
{
    HeadArgs a;
    memset(&a, 0, sizeof(a));
    a.P = P;
    a.Rh = Rh;
    a.s0 = s0;
    a.S = S;
    a.B = B;
    a.T = T;
    a.d = d;
    a.dh = dh;
    a.H = d / dh;
    a.n_ps = (long long)B * T * 4 * d;
    a.n_s0 = (long long)B * 4 * d;
    return a;
}

unsigned head_grid(int B, int H) { return (unsigned)((B * H + HW - 1) / HW); }

}  // namespace

cudaError_t head_sequential_launch(const float *P, const float *Rh, const float *s0, float *S, int B, int T, int d,
                                   int dh, int forget, cudaStream_t st)
{
    const HeadArgs a = head_args(P, Rh, s0, S, B, T, d, dh);
    if (forget == SLSTM_FORGET_EXP) head_seq_kernel<SLSTM_FORGET_EXP><<<head_grid(B, a.H), HW * 32, 0, st>>>(a);
    else head_seq_kernel<SLSTM_FORGET_SIGMOID><<<head_grid(B, a.H), HW * 32, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t head_newton_forward(const float *P, const float *Rh, const float *s0, float *S,
                                const slstm_newton_config &cfg, slstm_newton_stats *stats, int B, int T, int d,
                                int dh, void *ws, cudaStream_t st)
{
    NewtonCtrl *ctrl = nullptr;
    cudaError_t e = newton_guess_prepare(P, s0, S, cfg, stats, B, T, d, ws, st, &ctrl);
    if (e != cudaSuccess) return e;
    HeadArgs a = head_args(P, Rh, s0, S, B, T, d, dh);
    const int k0 = cfg.init == SLSTM_INIT_ZERO ? 0 : 1;
    const bool fixed = cfg.fixed_iters != 0;
    a.rule = StopRule{ctrl, stats, k0, cfg.max_iters, fixed ? 1 : 0,
                      cfg.residual_mode == SLSTM_RESIDUAL_RAW ? 1 : 0, 0, cfg.tol};
    const unsigned grid = head_grid(B, a.H);
    for (int k = k0; k < k0 + cfg.max_iters; ++k) {
        const bool resid = !fixed || (k + 1 - k0 == cfg.max_iters);
        const bool first = (k == 0);
        if (cfg.forget == SLSTM_FORGET_EXP) {
            if (first) {
                if (resid) head_newton_kernel<SLSTM_FORGET_EXP, true, true><<<grid, HW * 32, 0, st>>>(a, k);
                else head_newton_kernel<SLSTM_FORGET_EXP, true, false><<<grid, HW * 32, 0, st>>>(a, k);
            } else {
                if (resid) head_newton_kernel<SLSTM_FORGET_EXP, false, true><<<grid, HW * 32, 0, st>>>(a, k);
                else head_newton_kernel<SLSTM_FORGET_EXP, false, false><<<grid, HW * 32, 0, st>>>(a, k);
            }
        } else {
            if (first) {
                if (resid) head_newton_kernel<SLSTM_FORGET_SIGMOID, true, true><<<grid, HW * 32, 0, st>>>(a, k);
                else head_newton_kernel<SLSTM_FORGET_SIGMOID, true, false><<<grid, HW * 32, 0, st>>>(a, k);
            } else {
                if (resid) head_newton_kernel<SLSTM_FORGET_SIGMOID, false, true><<<grid, HW * 32, 0, st>>>(a, k);
                else head_newton_kernel<SLSTM_FORGET_SIGMOID, false, false><<<grid, HW * 32, 0, st>>>(a, k);
            }
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

namespace {

struct HeadBwdOffsets {
    size_t err, A, dP, hi, lo, part_r, part_b, wpart, total;
    int n_ch, splits;
};

HeadBwdOffsets head_bwd_offsets(int B, int T, int d_in, int d, int dh, bool tc)
{
    const size_t BT = (size_t)B * T;
    HeadBwdOffsets o;
    o.n_ch = (int)((BT + RCH - 1) / RCH);
    o.splits = tc ? gemm_tc_splits(4 * d, d_in, (int)BT, 2, 8) : 1;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += al256(bytes);
        return at;
    };
    o.err = take(256);
    o.A = take(BT * 4 * d * 4);
    o.dP = take(BT * 4 * d * 4);
    o.hi = take(tc ? BT * 4 * d * 2 : 0);
    o.lo = take(tc ? BT * 4 * d * 2 : 0);
    o.part_r = take((size_t)o.n_ch * 4 * d * dh * 4);
    o.part_b = take((size_t)o.n_ch * 4 * d * 4);
    o.wpart = take(tc ? (size_t)o.splits * 4 * d * d_in * 4 : 0);
    o.total = off;
    return o;
}

}  // namespace

size_t head_backward_workspace_bytes(int B, int T, int d_in, int d, int dh)
{
    // the larger of the fp32 and the tensor-core layouts, so that one size serves both dtypes
    const size_t a = head_bwd_offsets(B, T, d_in, d, dh, true).total;
    const size_t b = head_bwd_offsets(B, T, d_in, d, dh, false).total;
    return a > b ? a : b;
}

cudaError_t head_backward_launch(const void *x, const void *Wx, int dtype, const float *P, const float *Rh,
                                 const float *s0, const float *S, const float *dH, float *dx, float *dWx, float *dRh,
                                 float *db, float *ds0, int forget, int B, int T, int d_in, int d, int dh, void *ws,
                                 cudaStream_t st)
{
    // tensor cores for bf16 inputs whose rows are 16-byte multiples; CUDA cores otherwise
    const bool tc = dtype == SLSTM_BF16 && d_in % 8 == 0 && d % 2 == 0;
    const HeadBwdOffsets o = head_bwd_offsets(B, T, d_in, d, dh, tc);
    char *base = static_cast<char *>(ws);
    float *A = reinterpret_cast<float *>(base + o.A);
    float *dP = reinterpret_cast<float *>(base + o.dP);
    const HeadArgs a = head_args(P, Rh, s0, const_cast<float *>(S), B, T, d, dh);
    const int n_tch = (T + HCH - 1) / HCH;
    const long long pw = (long long)B * a.H * n_tch;
    head_preact_kernel<<<(unsigned)((pw + HW - 1) / HW), HW * 32, 0, st>>>(a, A);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (forget == SLSTM_FORGET_EXP)
        head_adjoint_kernel<SLSTM_FORGET_EXP><<<head_grid(B, a.H), HW * 32, 0, st>>>(a, A, dH, dP, ds0);
    else
        head_adjoint_kernel<SLSTM_FORGET_SIGMOID><<<head_grid(B, a.H), HW * 32, 0, st>>>(a, A, dH, dP, ds0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    float *part_r = reinterpret_cast<float *>(base + o.part_r);
    float *part_b = reinterpret_cast<float *>(base + o.part_b);
    head_dr_partial_kernel<<<dim3(a.H, o.n_ch), 256, 0, st>>>(a, dP, part_r, part_b);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long n_r = 4LL * d * dh, n_b = 4LL * d;
    head_dr_final_kernel<<<(unsigned)((n_r + n_b + 255) / 256), 256, 0, st>>>(part_r, part_b, o.n_ch, n_r, n_b, dRh,
                                                                             db);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int BT = B * T;
    const long long N4 = 4LL * d;
    if (tc) {
        unsigned *err = reinterpret_cast<unsigned *>(base + o.err);
        __nv_bfloat16 *hi = reinterpret_cast<__nv_bfloat16 *>(base + o.hi);
        __nv_bfloat16 *lo = reinterpret_cast<__nv_bfloat16 *>(base + o.lo);
        float *wpart = reinterpret_cast<float *>(base + o.wpart);
        if ((e = cudaMemsetAsync(err, 0, sizeof(unsigned), st)) != cudaSuccess) return e;
        const long long n = (long long)BT * N4;
        split_pair_rows_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(dP, hi, lo, n);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        // dx = (dP_hi + dP_lo) W_x: dP (B*T, 4d) K-major, W_x (4d, d_in) MN-major
        if ((e = gemm_tc_bf16_ex(hi, lo, (int)N4, false, Wx, d_in, true, nullptr, dx, BT, d_in, (int)N4, 1, err,
                                 st)) != cudaSuccess)
            return e;
        // dW_x = (dP_hi + dP_lo)^T x: dP read MN-major, x (B*T, d_in) MN-major; split over B*T
        if ((e = gemm_tc_bf16_ex(hi, lo, (int)N4, true, x, d_in, true, nullptr, wpart, (int)N4, d_in, BT, o.splits,
                                 err, st)) != cudaSuccess)
            return e;
        return sum_splits(wpart, dWx, N4 * d_in, o.splits, st);
    }
    GemmDesc gx;
    gx.M = BT;
    gx.N = d_in;
    gx.K = (int)N4;
    gx.A = dP;
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
    GemmDesc gw = gx;
    gw.M = (int)N4;
    gw.N = d_in;
    gw.K = BT;
    gw.A = dP;
    gw.sam = 1;
    gw.sak = N4;
    gw.B = x;
    gw.sbk = d_in;
    gw.sbn = 1;
    gw.C = dWx;
    return gemm_simt(gw, st);
}

}  // namespace slstm
