// Fused Newton iteration for the diag-mix sLSTM.
//
// One launch is one Newton iteration ("sLSTM in this library", section
// "Cell": the fused diag training cell runs Newton with a 4x4 Jacobian per
// feature and an O(d) combine; "pararnn-torch structure", section "Current
// surface": fused kernels prepend h0, residual early stop, divergence after
// K).  Per tile of 32 features x TT steps:
//   walk A  each thread (one feature, L consecutive steps) recomputes gates,
//           stabilizer, f(S_{t-1}, P_t) and J_t in registers from P and the
//           current guess, keeps (J_t, r_t = f - S_t) in registers and folds
//           the affine maps delta -> J_t delta + r_t;
//   scan    warp 0 combines the warps, publishes, looks back across tiles;
//   walk B  each thread replays its L steps from the incoming carry,
//           writes S + delta in place and (when asked) evaluates the residual
//           of the new iterate for the stopping test.
// In-place update is safe because the only value a tile reads from another
// tile (the state just before it) comes from a per-tile boundary buffer
// written by the previous launch.
#include "lookback.cuh"
#include "launchers.h"

#include <float.h>

namespace slstm {
namespace {

constexpr int NW = 8;   // warps per tile (time segments)
constexpr int L = 4;    // steps per thread
constexpr int TT = NW * L;

struct Args {
    const float *P;
    const float *R;
    const float *s0;
    float *S;
    NewtonCtrl *ctrl;
    LookbackArgs lb;
    float *bnd_in;   // [n_tiles][4][32]  S of the previous iterate at each tile's last step
    float *bnd_out;
    slstm_newton_stats *stats;
    int B, T, d, groups_per_row, n_tiles, max_iters, fixed, fault_ticket;
    float tol;
};

__device__ void finalize(const Args &a, int k, bool resid)
{
    NewtonCtrl *c = a.ctrl;
    slstm_newton_stats *st = a.stats;
    NewtonSlot &s = c->slot[k & 1];
    const float raw = __uint_as_float(atomicOr(&s.maxF_raw, 0u));
    const float sc = __uint_as_float(atomicOr(&s.maxF_scaled, 0u));
    const unsigned err = atomicOr(&c->error, 0u);
    const bool last = (k + 1 == a.max_iters);
    // the next iteration starts from a clean slot (its previous user,
    // iteration k - 1, finished before this launch began)
    NewtonSlot &nx = c->slot[(k + 1) & 1];
    nx.ticket = 0u;
    nx.finished = 0u;
    nx.maxF_raw = 0u;
    nx.maxF_scaled = 0u;
    st->iters = k + 1;
    st->max_abs_F[k % SLSTM_STATS_HISTORY] = resid ? raw : -1.0f;
    st->max_scaled_F[k % SLSTM_STATS_HISTORY] = resid ? sc : -1.0f;
    bool done = last;
    if (err) {
        st->error = SLSTM_ERR_TIMEOUT;
        done = true;
    } else if (resid) {
        const bool bad = !(raw <= FLT_MAX) || !(sc <= FLT_MAX);
        if (bad) {
            st->diverged = 1;
            st->error = SLSTM_ERR_DIVERGED;
            done = true;
        } else if (sc <= a.tol && (!a.fixed || last)) {
            st->converged = 1;
            done = done || !a.fixed;
        } else if (last && raw > 1.0f) {
            st->diverged = 1;
            st->error = SLSTM_ERR_DIVERGED;
        }
    }
    __threadfence();
    if (done) atomicExch(&c->done, 1u);
}

template <int FORGET, bool FIRST, bool RESID>
__global__ void __launch_bounds__(NW * 32, 2) newton_iter(Args a, int k)
{
    __shared__ float s_agg[NW][20][32];
    __shared__ float s_cin[4][32];
    __shared__ float s_red[2][NW];
    __shared__ unsigned s_ticket;
    __shared__ int s_exit;

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        const unsigned ex = *(volatile unsigned *)&a.ctrl->done;
        s_exit = (int)ex;
        if (!ex) s_ticket = atomicAdd(&a.ctrl->slot[k & 1].ticket, 1u);
    }
    __syncthreads();
    if (s_exit) return;

    const unsigned ticket = s_ticket;
    const int G = a.lb.n_groups;
    const int chunk = (int)(ticket / (unsigned)G);
    const int grp = (int)(ticket % (unsigned)G);
    const int b = grp / a.groups_per_row;
    const int j = (grp % a.groups_per_row) * 32 + lane;
    const bool jv = j < a.d;
    const size_t d = (size_t)a.d;
    const int T = a.T;
    const int t_seg = chunk * TT + warp * L;
    const size_t row0 = (size_t)b * T;  // (b, t) row = row0 + t
    const size_t jj = jv ? (size_t)j : 0;

    float rz = 0.f, ri = 0.f, rf = 0.f, ro = 0.f;
    if (jv) {
        rz = a.R[jj];
        ri = a.R[d + jj];
        rf = a.R[2 * d + jj];
        ro = a.R[3 * d + jj];
    }

    // old state just before this warp's segment
    float sp[4] = {0.f, 0.f, 0.f, 0.f};
    if (t_seg == 0) {
        if (a.s0 && jv) {
#pragma unroll
            for (int e = 0; e < 4; ++e) sp[e] = a.s0[((size_t)b * 4 + e) * d + jj];
        }
    } else if (!FIRST) {
        if (warp == 0) {
            const float *src = a.bnd_in + (size_t)(ticket - (unsigned)G) * 4 * 32;
#pragma unroll
            for (int e = 0; e < 4; ++e) sp[e] = src[e * 32 + lane];
        } else if (jv) {
            const float *src = a.S + (row0 + t_seg - 1) * 4 * d + jj;
#pragma unroll
            for (int e = 0; e < 4; ++e) sp[e] = src[e * d];
        }
    }

    // ---- walk A ----
    Cell Jc[L];
    float rr[L][4];
    Aff agg;
    aff_identity(agg);
    {
        float cur[4] = {sp[0], sp[1], sp[2], sp[3]};
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int t = t_seg + i;
            if (t < T) {
                float p[4] = {0.f, 0.f, 0.f, 0.f}, so[4] = {0.f, 0.f, 0.f, 0.f};
                if (jv) {
                    const float *pp = a.P + (row0 + t) * 4 * d + jj;
#pragma unroll
                    for (int e = 0; e < 4; ++e) p[e] = __ldg(pp + e * d);
                    if (!FIRST) {
                        const float *sq = a.S + (row0 + t) * 4 * d + jj;
#pragma unroll
                        for (int e = 0; e < 4; ++e) so[e] = sq[e * d];
                    }
                }
                cell_eval<FORGET, true>(cur[0], cur[1], cur[2], cur[3], p[0], p[1], p[2], p[3], rz,
                                        ri, rf, ro, Jc[i]);
                rr[i][0] = Jc[i].c - so[0];
                rr[i][1] = Jc[i].n - so[1];
                rr[i][2] = Jc[i].m - so[2];
                rr[i][3] = Jc[i].h - so[3];
#pragma unroll
                for (int e = 0; e < 4; ++e) cur[e] = so[e];
            } else {
                cell_identity(Jc[i]);
#pragma unroll
                for (int e = 0; e < 4; ++e) rr[i][e] = 0.f;
            }
            fold_jac(agg, Jc[i], rr[i]);
        }
    }
    store_aff_smem(s_agg, warp, lane, agg);
    __syncthreads();
    tile_prefix_tree<NW>(s_agg, agg);

    if (warp == 0) {
        const float zero[4] = {0.f, 0.f, 0.f, 0.f};
        const bool withhold = (k == 0) && ((int)ticket == a.fault_ticket);
        tile_lookback_warp0<NW>(s_agg, s_cin, a.lb, ticket, chunk, zero, withhold);
    }
    __syncthreads();

    // ---- walk B ----
    float dl[4];
    warp_carry(s_agg, s_cin, warp, lane, dl);
    float snp[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) snp[e] = sp[e] + dl[e];
    float mx_raw = 0.f, mx_sc = 0.f;
#pragma unroll
    for (int i = 0; i < L; ++i) {
        const int t = t_seg + i;
        if (t < T) {
            jac_mul(Jc[i], dl[0], dl[1], dl[2], dl[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) dl[e] += rr[i][e];
            float sn[4];
            if (jv) {
                float *sq = a.S + (row0 + t) * 4 * d + jj;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float so = FIRST ? 0.f : sq[e * d];
                    sn[e] = so + dl[e];
                    sq[e * d] = sn[e];
                }
                if (RESID) {
                    const float *pp = a.P + (row0 + t) * 4 * d + jj;
                    Cell f;
                    cell_eval<FORGET, false>(snp[0], snp[1], snp[2], snp[3], __ldg(pp), __ldg(pp + d),
                                             __ldg(pp + 2 * d), __ldg(pp + 3 * d), rz, ri, rf, ro, f);
                    const float F[4] = {sn[0] - f.c, sn[1] - f.n, sn[2] - f.m, sn[3] - f.h};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float af = fabsf(F[e]);
                        const float sc = af / (1.0f + fabsf(sn[e]));
                        // propagate NaN: a NaN compares false, so test "not <="
                        mx_raw = (af <= mx_raw) ? mx_raw : af;
                        mx_sc = (sc <= mx_sc) ? mx_sc : sc;
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) sn[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) snp[e] = sn[e];
        }
    }
    // state at the tile's last step, for the next launch's successor tile
    if (warp == NW - 1 && t_seg + L - 1 < T) {
        float *dst = a.bnd_out + (size_t)ticket * 4 * 32;
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e * 32 + lane] = snp[e];
    }

    if (RESID) {
        mx_raw = warp_max(mx_raw);
        mx_sc = warp_max(mx_sc);
        if (lane == 0) {
            s_red[0][warp] = mx_raw;
            s_red[1][warp] = mx_sc;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (RESID) {
            float r0 = s_red[0][0], r1 = s_red[1][0];
            for (int w = 1; w < NW; ++w) {
                r0 = (__float_as_uint(s_red[0][w]) > __float_as_uint(r0)) ? s_red[0][w] : r0;
                r1 = (__float_as_uint(s_red[1][w]) > __float_as_uint(r1)) ? s_red[1][w] : r1;
            }
            atomic_max_nonneg(&a.ctrl->slot[k & 1].maxF_raw, r0);
            atomic_max_nonneg(&a.ctrl->slot[k & 1].maxF_scaled, r1);
        }
        __threadfence();
        const unsigned fin = atomicAdd(&a.ctrl->slot[k & 1].finished, 1u);
        if (fin == (unsigned)a.n_tiles - 1u) {
            __threadfence();
            finalize(a, k, RESID);
        }
    }
}

template <int FORGET>
cudaError_t launch_iters(const Args &base, int max_iters, bool fixed, cudaStream_t st)
{
    const dim3 block(NW * 32);
    const dim3 grid(base.n_tiles);
    for (int k = 0; k < max_iters; ++k) {
        Args a = base;
        a.lb.epoch = (unsigned)(k + 1);
        a.bnd_in = (k & 1) ? base.bnd_out : base.bnd_in;
        a.bnd_out = (k & 1) ? base.bnd_in : base.bnd_out;
        const bool resid = !fixed || (k + 1 == max_iters);
        if (k == 0) {
            if (resid)
                newton_iter<FORGET, true, true><<<grid, block, 0, st>>>(a, k);
            else
                newton_iter<FORGET, true, false><<<grid, block, 0, st>>>(a, k);
        } else {
            if (resid)
                newton_iter<FORGET, false, true><<<grid, block, 0, st>>>(a, k);
            else
                newton_iter<FORGET, false, false><<<grid, block, 0, st>>>(a, k);
        }
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

struct Layout {
    size_t ctrl, flags, agg, inc, bnd0, bnd1, total;
    int groups_per_row, n_groups, n_chunks, n_tiles;
};

Layout layout(int B, int T, int d)
{
    Layout l;
    l.groups_per_row = (d + 31) / 32;
    l.n_groups = B * l.groups_per_row;
    l.n_chunks = (T + TT - 1) / TT;
    l.n_tiles = l.n_groups * l.n_chunks;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~(size_t)255;
        return at;
    };
    l.ctrl = take(sizeof(NewtonCtrl));
    l.flags = take(sizeof(unsigned) * (size_t)l.n_tiles);
    l.agg = take(sizeof(float) * 20 * 32 * (size_t)l.n_tiles);
    l.inc = take(sizeof(float) * 4 * 32 * (size_t)l.n_tiles);
    l.bnd0 = take(sizeof(float) * 4 * 32 * (size_t)l.n_tiles);
    l.bnd1 = take(sizeof(float) * 4 * 32 * (size_t)l.n_tiles);
    l.total = off;
    return l;
}

}  // namespace

size_t newton_workspace_bytes(int B, int T, int d) { return layout(B, T, d).total; }

cudaError_t newton_forward(const float *P, const float *R, const float *s0, float *S,
                           const slstm_newton_config &cfg, slstm_newton_stats *stats, int B, int T,
                           int d, void *ws, cudaStream_t st)
{
    const Layout l = layout(B, T, d);
    char *base = static_cast<char *>(ws);
    Args a;
    a.P = P;
    a.R = R;
    a.s0 = s0;
    a.S = S;
    a.ctrl = reinterpret_cast<NewtonCtrl *>(base + l.ctrl);
    a.lb.flags = reinterpret_cast<unsigned *>(base + l.flags);
    a.lb.agg = reinterpret_cast<float *>(base + l.agg);
    a.lb.inc = reinterpret_cast<float *>(base + l.inc);
    a.lb.error = &a.ctrl->error;
    a.lb.epoch = 1;
    a.lb.wait_ns = (uint64_t)(cfg.wait_limit_us > 0 ? cfg.wait_limit_us : 2000000) * 1000ull;
    a.lb.n_groups = l.n_groups;
    a.bnd_in = reinterpret_cast<float *>(base + l.bnd0);
    a.bnd_out = reinterpret_cast<float *>(base + l.bnd1);
    a.stats = stats;
    a.B = B;
    a.T = T;
    a.d = d;
    a.groups_per_row = l.groups_per_row;
    a.n_tiles = l.n_tiles;
    a.max_iters = cfg.max_iters;
    a.fixed = cfg.fixed_iters ? 1 : 0;
    a.tol = cfg.tol;
    // fault injection: the first tile of chunk 1 withholds its publications,
    // so the first tile of chunk 2 has nothing to wait for
    a.fault_ticket = (cfg.debug_fault == 1 && l.n_chunks >= 3) ? l.n_groups : -1;

    cudaError_t e = cudaMemsetAsync(base + l.ctrl, 0, sizeof(NewtonCtrl), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(base + l.flags, 0, sizeof(unsigned) * l.n_tiles, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(stats, 0, sizeof(slstm_newton_stats), st);
    if (e != cudaSuccess) return e;
    if (cfg.forget == SLSTM_FORGET_EXP) return launch_iters<SLSTM_FORGET_EXP>(a, cfg.max_iters, a.fixed, st);
    return launch_iters<SLSTM_FORGET_SIGMOID>(a, cfg.max_iters, a.fixed, st);
}

}  // namespace slstm
