// Backward pass of the Newton-solved diag-mix sLSTM ("sLSTM in this
// library", section "Backward": one reverse associative scan of J^T, then a
// packed cell VJP for the gradients of R and W_x).
//
// Fused adjoint + VJP kernel, tiles in reverse time order:
//   lambda_t = e_h dH_t + J_{t+1}^T lambda_{t+1}
//   dP_t     = G_t^T lambda_t,  G_t = d s_t / d a_t
//   dR      += dP_t * h_{t-1},  db += dP_t   (per-tile partials, reduced after)
//   ds0      = J_0^T lambda_0
// then dx = dP W_x and dW_x = dP^T x.  The scan runs on kappa_{t-1} =
// J_t^T lambda_t (so lambda_t = kappa_t + e_h dH_t), whose step map needs
// only the cell of step t itself; each step's cell (J_t and G_t, recomputed
// from S_{t-1} and P_t) is evaluated once, and the second walk forms G_t^T
// lambda_t and J_t^T lambda_t from eight of its numbers (CellB).
#include <cuda_bf16.h>
#include <string.h>

#define SLSTM_FILE_ID 2
#include "launchers.h"
#include "lookback.cuh"
#include "tma.cuh"

namespace slstm {
namespace {

constexpr int NW = 8;
constexpr int L = 4;
constexpr int TT = NW * L;
constexpr int DPT_LD = 36;   // bf16 row stride of the dP staging: 8-byte rows, conflict-free 8-byte stores

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
    float *cin_buf;   // two-pass carry: [n_tiles][4][32] carry entering each tile (chain layout)
    const unsigned *vmask;   // packed sequences: head-flag words (one per 32 steps), else null
    const int *vseq;         // packed sequences: sequence index at each head step
    int T, d, groups_per_row, n_tiles, vec16, dpt_vec8;
    long long n_ps, n_s0, n_dpt;   // elements of S and P (and dP), of s0 (and ds0), of each half of the pair
    FastDiv div_groups, div_gpr;   // by n_groups and by groups_per_row
};

// A ticket decoded once (by thread 0) for the whole CTA.  The tile covers
// steps t in [t_lo, t_lo + 31], chunk c in reverse time order.
struct BwdInfo {
    unsigned ticket;
    int chunk;
    int b;
    int j0;
    int t_lo;
    int pad;
    unsigned long long hmask;   // packed sequences: bit r set when step t_lo + r (r <= 32) starts a sequence
};

// Shared memory of one CTA.  A tile needs S at t_lo-1 .. t_hi, P and dH at
// t_lo .. t_hi (t_hi = t_lo + 31).
struct BwdSmem {
    float S[2][TT + 1][4][32];   // row r <-> t = t_lo - 1 + r
    float P[2][TT][4][32];       // row r <-> t = t_lo + r
    float dH[2][TT][32];         // row r <-> t = t_lo + r
    float R[2][4][32];           // TMA path: the tile's recurrent weights
    union {
        MapArr m[NW];            // warp maps, dead once the carries are known
        struct {
            __nv_bfloat16 dpt[2][4][32][DPT_LD];   // transposed staging of the dP pair: [part][gate][feature][t]
            float part[NW][8][32];                 // per-warp dR, db partial sums
        } o;
    } u;
    CinArr cin[NW];
    BwdInfo info[3];
    uint64_t bar[2];
};
constexpr size_t BWD_SMEM_BYTES = sizeof(BwdSmem) + 1024;
constexpr int BWD_TMA_THREAD = (NW - 1) * 32;
constexpr uint64_t BWD_TMA_WAIT_NS = 1000000000ull;

// Tensor maps: S and P as (d, 4T, B) with boxes of 32 features x 132 (S) or
// 128 (P) (step, slot) rows, dH as (d, T, B) with boxes of 32 x 32.
struct BwdMaps {
    CUtensorMap S, P, H;
};

SLSTM_DEVINL void bwd_decode(const BwdArgs &a, unsigned ticket, BwdInfo &ti)
{
    ti.ticket = ticket;
    ti.chunk = ti.b = ti.j0 = ti.t_lo = 0;
    ti.hmask = 0ull;
    if (ticket < (unsigned)a.n_tiles) {
        const unsigned G = (unsigned)a.ca.n_groups;
        const unsigned chunk = fast_div(ticket, a.div_groups);
        const unsigned grp = ticket - chunk * G;
        const unsigned b = fast_div(grp, a.div_gpr);
        ti.chunk = (int)chunk;
        ti.b = (int)b;
        ti.j0 = (int)(grp - b * (unsigned)a.groups_per_row) * 32;
        ti.t_lo = a.T - ((int)chunk + 1) * TT;
        if (a.vmask) {
            // bits of steps t_lo .. t_lo + 32 from the (up to three) words they span
            const int q = (ti.t_lo >= 0) ? (ti.t_lo >> 5) : -((31 - ti.t_lo) >> 5);
            const int sh = ti.t_lo - 32 * q;   // 0 .. 31
            const int nw = (a.T + 31) >> 5;
            unsigned long long w[3];
#pragma unroll
            for (int i = 0; i < 3; ++i) w[i] = (q + i >= 0 && q + i < nw) ? a.vmask[q + i] : 0u;
            ti.hmask = (w[0] >> sh) | (w[1] << (32 - sh)) | (sh ? (w[2] << (64 - sh)) : 0ull);
        }
    }
}

// cp.async path: copies of one tile's S, P and dH rows into stage `st`; rows
// outside [0, T) and features past d arrive as zeros.
SLSTM_DEVINL void bwd_prefetch(const BwdArgs &a, BwdSmem &sm, int st, const BwdInfo &ti)
{
    if (ti.ticket >= (unsigned)a.n_tiles) return;
    const int j0 = ti.j0, t_lo = ti.t_lo;
    const size_t d = (size_t)a.d;
    const size_t row0 = (size_t)ti.b * a.T;
    const int T = a.T;
    constexpr int RS = (TT + 1) * 4;           // (row, slot) pairs of S; P has TT * 4
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
                const int tS = t_lo - 1 + r, tP = t_lo + r;
                const int bS = (tS >= 0 && tS < T && SLSTM_IN(((row0 + tS) * 4 + slot) * d + jj + fbytes / 4 - 1, a.n_ps))
                                   ? fbytes : 0;
                cp_async16(&sm.S[st][r][slot][4 * c], bS ? a.S + ((row0 + tS) * 4 + slot) * d + jj : a.S, bS);
                if (r < TT) {
                    const int bP = (tP >= 0 && tP < T && SLSTM_IN(((row0 + tP) * 4 + slot) * d + jj + fbytes / 4 - 1,
                                                                  a.n_ps)) ? fbytes : 0;
                    cp_async16(&sm.P[st][r][slot][4 * c], bP ? a.P + ((row0 + tP) * 4 + slot) * d + jj : a.P, bP);
                }
            }
        }
        const int t = t_lo + q;   // dH row q
        const int bH = (t >= 0 && t < T && SLSTM_IN((row0 + t) * d + jj + fbytes / 4 - 1, a.n_ps / 4)) ? fbytes : 0;
        cp_async16(&sm.dH[st][q][4 * c], bH ? a.dH + (row0 + t) * d + jj : a.dH, bH);
    } else {
        // 4-byte copies, lane = feature, warp w takes every 8th row
        const int jl = threadIdx.x & 31, w = threadIdx.x >> 5;
        const bool fj = j0 + jl < a.d;
        const size_t jj = (size_t)j0 + jl;
        for (int rs = w; rs < RS; rs += NW) {
            const int r = rs >> 2, slot = rs & 3;
            const int tS = t_lo - 1 + r, tP = t_lo + r;
            const int bS = (fj && tS >= 0 && tS < T && SLSTM_IN(((row0 + tS) * 4 + slot) * d + jj, a.n_ps)) ? 4 : 0;
            cp_async4(&sm.S[st][r][slot][jl], bS ? a.S + ((row0 + tS) * 4 + slot) * d + jj : a.S, bS);
            if (r < TT) {
                const int bP = (fj && tP >= 0 && tP < T && SLSTM_IN(((row0 + tP) * 4 + slot) * d + jj, a.n_ps)) ? 4 : 0;
                cp_async4(&sm.P[st][r][slot][jl], bP ? a.P + ((row0 + tP) * 4 + slot) * d + jj : a.P, bP);
            }
        }
        for (int r = w; r < TT; r += NW) {
            const int t = t_lo + r;
            const int bH = (fj && t >= 0 && t < T && SLSTM_IN((row0 + t) * d + jj, a.n_ps / 4)) ? 4 : 0;
            cp_async4(&sm.dH[st][r][jl], bH ? a.dH + (row0 + t) * d + jj : a.dH, bH);
        }
    }
}

// TMA path, BWD_TMA_THREAD only: start the loads of one tile into stage st.
// Boxes that start before t = 0 or end past T - 1 read zeros there.
SLSTM_DEVINL void bwd_issue_load(const BwdArgs &a, const BwdMaps &m, BwdSmem &sm, int st, const BwdInfo &ti)
{
    if (ti.ticket >= (unsigned)a.n_tiles) return;
    const uint32_t rbytes = 4u * (uint32_t)min(32, a.d - ti.j0);
    mbar_expect_tx(&sm.bar[st], (uint32_t)(sizeof(sm.S[0]) + sizeof(sm.P[0]) + sizeof(sm.dH[0])) + 4u * rbytes);
    tma_load_3d(&sm.S[st][0][0][0], &m.S, &sm.bar[st], ti.j0, (ti.t_lo - 1) * 4, ti.b);
    tma_load_3d(&sm.P[st][0][0][0], &m.P, &sm.bar[st], ti.j0, ti.t_lo * 4, ti.b);
    tma_load_3d(&sm.dH[st][0][0], &m.H, &sm.bar[st], ti.j0, ti.t_lo, ti.b);
#pragma unroll
    for (int g = 0; g < 4; ++g)
        if (SLSTM_IN((size_t)g * a.d + ti.j0 + rbytes / 4 - 1, 4LL * a.d))
            bulk_load(&sm.R[st][g][0], a.R + (size_t)g * a.d + ti.j0, rbytes, &sm.bar[st]);
}

// TMA: tiles arrive by TMA (BWD_TMA_THREAD, mbarrier per stage); otherwise by
// cp.async.  BF16OUT: dP leaves as the transposed bf16 pair, else as fp32.
// VARLEN: packed ragged sequences (B = 1): J_{t+1} is zero when step t + 1
// starts a sequence, and a sequence's first step takes its s0 (and yields its
// ds0) as the dense kernel does at t = 0.
// MODE: as the Newton iteration's (BWD_FUSED: carry by decoupled look-back;
// BWD_AGG: store each tile's aggregate map only; BWD_APPLY: the fused pass
// with the carry entering every tile known from the scan of the aggregates).
constexpr int BWD_FUSED = 0, BWD_AGG = 1, BWD_APPLY = 2;

template <int FORGET, bool BF16OUT, bool TMA, bool VARLEN, int MODE>
__global__ void __launch_bounds__(NW * 32, 2) adjoint_vjp_kernel(BwdArgs a, const __grid_constant__ BwdMaps maps)
{
    extern __shared__ unsigned char smem_raw[];
    BwdSmem &sm = *reinterpret_cast<BwdSmem *>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const unsigned G = (unsigned)a.ca.n_groups;
    const int T = a.T;
    const size_t d = (size_t)a.d;
    const bool chain_warp = warp < 4;

    if (threadIdx.x == 0) {
        // BWD_AGG tiles are independent: a static order needs no counter
        bwd_decode(a, MODE == BWD_AGG ? blockIdx.x : atomicAdd(a.ticket, 1u), sm.info[0]);
        bwd_decode(a, MODE == BWD_AGG ? blockIdx.x + gridDim.x : atomicAdd(a.ticket, 1u), sm.info[1]);
    }
    if (TMA && threadIdx.x == BWD_TMA_THREAD) {
        mbar_init(&sm.bar[0], 1);
        mbar_init(&sm.bar[1], 1);
        mbar_init_fence();
    }
    __syncthreads();
    int ring = 0, st = 0;
    unsigned it = 0;
    bool tma_ok = true;
    if (TMA) {
        if (threadIdx.x == BWD_TMA_THREAD) bwd_issue_load(a, maps, sm, 0, sm.info[0]);
    } else {
        bwd_prefetch(a, sm, 0, sm.info[0]);
        cp_async_commit();
    }

    for (;;) {
        const BwdInfo ti = sm.info[ring];
        if (ti.ticket >= (unsigned)a.n_tiles) break;
        const int rn = ring == 2 ? 0 : ring + 1;
        unsigned after = 0;
        if (threadIdx.x == 0) after = MODE == BWD_AGG ? blockIdx.x + (it + 2u) * gridDim.x : atomicAdd(a.ticket, 1u);
        if (TMA) {
            if (tma_ok && !mbar_wait(&sm.bar[st], (it >> 1) & 1u, BWD_TMA_WAIT_NS)) {
                atomicOr(a.ca.error, 2u);
                (void)mbar_wait(&sm.bar[st], (it >> 1) & 1u, BWD_TMA_WAIT_NS);
                tma_ok = false;
            }
        } else {
            bwd_prefetch(a, sm, st ^ 1, sm.info[rn]);
            cp_async_commit();
            cp_async_wait_prev();
            __syncthreads();
        }

        const unsigned ticket = ti.ticket;
        const int chunk = ti.chunk;
        const bool jv = ti.j0 + lane < a.d;
        const size_t jj = jv ? (size_t)(ti.j0 + lane) : 0;
        const size_t row0 = (size_t)ti.b * T;
        const int t_lo = ti.t_lo;

        float rz = 0.f, ri = 0.f, rf = 0.f, ro = 0.f;
        if (TMA) {
            if (jv) {
                rz = sm.R[st][0][lane];
                ri = sm.R[st][1][lane];
                rf = sm.R[st][2][lane];
                ro = sm.R[st][3][lane];
            }
        } else if (jv && SLSTM_IN(3 * d + jj, 4 * d)) {
            rz = __ldg(a.R + jj);
            ri = __ldg(a.R + d + jj);
            rf = __ldg(a.R + 2 * d + jj);
            ro = __ldg(a.R + 3 * d + jj);
        }

        // looks at the predecessor's (later-in-time) inclusive prefix
        const bool look = MODE == BWD_FUSED && chain_warp && chunk > 0 && SLSTM_IN(ticket - G, a.n_tiles);
        const unsigned long long *predw = a.ca.incw + chain_word(ticket - G, warp, lane);
        unsigned long long w1 = 0ull, w2 = 0ull;
        if (look) w1 = ld_relaxed_u64(predw);

        // ---- walk A: fold kappa -> J_t^T (kappa + e_h dH_t), t descending ----
        // Each step's cell is evaluated here, once: J_t for the fold, the
        // factors of G_t and J_t (CellB) and h_{t-1} for walk B.  A sequence's
        // first step takes its s0 as the state before it; its J is the true
        // one (walk B forms ds0 from it), but what leaves it towards the
        // previous sequence is zero.  Rows before t = 0 (the last chunk only)
        // are zero-filled and come last in this order: nothing they reach is
        // stored.
        CellB cb[L];
        float hp[L];   // h_{t-1} of each step
        AffP agg;
#pragma unroll
        for (int i = 0; i < L; ++i) {
            if (i == L / 2 && look) w2 = ld_relaxed_u64(predw);
            const int rl = TT - 1 - (warp * L + i);   // t - t_lo
            const int t = t_lo + rl;
            float prev[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) prev[e] = sm.S[st][rl][e][lane];
            const bool head = VARLEN ? (((ti.hmask >> rl) & 1ull) != 0ull) : (t == 0);
            if (head) {
                const size_t sq = VARLEN ? (SLSTM_IN(t, T) ? (size_t)a.vseq[t] : 0) : (size_t)ti.b;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    prev[e] = (a.s0 && jv && SLSTM_IN((sq * 4 + e) * d + jj, a.n_s0)) ? __ldg(a.s0 + (sq * 4 + e) * d + jj)
                                                                                      : 0.f;
            }
            Cell J;
            cell_eval<FORGET, true, false, true>(prev[0], prev[1], prev[2], prev[3], sm.P[st][rl][0][lane],
                                                 sm.P[st][rl][1][lane], sm.P[st][rl][2][lane], sm.P[st][rl][3][lane],
                                                 rz, ri, rf, ro, J, nullptr, &cb[i]);
            hp[i] = prev[3];
            const bool reset = VARLEN && head;
            if (reset) cell_zero_jac(J);
            const float dh = sm.dH[st][rl][lane];
            const float r[4] = {J.jhc * dh, J.jhn * dh, J.jhm * dh, J.jhh * dh};   // J^T e_h dH_t
            if (i == 0 || reset) affp_from_cell<true>(agg, J, r);
            else fold_p<true>(agg, J, r);
        }
        maps_store(sm.u.m, warp, lane, agg);
        if (threadIdx.x == 0) bwd_decode(a, after, sm.info[rn == 2 ? 0 : rn + 1]);

        // warps whose steps contain a sequence start (bits rl of their steps)
        unsigned whead = 0u;
        if (VARLEN) {
#pragma unroll
            for (int w = 0; w < NW; ++w)
                whead |= (((ti.hmask >> (TT - L - w * L)) & ((1ull << L) - 1ull)) != 0ull) ? (1u << w) : 0u;
        }
        if constexpr (MODE == BWD_AGG) {
            if (TMA && threadIdx.x == BWD_TMA_THREAD) bwd_issue_load(a, maps, sm, st ^ 1, sm.info[rn]);
            // the tile's aggregate map: a tree over the warp maps in processing
            // order (at step h, warp w composes slot (2w+2)h - 1 with slot
            // (2w+1)h - 1 into the former; a part holding a reset ignores what
            // enters it and is kept as it is)
#pragma unroll
            for (int h = 1; h < NW; h *= 2) {
                __syncthreads();
                if (warp < NW / (2 * h)) {
                    const int hi = (2 * warp + 2) * h - 1, lo = (2 * warp + 1) * h - 1;
                    const bool hhead = VARLEN && (((whead >> ((2 * warp + 1) * h)) & ((1u << h) - 1u)) != 0u);
                    if (!hhead) {
                        Aff x, y;
                        maps_load(sm.u.m, hi, lane, x);
                        maps_load(sm.u.m, lo, lane, y);
                        aff_compose(x, y, x);
                        maps_store(sm.u.m, hi, lane, x);
                    }
                }
            }
            __syncthreads();
            if (warp == 0) {
                Aff x;
                maps_load(sm.u.m, NW - 1, lane, x);
                float *dst = a.ca.agg + (size_t)ticket * 20 * 32 + lane;
                if (SLSTM_IN(ticket, a.n_tiles)) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) dst[e * 32] = x.a[e];
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[(16 + e) * 32] = x.b[e];
                    if (lane == 0) a.ca.flags[ticket] = whead ? 1u : 0u;
                }
            }
        } else {

            // ---- carry ----
            float c = 0.f;   // chunk 0: nothing enters after the sequence's last step
            bool ok = true;
            if (MODE == BWD_APPLY && chain_warp && SLSTM_IN(chain_word(ticket, warp, lane), (long long)a.n_tiles * 128))
                c = a.cin_buf[chain_word(ticket, warp, lane)];
            if (look) {
                if ((unsigned)(w1 >> 32) == a.ca.epoch) {
                    c = __uint_as_float((unsigned)w1);
                } else {
                    ok = (unsigned)(w2 >> 32) == a.ca.epoch;
                    c = __uint_as_float((unsigned)w2);
                }
            }
            const bool fast = __syncthreads_and(ok);
            if (TMA && threadIdx.x == BWD_TMA_THREAD) bwd_issue_load(a, maps, sm, st ^ 1, sm.info[rn]);
            if (fast) {
                if (chain_warp) {
                    c = carry_chain4<NW>(sm.u.m, sm.cin, c, warp, lane, whead);
                    if (MODE == BWD_FUSED && SLSTM_IN(chain_word(ticket, warp, lane), (long long)a.n_tiles * 128))
                        st_relaxed_u64(a.ca.incw + chain_word(ticket, warp, lane), inc_word(a.ca.epoch, c));
                }
            } else if (warp == 0) {
                tile_carry_fallback<NW>(a.ca, sm.u.m, sm.cin, ticket, chunk, (int)(ticket - (unsigned)chunk * G), false,
                                        whead);
            }
            __syncthreads();   // every warp's carry is stored; the maps are dead from here on

            // ---- walk B: lambda_t = kappa_t + e_h dH_t, dP_t = G_t^T lambda_t,
            // kappa_{t-1} = J_t^T lambda_t ----
            float kap[4];
    #pragma unroll
            for (int e = 0; e < 4; ++e) kap[e] = sm.cin[warp][e][sw(e, lane)];
            float dr[4] = {0.f, 0.f, 0.f, 0.f}, dbs[4] = {0.f, 0.f, 0.f, 0.f};
            float dv[L][4];   // dP of the thread's steps (gate order z, i, f, o)
    #pragma unroll
            for (int i = 0; i < L; ++i) {
                const int rl = TT - 1 - (warp * L + i);
                const int t = t_lo + rl;
                const CellB &q = cb[i];
                const float lc = kap[0], ln = kap[1], lm = kap[2];
                const float lh = kap[3] + sm.dH[st][rl][lane];
                const float muc = fmaf(q.on, lh, lc);
                const float mun = fmaf(-q.ony, lh, ln);
                const float X = fmaf(q.gci, muc, q.gni * mun);
                const bool fb = __float_as_int(q.dlfs) >= 0;
                const float jtm = fb ? lm - X : -X;
                const float g[4] = {q.gcz * muc, fb ? X : lm + X, fabsf(q.dlfs) * jtm, q.gho * lh};
                kap[0] = q.fp * muc;
                kap[1] = q.fp * mun;
                kap[2] = jtm;
                kap[3] = fmaf(rz, g[0], fmaf(ri, g[1], fmaf(rf, g[2], ro * g[3])));
                const bool head = VARLEN ? (((ti.hmask >> rl) & 1ull) != 0ull) : (t == 0);
                if (head) {
                    // ds0 = J^T lambda at the sequence's first step; nothing
                    // enters the step before it (another sequence, or none)
                    const size_t sq = VARLEN ? (SLSTM_IN(t, T) ? (size_t)a.vseq[t] : 0) : (size_t)ti.b;
                    if (a.ds0 && jv && SLSTM_IN(sq * 4 * d + 3 * d + jj, a.n_s0)) {
                        float *qd = a.ds0 + sq * 4 * d + jj;
    #pragma unroll
                        for (int e = 0; e < 4; ++e) qd[e * d] = kap[e];
                    }
    #pragma unroll
                    for (int e = 0; e < 4; ++e) kap[e] = 0.0f;
                }
                const bool tv = t >= 0;   // steps before 0 (last chunk only) contribute nothing
    #pragma unroll
                for (int e = 0; e < 4; ++e) dv[i][e] = tv ? g[e] : 0.f;
                if (!BF16OUT && jv && tv && SLSTM_IN((row0 + t) * 4 * d + 3 * d + jj, a.n_ps)) {
                    float *pd = a.dP + (row0 + t) * 4 * d + jj;
    #pragma unroll
                    for (int e = 0; e < 4; ++e) pd[e * d] = dv[i][e];
                }
    #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    dr[e] = fmaf(dv[i][e], hp[i], dr[e]);
                    dbs[e] += dv[i][e];
                }
            }
            // the dP staging takes the dead maps' place
    #pragma unroll
            for (int e = 0; e < 4; ++e) {
                sm.u.o.part[warp][e][lane] = jv ? dr[e] : 0.f;
                sm.u.o.part[warp][4 + e][lane] = jv ? dbs[e] : 0.f;
            }
            if (BF16OUT) {
                // the thread's 4 steps are 4 consecutive t: t_lo + 28 - 4w .. t_lo + 31 - 4w
                const int rb = TT - L - warp * L;
    #pragma unroll
                for (int gi = 0; gi < 4; ++gi) {
                    const __nv_bfloat162 h01 = __floats2bfloat162_rn(dv[3][gi], dv[2][gi]);
                    const __nv_bfloat162 h23 = __floats2bfloat162_rn(dv[1][gi], dv[0][gi]);
                    const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
                    const __nv_bfloat162 l01 = __floats2bfloat162_rn(dv[3][gi] - f01.x, dv[2][gi] - f01.y);
                    const __nv_bfloat162 l23 = __floats2bfloat162_rn(dv[1][gi] - f23.x, dv[0][gi] - f23.y);
                    uint2 hv, lv;
                    hv.x = *reinterpret_cast<const unsigned *>(&h01);
                    hv.y = *reinterpret_cast<const unsigned *>(&h23);
                    lv.x = *reinterpret_cast<const unsigned *>(&l01);
                    lv.y = *reinterpret_cast<const unsigned *>(&l23);
                    *reinterpret_cast<uint2 *>(&sm.u.o.dpt[0][gi][lane][rb]) = hv;
                    *reinterpret_cast<uint2 *>(&sm.u.o.dpt[1][gi][lane][rb]) = lv;
                }
            }
            __syncthreads();
            {
                // 256 threads: thread (e, lane) sums entry e over the warps
                const int e = threadIdx.x >> 5;   // 0..7
                float acc = 0.f;
    #pragma unroll
                for (int w = 0; w < NW; ++w) acc += sm.u.o.part[w][e][lane];
                if (SLSTM_IN(ticket, a.n_tiles)) a.partial[((size_t)ticket * 8 + e) * 32 + lane] = acc;
            }
            if (BF16OUT) {
                // rows (part, gate, feature) of the transposed pair, 32 steps each;
                // nothing before t = 0 (those addresses hold the previous batch row)
                if (a.dpt_vec8) {
                    // 8-byte pieces of 4 steps: thread (feature jl, piece q) copies
                    // piece q of the 8 rows (part, gate) of feature jl
                    static_assert(NW * 32 == 256, "one thread per (feature, piece)");
                    const int q = threadIdx.x & 7, jl = threadIdx.x >> 3;
                    const int t = t_lo + 4 * q;
                    if (t >= 0 && ti.j0 + jl < a.d) {
                        const size_t base = (size_t)(ti.j0 + jl) * a.ldT + row0 + t;
                        const size_t gstride = d * (size_t)a.ldT;
    #pragma unroll
                        for (int part = 0; part < 2; ++part) {
                            __nv_bfloat16 *dst = (part ? a.dpt_lo : a.dpt_hi) + base;
    #pragma unroll
                            for (int gi = 0; gi < 4; ++gi)
                                if (SLSTM_IN(base + gi * gstride + 3, a.n_dpt))
                                    *reinterpret_cast<uint2 *>(dst + gi * gstride) =
                                        *reinterpret_cast<const uint2 *>(&sm.u.o.dpt[part][gi][jl][4 * q]);
                        }
                    }
                } else {
                    const int tl = threadIdx.x & 31;
                    const int t = t_lo + tl;
                    for (int r = warp; r < 2 * 4 * 32; r += NW) {
                        const int part = r >> 7, gi = (r >> 5) & 3, jl = r & 31;
                        if (t >= 0 && ti.j0 + jl < a.d &&
                            SLSTM_IN(((size_t)gi * d + ti.j0 + jl) * a.ldT + row0 + t, a.n_dpt)) {
                            __nv_bfloat16 *dst = part ? a.dpt_lo : a.dpt_hi;
                            dst[((size_t)gi * d + ti.j0 + jl) * a.ldT + row0 + t] = sm.u.o.dpt[part][gi][jl][tl];
                        }
                    }
                }
            }
        }
        __syncthreads();   // the staging and the stage are free again
        ring = rn;
        st ^= 1;
        ++it;
    }
    if (!TMA) cp_async_wait_all();
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

}  // namespace

cudaError_t sum_splits(const float *part, float *out, long long n, int splits, cudaStream_t st)
{
    sum_splits_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(part, out, n, splits);
    return cudaGetLastError();
}

namespace {

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
        if (SLSTM_IN(ticket, (long long)n_chunks * G)) acc += partial[(ticket * 8 + e) * 32 + lane];
    }
    s_sum[warp][lane] = acc;
    __syncthreads();
    if (warp == 0) {
        double t = 0.0;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += s_sum[w][lane];
        const int j = jb * 32 + lane;
        if (j < d && SLSTM_IN((size_t)(e & 3) * d + j, 4LL * d)) {
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

template <int FORGET, bool BF16OUT, bool TMA, bool VARLEN, int MODE>
cudaError_t launch_adjoint_mode(const BwdArgs &a, const BwdMaps &m, cudaStream_t st)
{
    auto kern = adjoint_vjp_kernel<FORGET, BF16OUT, TMA, VARLEN, MODE>;
    static int blocks_per_sm = 0;
    if (blocks_per_sm == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BWD_SMEM_BYTES);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, kern, NW * 32, BWD_SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (blocks_per_sm < 1) blocks_per_sm = 1;
    }
    const int grid = min(a.n_tiles, sm_count_bwd() * blocks_per_sm);
    kern<<<grid, NW * 32, BWD_SMEM_BYTES, st>>>(a, m);
    return cudaGetLastError();
}

// Scratch of the two-pass carry (null scan.cin: one fused pass).
struct TwoPass {
    TileScanArgs scan;
};

template <int FORGET, bool BF16OUT, bool TMA, bool VARLEN>
cudaError_t launch_adjoint(const BwdArgs &a, const BwdMaps &m, const TwoPass &tp, cudaStream_t st)
{
    if (!tp.scan.cin) return launch_adjoint_mode<FORGET, BF16OUT, TMA, VARLEN, BWD_FUSED>(a, m, st);
    cudaError_t e = launch_adjoint_mode<FORGET, BF16OUT, TMA, VARLEN, BWD_AGG>(a, m, st);
    if (e == cudaSuccess) e = launch_tile_scan(tp.scan, st);
    if (e == cudaSuccess) e = launch_adjoint_mode<FORGET, BF16OUT, TMA, VARLEN, BWD_APPLY>(a, m, st);
    return e;
}

template <int FORGET, bool VARLEN>
cudaError_t launch_adjoint_v(const BwdArgs &a, const BwdMaps &m, const TwoPass &tp, bool tma, bool bf16out,
                             cudaStream_t st)
{
    if (tma)
        return bf16out ? launch_adjoint<FORGET, true, true, VARLEN>(a, m, tp, st)
                       : launch_adjoint<FORGET, false, true, VARLEN>(a, m, tp, st);
    return bf16out ? launch_adjoint<FORGET, true, false, VARLEN>(a, m, tp, st)
                   : launch_adjoint<FORGET, false, false, VARLEN>(a, m, tp, st);
}

template <int FORGET>
cudaError_t launch_adjoint_any(const BwdArgs &a, const BwdMaps &m, const TwoPass &tp, bool tma, bool bf16out,
                               bool varlen, cudaStream_t st)
{
    return varlen ? launch_adjoint_v<FORGET, true>(a, m, tp, tma, bf16out, st)
                  : launch_adjoint_v<FORGET, false>(a, m, tp, tma, bf16out, st);
}

struct Layout {
    size_t ticket, flags, incw, agg, partial, dP, dpt, wpart, err, cin, blk_agg, blk_head, blk_cin, total;
    int groups_per_row, n_groups, n_chunks, n_tiles, splits;
    long long n, ldT, ld4;
};

long long round8(long long v) { return (v + 7) & ~7LL; }

// split-K count of the W_x-gradient GEMM: the count (up to 16) whose work
// items fill whole waves of the persistent CTAs (or CTA pairs) best; a larger count only
// when it fills them at least 2% better (each split adds an M x N partial).
int wgrad_splits(int B, int T, int d_in, int d_h)
{
    int rows = 128, units = 148;
    gemm_tc_waves(&rows, &units);
    const long long tiles = ((4LL * d_h + rows - 1) / rows) * ((d_in + 255) / 256);
    const long long sms = units;
    int best = 1;
    double best_eff = 0.0;
    for (int want = 1; want <= 16; ++want) {
        const int s = gemm_tc_splits(4 * d_h, d_in, B * T, 2, want);
        const long long work = tiles * s;
        const double eff = (double)work / (double)(((work + sms - 1) / sms) * sms);
        if (eff > best_eff + 0.02) {
            best_eff = eff;
            best = s;
        }
    }
    return best;
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
    l.cin = take(sizeof(float) * 4 * 32 * (size_t)l.n_tiles);
    const size_t nblk = (size_t)l.n_groups * scan_blocks(l.n_chunks);
    l.blk_agg = take(sizeof(float) * 20 * 32 * nblk);
    l.blk_head = take(sizeof(unsigned) * nblk);
    l.blk_cin = take(sizeof(float) * 4 * 32 * nblk);
    l.total = off;
    return l;
}

}  // namespace

size_t backward_workspace_bytes(int B, int T, int d_in, int d_h) { return layout(B, T, d_in, d_h).total; }

cudaError_t backward_launch(const void *x, const void *Wx, int dtype, const float *P, const float *R,
                            const float *s0, const float *S, const float *dH, float *dx, float *dWx,
                            float *dR, float *db, float *ds0, int forget, int B, int T, int d_in,
                            int d_h, void *ws, cudaStream_t st, const Varlen *vl)
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
    a.n_ps = l.n;
    a.n_dpt = 4LL * d_h * l.ldT;
    a.n_s0 = (long long)(vl ? vl->n_seq : B) * 4 * d_h;
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
    a.ca.n_tiles = l.n_tiles;
    a.T = T;
    a.d = d_h;
    a.groups_per_row = l.groups_per_row;
    a.div_groups = make_fastdiv((unsigned)l.n_groups);
    a.div_gpr = make_fastdiv((unsigned)l.groups_per_row);
    a.n_tiles = l.n_tiles;
    a.dpt_vec8 = (T % 4 == 0) ? 1 : 0;   // 8-byte pieces of the transposed pair stay aligned
    a.vec16 = ((d_h & 3) == 0 && (reinterpret_cast<uintptr_t>(S) & 15) == 0 &&
               (reinterpret_cast<uintptr_t>(P) & 15) == 0 && (reinterpret_cast<uintptr_t>(dH) & 15) == 0) ? 1 : 0;
    // ticket, error word, flags and the epoch tags of the inclusive prefixes
    // start cleared
    cudaError_t e = cudaMemsetAsync(base, 0, l.agg, st);
    if (e != cudaSuccess) return e;
    a.vmask = nullptr;
    a.vseq = nullptr;
    if (vl) {
        if ((e = varlen_build(*vl, T, nullptr, nullptr, st)) != cudaSuccess) return e;
        a.vmask = vl->mask;
        a.vseq = vl->seq;
        // empty sequences get a zero ds0; the others are written at their first step
        if (ds0 && (e = cudaMemsetAsync(ds0, 0, sizeof(float) * 4 * (size_t)d_h * vl->n_seq, st)) != cudaSuccess)
            return e;
    }
    // TMA moves the tiles when the rows are 16-byte aligned and every row
    // coordinate fits a signed 32-bit box coordinate
    BwdMaps m;
    memset(&m, 0, sizeof(m));
    const uint64_t rows = 4 * (uint64_t)T;
    const bool tma = a.vec16 && (reinterpret_cast<uintptr_t>(R) & 15) == 0 && rows < (1ull << 31) &&
                     make_map_f32_3d(&m.S, S, d_h, rows, B, d_h, rows * d_h, 32, (TT + 1) * 4) &&
                     make_map_f32_3d(&m.P, P, d_h, rows, B, d_h, rows * d_h, 32, TT * 4) &&
                     make_map_f32_3d(&m.H, dH, d_h, T, B, d_h, (uint64_t)T * d_h, 32, TT);
    // few feature groups and a long time axis: two passes with a scan of the
    // tile aggregates in between instead of waiting for predecessors
    TwoPass tp;
    memset(&tp, 0, sizeof(tp));
    a.cin_buf = nullptr;
    if (prefer_two_pass(l.n_groups, (long long)l.n_chunks * TT, sm_count_bwd())) {
        a.cin_buf = reinterpret_cast<float *>(base + l.cin);
        tp.scan = TileScanArgs{a.ca.agg, a.ca.flags, reinterpret_cast<float *>(base + l.blk_agg),
                               reinterpret_cast<unsigned *>(base + l.blk_head), reinterpret_cast<float *>(base + l.blk_cin),
                               a.cin_buf, nullptr, l.n_groups, l.n_chunks, scan_blocks(l.n_chunks)};
    }
    e = (forget == SLSTM_FORGET_EXP) ? launch_adjoint_any<SLSTM_FORGET_EXP>(a, m, tp, tma, tc, vl != nullptr, st)
                                     : launch_adjoint_any<SLSTM_FORGET_SIGMOID>(a, m, tp, tma, tc, vl != nullptr, st);
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
