// The Newton solve's stopping rule, shared by the diag and head-mixing
// iterations ("pararnn-torch structure", section "Current surface":
// NewtonStats, residual early stop, NewtonDivergenceError if max|F| > 1
// after K).  Launch k of a call is Newton iteration n = k - k0 (k0 launches,
// the initial guess, come first); iteration n uses control slot k & 1, and
// the CTA that finishes it last calls finalize_iteration.
#pragma once

#include <float.h>

#include "launchers.h"

namespace slstm {

struct StopRule {
    NewtonCtrl *ctrl;
    slstm_newton_stats *stats;
    int k0;             // launches before the first Newton iteration
    int max_iters;
    int fixed;          // run exactly max_iters iterations
    int resid_raw;      // test max|F| (else the scaled residual)
    int guess_tested;   // the first iteration recorded the guess's residual in ctrl
    float tol;
};

__device__ inline void finalize_iteration(const StopRule &a, int k, bool resid)
{
    NewtonCtrl *c = a.ctrl;
    slstm_newton_stats *st = a.stats;
    NewtonSlot &s = c->slot[k & 1];
    const float raw = __uint_as_float(atomicOr(&s.maxF_raw, 0u));
    const float sc = __uint_as_float(atomicOr(&s.maxF_scaled, 0u));
    const unsigned err = atomicOr(&c->error, 0u);
    const int n = k - a.k0;
    const bool last = (n + 1 == a.max_iters);
    // the next iteration starts from a clean slot (its previous user,
    // iteration k - 1, finished before this launch began)
    NewtonSlot &nx = c->slot[(k + 1) & 1];
    nx.ticket = 0u;
    nx.finished = 0u;
    nx.maxF_raw = 0u;
    nx.maxF_scaled = 0u;
    nx.failed = 0u;
    st->iters = n + 1;
    st->max_abs_F[n % SLSTM_STATS_HISTORY] = resid ? raw : -1.0f;
    st->max_scaled_F[n % SLSTM_STATS_HISTORY] = resid ? sc : -1.0f;
    if (n == 0) {
        st->init_max_abs_F = a.guess_tested ? __uint_as_float(atomicOr(&c->init_raw, 0u)) : -1.0f;
        st->init_max_scaled_F = a.guess_tested ? __uint_as_float(atomicOr(&c->init_scaled, 0u)) : -1.0f;
    }
    const float test = a.resid_raw ? raw : sc;
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
        } else if (test <= a.tol && (!a.fixed || last)) {
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

}  // namespace slstm
