// Fused Newton iteration for the diag-mix sLSTM.
//
// One launch is one Newton iteration ("sLSTM in this library", section
// "Cell": the fused diag training cell runs Newton with a 4x4 Jacobian per
// feature and an O(d) combine; "pararnn-torch structure", section "Current
// surface": fused kernels prepend h0, residual early stop, divergence after
// K).  The iteration is tiled: a tile is 32 features x 64 steps, handled by
// one CTA of 16 warps (lane = feature, warp = 4 consecutive steps).
//
// Persistent CTAs walk the tiles in ticket order and keep the next tile's P
// and old S arriving in shared memory (TMA, or cp.async when rows are not
// 16-byte aligned; double buffered) while they work on the current one:
//   walk A  each thread recomputes gates, stabilizer, f(S_{t-1}, P_t) and the
//           4x4 Jacobian J_t in registers for its 4 steps, keeps (J_t, r_t =
//           f - S_t) in registers and folds the maps delta -> J_t delta + r_t;
//   carry   the carry entering the tile is the predecessor tile's inclusive
//           prefix (looked at twice: before and after walk A); the last four
//           warps apply the 16 warp maps to it, one (feature, slot) pair per
//           lane, release every other warp as soon as the carry entering it
//           is stored, and publish this tile's prefix; a tile whose
//           predecessor has not published falls back to the look-back in
//           lookback.cuh;
//   walk B  each thread replays its steps from its carry, writes S + delta in
//           place and, when asked, accumulates the residual of the new
//           iterate for the stopping test.
//
// In-place update is safe because the only value a tile reads from another
// tile (the state just before it) comes from a per-tile boundary buffer
// written by the previous launch.
#include <float.h>
#include <string.h>

#include <type_traits>

#define SLSTM_FILE_ID 1
#include "launchers.h"
#include "lookback.cuh"
#include "stop_rule.cuh"
#include "tma.cuh"

namespace slstm {
namespace {

constexpr int NW = 16;   // warps per tile (time segments)
// Guess stages (the decoupled guess and its sweeps) that one launch runs per
// tile; each has its own look-back state (flags, runs in the aggregate
// buffer, published states).
constexpr int GUESS_STAGES = 4;
// How a launch gets the carry entering each tile.  FUSED: from the tile
// before it in the same launch (decoupled look-back).  With few feature
// groups most tiles would wait on their predecessors, so an iteration can
// instead run as two passes over the tiles with a scan in between: AGG
// stores each tile's aggregate map, a blocked scan (scan_block_agg,
// scan_block_carry, scan_tile_carry) turns the aggregates of every feature
// group into the carry entering each tile, and APPLY is the fused iteration
// with that carry known.
constexpr int MODE_FUSED = 0, MODE_AGG = 1, MODE_APPLY = 2;
constexpr int L = 4;    // steps per thread
constexpr int TT = NW * L;

struct Args {
    const float *P;
    const float *R;
    const float *s0;
    const float *s0h;             // sweeps: the state whose h the gates of step 0 see (s0, or a time slice's
                                  // previous guess just before it)
    float *S;
    NewtonCtrl *ctrl;
    unsigned *flags;              // [n_tiles] aggregate-published flags
    float *agg;                   // [n_tiles][20][32]
    unsigned long long *incw;     // [n_tiles][4][32] (value bits | epoch << 32)
    float *bnd_in;                // [n_tiles][4][32] S of the previous iterate at each tile's last step
    float *bnd_out;
    float *cin_buf;               // two-pass carry: [n_tiles][4][32] carry entering each tile (chain layout)
    float *blk_agg;               // two-pass scan scratch (see scan_block_agg)
    unsigned *blk_head;
    float *blk_cin;
    slstm_newton_stats *stats;
    unsigned *error;
    const unsigned *vmask;        // packed sequences: head-flag words (one per 32 steps), else null
    const int *vseq;              // packed sequences: sequence index at each head step
    unsigned epoch;
    unsigned long long wait_ns;
    int B, T, d, groups_per_row, n_groups, n_tiles, max_iters, fixed, fault_ticket, vec16;
    int k0;             // launches before the first Newton iteration (the guess and its sweeps)
    int guess_sweeps;   // refinement sweeps of the decoupled guess
    int resid_raw;      // stopping test on max|F| (else on the scaled residual)
    int exact_hist;     // every iteration evaluates its whole residual (else a failed test ends that work)
    int guess_tested;   // the first iteration records the residual of the guess
    int check_plant;    // checked build: one bounds check made to fail on purpose (a self-test)
    int loop_from;      // tolerance mode, fused carry: iterations from this one on loop on the device (0: never)
    int loop_fault;     // self-test: CTA 0 of the device loop leaves before its first grid barrier
    float tol;
    long long n_s0;     // elements of s0 (and of s0h)
    FastDiv div_groups, div_gpr;   // by n_groups and by groups_per_row
};

// Launch k of a solve: epoch k + 1; it reads the boundary buffer launch
// k - 1 wrote and writes the other one.  (On the device: the iterations of
// newton_iter_loop.)
__host__ __device__ inline Args launch_args(const Args &base, int k)
{
    Args a = base;
    a.epoch = (unsigned)(k + 1);
    a.bnd_in = (k & 1) ? base.bnd_out : base.bnd_in;
    a.bnd_out = (k & 1) ? base.bnd_in : base.bnd_out;
    return a;
}

// Element counts of the buffers that Args names, for the guards of the
// checked build.
[[maybe_unused]] SLSTM_DEVINL long long ext_ps(const Args &a) { return (long long)a.B * a.T * 4 * a.d; }
[[maybe_unused]] SLSTM_DEVINL long long ext_tiles(const Args &a) { return (long long)a.n_tiles * 128; }
#define SLSTM_RANGE(p, base, n, cnt) (SLSTM_PIN(p, base, n) && SLSTM_PIN((p) + (cnt) - 1, base, n))

// A ticket decoded once (by thread 0) for the whole CTA.
struct TileInfo {
    unsigned ticket;
    int chunk;
    int b;
    int j0;
    unsigned long long off;    // element offset of (b, chunk * TT, slot 0, feature j0) in P and S
    unsigned long long mask;   // packed sequences: bit i set when step chunk * TT + i starts a sequence
};

struct Smem {
    float P[2][TT][4][32];   // stage s: rows (step, slot) of 32 features; TMA boxes land here
    float S[2][TT][4][32];
    float O[TT][4][32];    // TMA path: S_new of the tile, source of the warps' TMA stores
    float R[2][4][32];     // TMA path: the tile's recurrent weights (gate-major)
    float bnd[2][4][32];   // TMA path: S_old just before the tile (previous launch's boundary)
    TileMaps<NW> maps;
    TileInfo info[3];   // ring: current, next and the one after
    uint64_t bar[2];    // TMA completion, one per stage
    float red[2][NW];
    int exit_flag;
    int resid_skip;     // this tile: the iteration's test has already failed elsewhere
};
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;   // + room to align the stages to 1 KB
// Warps CHAIN0 .. NW-1 walk the carry through the warp maps (chain lanes);
// warp w < CHAIN0 starts walk B as soon as the carry entering it is stored
// (named barrier 1 + w), the chain warps themselves after CHAIN_BAR.
constexpr int CHAIN0 = NW - 4;
constexpr int CHAIN_BAR = CHAIN0 + 1;   // the chain warps' own barrier (ids 1 .. CHAIN0 are per warp)
constexpr int TMA_THREAD = (CHAIN0 - 1) * 32;   // issues the first tile's loads (a warp with no chain lane)
constexpr int TMA_WARP0 = CHAIN0 - 4;           // lane 0 of warps TMA_WARP0 .. +3 issue the later tiles' loads
constexpr uint64_t TMA_WAIT_NS = 1000000000ull;

// Tensor maps of P and S viewed as (d, 4T, B): boxes of 32 features x 128
// (step, slot) rows for the tile loads, 32 x 16 rows for a warp's stores.
struct NewtonMaps {
    CUtensorMap P, S, Sw;
    CUtensorMap H;   // S as (d, 4, T, B): boxes of 32 features x 1 slot x 64 steps (the guess sweeps' h rows)
};

// TMA_THREAD only: start the loads of one tile into stage `st`: the P (and
// S_old) boxes, the R entries of its features and, after the first launch,
// the boundary state before it, all counted on the stage's mbarrier.
SLSTM_DEVINL void issue_tile_load(const Args &a, const NewtonMaps &m, Smem &sm, int st, const TileInfo &ti, bool with_s)
{
    if (ti.ticket >= (unsigned)a.n_tiles) return;
    const int row = ti.chunk * TT * 4;
    const uint32_t rbytes = 4u * (uint32_t)min(32, a.d - ti.j0);   // a multiple of 16 (d % 4 == 0)
    const bool bnd = with_s && ti.chunk > 0;
    mbar_expect_tx(&sm.bar[st], (with_s ? 2u : 1u) * (uint32_t)sizeof(sm.P[0]) + 4u * rbytes +
                                    (bnd ? (uint32_t)sizeof(sm.bnd[0]) : 0u));
    tma_load_3d(&sm.P[st][0][0][0], &m.P, &sm.bar[st], ti.j0, row, ti.b);
    if (with_s) tma_load_3d(&sm.S[st][0][0][0], &m.S, &sm.bar[st], ti.j0, row, ti.b);
#pragma unroll
    for (int g = 0; g < 4; ++g)
        if (SLSTM_RANGE(a.R + (size_t)g * a.d + ti.j0, a.R, 4LL * a.d, rbytes / 4))
            bulk_load(&sm.R[st][g][0], a.R + (size_t)g * a.d + ti.j0, rbytes, &sm.bar[st]);
    if (bnd && SLSTM_RANGE(a.bnd_in + (size_t)(ti.ticket - (unsigned)a.n_groups) * 4 * 32, a.bnd_in, ext_tiles(a), 128))
        bulk_load(&sm.bnd[st][0][0], a.bnd_in + (size_t)(ti.ticket - (unsigned)a.n_groups) * 4 * 32,
                  (uint32_t)sizeof(sm.bnd[0]), &sm.bar[st]);
}

// The same loads split over four issuing threads (lane 0 of warps
// TMA_WARP0 .. TMA_WARP0 + 3), so that no single warp starts its walk late:
// part 0 announces the stage's bytes and loads P, part 1 S_old, part 2 the R
// rows, part 3 the boundary block.  Bytes may land before they are announced.
SLSTM_DEVINL void issue_tile_load_part(const Args &a, const NewtonMaps &m, Smem &sm, int st, const TileInfo &ti,
                                       bool with_s, int part)
{
    if (ti.ticket >= (unsigned)a.n_tiles) return;
    const int row = ti.chunk * TT * 4;
    const uint32_t rbytes = 4u * (uint32_t)min(32, a.d - ti.j0);
    const bool bnd = with_s && ti.chunk > 0;
    if (part == 0) {
        mbar_expect_tx(&sm.bar[st], (with_s ? 2u : 1u) * (uint32_t)sizeof(sm.P[0]) + 4u * rbytes +
                                        (bnd ? (uint32_t)sizeof(sm.bnd[0]) : 0u));
        tma_load_3d(&sm.P[st][0][0][0], &m.P, &sm.bar[st], ti.j0, row, ti.b);
    } else if (part == 1) {
        if (with_s) tma_load_3d(&sm.S[st][0][0][0], &m.S, &sm.bar[st], ti.j0, row, ti.b);
    } else if (part == 2) {
#pragma unroll
        for (int g = 0; g < 4; ++g)
            if (SLSTM_RANGE(a.R + (size_t)g * a.d + ti.j0, a.R, 4LL * a.d, rbytes / 4))
                bulk_load(&sm.R[st][g][0], a.R + (size_t)g * a.d + ti.j0, rbytes, &sm.bar[st]);
    } else if (bnd && SLSTM_RANGE(a.bnd_in + (size_t)(ti.ticket - (unsigned)a.n_groups) * 4 * 32, a.bnd_in,
                                  ext_tiles(a), 128)) {
        bulk_load(&sm.bnd[st][0][0], a.bnd_in + (size_t)(ti.ticket - (unsigned)a.n_groups) * 4 * 32,
                  (uint32_t)sizeof(sm.bnd[0]), &sm.bar[st]);
    }
}

SLSTM_DEVINL void decode_tile(const Args &a, unsigned ticket, TileInfo &ti)
{
    ti.ticket = ticket;
    ti.chunk = ti.b = ti.j0 = 0;
    ti.off = 0;
    ti.mask = 0ull;
    if (ticket < (unsigned)a.n_tiles) {
        const unsigned chunk = fast_div(ticket, a.div_groups);
        const unsigned grp = ticket - chunk * (unsigned)a.n_groups;
        const unsigned b = fast_div(grp, a.div_gpr);
        ti.chunk = (int)chunk;
        ti.b = (int)b;
        ti.j0 = (int)(grp - b * (unsigned)a.groups_per_row) * 32;
        ti.off = ((size_t)b * a.T + (size_t)chunk * TT) * 4 * (size_t)a.d + (size_t)ti.j0;
        if (a.vmask) {
            // head flags of steps chunk * TT .. chunk * TT + TT - 1, from the
            // words of 32 steps that hold them
            const unsigned t0 = chunk * (unsigned)TT;
            const unsigned nwords = ((unsigned)a.T + 31u) >> 5;
            unsigned long long mk = 0ull;
#pragma unroll
            for (int q = 0; q < (TT + 31) / 32; ++q)
                if ((t0 >> 5) + q < nwords) mk |= (unsigned long long)a.vmask[(t0 >> 5) + q] << (32 * q);
            if constexpr (TT < 32) mk = (mk >> (t0 & 31u)) & ((1ull << (TT % 32)) - 1ull);
            ti.mask = mk;
        }
    }
}

// Packed sequences: the initial state of the sequence that starts at step t.
SLSTM_DEVINL void head_state(const Args &a, int t, size_t jj, bool jv, float s[4])
{
    const size_t k = SLSTM_IN(t, a.T) ? (size_t)a.vseq[t] : 0;
#pragma unroll
    for (int e = 0; e < 4; ++e)
        s[e] = (a.s0 && jv && SLSTM_IN((k * 4 + e) * (size_t)a.d + jj, a.n_s0))
                   ? __ldg(a.s0 + (k * 4 + e) * (size_t)a.d + jj) : 0.0f;
}

// Per-thread part of the copy offsets (see prefetch_tile).
SLSTM_DEVINL size_t prefetch_offset(const Args &a)
{
    const int w = threadIdx.x >> 5;
    if (a.vec16) return (size_t)(w * 4 + ((threadIdx.x >> 3) & 3)) * a.d + 4 * (threadIdx.x & 7);
    return (size_t)w * a.d + (threadIdx.x & 31);
}

// Issue the copies of one tile's P (and old S unless `with_s` is false) into
// shared-memory stage `st`.  Rows past T and features past d read nothing and
// arrive as zeros.  `toff` = prefetch_offset(a).
SLSTM_DEVINL void prefetch_tile(const Args &a, Smem &sm, int st, const TileInfo &ti, size_t toff, bool with_s)
{
    if (ti.ticket >= (unsigned)a.n_tiles) return;
    const int t0 = ti.chunk * TT;
    const int w = threadIdx.x >> 5;
    const float *p = a.P + ti.off + toff;
    const float *s = a.S + ti.off + toff;
    if (a.vec16) {
        // 8 chunks of 16 bytes per (step, slot) row of 32 features; thread
        // (w, slot, c) copies chunk c of slot `slot` for steps w, w + NW, ...
        const int c = threadIdx.x & 7, slot = (threadIdx.x >> 3) & 3;
        const int rem = a.d - ti.j0 - 4 * c;
        const int fbytes = rem > 0 ? 4 * min(4, rem) : 0;
        const size_t stepw = (size_t)NW * 4 * a.d;   // NW steps of 4 slots
#pragma unroll
        for (int r = 0; r < L; ++r) {
            const int step = r * NW + w;
            const int bytes = (t0 + step < a.T && SLSTM_RANGE(p + r * stepw, a.P, ext_ps(a), fbytes / 4)) ? fbytes : 0;
            cp_async16(&sm.P[st][step][slot][4 * c], bytes ? p + r * stepw : a.P, bytes);
            if (with_s) cp_async16(&sm.S[st][step][slot][4 * c], bytes ? s + r * stepw : a.S, bytes);
        }
    } else {
        // 4-byte copies, lane = feature; warp w copies rows w, w + NW, ... of
        // the 4 TT (step, slot) rows
        const int jl = threadIdx.x & 31;
        const bool fj = ti.j0 + jl < a.d;
        const size_t roww = (size_t)NW * a.d;
#pragma unroll 4
        for (int r = 0; r < 4 * L; ++r) {
            const int rs = r * NW + w;
            const int step = rs >> 2, slot = rs & 3;
            const int bytes = (fj && t0 + step < a.T && SLSTM_PIN(p + r * roww, a.P, ext_ps(a))) ? 4 : 0;
            cp_async4(&sm.P[st][step][slot][jl], bytes ? p + r * roww : a.P, bytes);
            if (with_s) cp_async4(&sm.S[st][step][slot][jl], bytes ? s + r * roww : a.S, bytes);
        }
    }
}

// Last CTA of launch k: records the residual of Newton iteration k - k0
// and decides whether the solve goes on (stop_rule.cuh).
__device__ void finalize(const Args &a, int k, bool resid)
{
    const StopRule r{a.ctrl, a.stats, a.k0, a.max_iters, a.fixed, a.resid_raw, a.guess_tested, a.tol};
    finalize_iteration(r, k, resid);
}

// ---- the decoupled initial guess --------------------------------------------
// The default initial guess is the trajectory of the cell with its gates
// blind to h_{t-1} (R taken as 0): z, o, log i and log f then depend on P
// alone and only c, n, m recur.  In unstabilised form (C, N) = (c, n) e^m that
// recurrence is linear, C_t = f_t C_{t-1} + i_t z_t, so a run of steps maps
// (C, N) to e^A (C, N) + e^mu (u, v) with A = sum log f, and the guess is an
// associative scan over such runs, kept stabilised: the run is stored as
// (A, mu, u, v) with mu the largest exponent of its own inputs.  The launch
// has the Newton iteration's tiles, tickets and look-back, with five floats
// per run instead of a 4x4 affine map, reads P and writes S (and the tile
// boundary states the first Newton iteration reads).

// A run of steps.  head: the run contains a sequence start, so its result
// ignores what enters it; (mu, u, v) then hold the state (m, c, n) at its
// end and A is unused.
struct Seg {
    float A, mu, u, v;
    float o;      // output gate of the run's last step (h = o c / n there)
    bool head;
};

// (m, c, n) <- the run (A, mu, u, v) applied to the state (m, c, n):
//   m' = max(A + m, mu),  (c', n') = e^{A + m - m'} (c, n) + e^{mu - m'} (u, v).
// With (A, mu, u, v) = (log f_t, log i_t, z_t, 1) this is one step of the cell
// with R = 0, ties going to the forget branch as in the cell.
SLSTM_DEVINL void seg_apply(float A, float mu, float u, float v, float &m, float &c, float &n)
{
    const float x = A + m;
    const bool fb = x >= mu;
    const float e = __expf(-fabsf(x - mu));
    const float f1 = fb ? 1.0f : e;
    const float f2 = fb ? e : 1.0f;
    m = fb ? x : mu;
    c = fmaf(f1, c, f2 * u);
    n = fmaf(f1, n, f2 * v);
}

// out = second o first (the run `first`, then the run `second`).
SLSTM_DEVINL void seg_compose(const Seg &second, const Seg &first, Seg &out)
{
    if (second.head) {
        out = second;
        return;
    }
    Seg r = first;
    seg_apply(second.A, second.mu, second.u, second.v, r.mu, r.u, r.v);
    r.A = first.A + second.A;
    r.o = second.o;
    out = r;
}

// h = o c / n, written the same way wherever the guess forms it.
SLSTM_DEVINL float guess_h(float o, float c, float n) { return o * (c * __fdividef(1.0f, n)); }

// Gates of one step with R = 0.
template <int FORGET>
SLSTM_DEVINL void guess_gates(float pz, float pf, float po, float &z, float &lf, float &o)
{
    z = tanh_fast(pz);
    o = sigmoid_fast(po);
    if (FORGET == SLSTM_FORGET_EXP) {
        lf = pf;
    } else {
        lf = fminf(pf, 0.0f) - __logf(1.0f + __expf(-fabsf(pf)));
    }
}

// Runs of the tile in shared memory: [entry][feature][warp], the warp index
// padded to 17 so that both the walk (lane = feature, one warp) and the scan
// (lane = warp, two features per warp) touch 32 distinct banks.
constexpr int SEG_LD = NW + 1;

struct GuessSmem {
    float P[2][TT][4][32];   // stage s: rows (step, slot) of 32 features; TMA boxes land here
    float Hs[2][TT][32];     // sweeps: h of the previous guess at every step of the tile
    float O[TT][4][32];      // TMA path: S of the tile, source of the warps' TMA stores
    float seg[5][32][SEG_LD];   // each warp's run (A, mu, u, v, o), then the inclusive prefixes
    float cin[4][32];        // state (c, n, m, h) entering the tile
    float hlast[NW][32];     // in-tile sweeps: the stage before's h at each warp's last step
    float hb[2][32];         // sweeps: h of the previous guess just before the tile
    TileInfo info[3];
    uint64_t bar[2];
    unsigned whead;
    int exit_flag;
};
constexpr size_t GUESS_SMEM_BYTES = sizeof(GuessSmem) + 1024;

// Loads of one tile: P, and for a sweep the previous guess's h rows (TMA
// box of slot 3) and the h just before the tile (the previous launch's
// boundary buffer).
template <bool SWEEP>
SLSTM_DEVINL void guess_issue_load(const Args &a, const NewtonMaps &m, GuessSmem &sm, int st, const TileInfo &ti)
{
    if (ti.ticket >= (unsigned)a.n_tiles) return;
    const bool bnd = SWEEP && ti.chunk > 0;
    mbar_expect_tx(&sm.bar[st], (uint32_t)sizeof(sm.P[0]) + (SWEEP ? (uint32_t)sizeof(sm.Hs[0]) : 0u) +
                                    (bnd ? 128u : 0u));
    tma_load_3d(&sm.P[st][0][0][0], &m.P, &sm.bar[st], ti.j0, ti.chunk * TT * 4, ti.b);
    if (SWEEP) {
        tma_load_4d(&sm.Hs[st][0][0], &m.H, &sm.bar[st], ti.j0, 3, ti.chunk * TT, ti.b);
        if (bnd && SLSTM_RANGE(a.bnd_in + (size_t)(ti.ticket - (unsigned)a.n_groups) * 4 * 32 + 3 * 32, a.bnd_in,
                               ext_tiles(a), 32))
            bulk_load(&sm.hb[st][0], a.bnd_in + (size_t)(ti.ticket - (unsigned)a.n_groups) * 4 * 32 + 3 * 32, 128u,
                      &sm.bar[st]);
    }
}

// cp.async path: 4-byte copies, lane = feature; rows past T and features
// past d arrive as zeros.
template <bool SWEEP>
SLSTM_DEVINL void guess_prefetch(const Args &a, GuessSmem &sm, int st, const TileInfo &ti)
{
    if (ti.ticket >= (unsigned)a.n_tiles) return;
    const int w = threadIdx.x >> 5, jl = threadIdx.x & 31;
    const bool fj = ti.j0 + jl < a.d;
    const float *p = a.P + ti.off + (size_t)w * a.d + jl;
    const size_t roww = (size_t)NW * a.d;
    const int t0 = ti.chunk * TT;
#pragma unroll 4
    for (int r = 0; r < 4 * L; ++r) {
        const int rs = r * NW + w;
        const int step = rs >> 2, slot = rs & 3;
        const int bytes = (fj && t0 + step < a.T && SLSTM_PIN(p + r * roww, a.P, ext_ps(a))) ? 4 : 0;
        cp_async4(&sm.P[st][step][slot][jl], bytes ? p + r * roww : a.P, bytes);
    }
    if (SWEEP) {
        // h rows: warp w copies steps w, w + NW, ...
        const float *hs = a.S + ti.off + 3 * (size_t)a.d + jl;
#pragma unroll
        for (int r = 0; r < L; ++r) {
            const int step = r * NW + w;
            const int bytes = (fj && t0 + step < a.T && SLSTM_PIN(hs + (size_t)step * 4 * a.d, a.S, ext_ps(a))) ? 4 : 0;
            cp_async4(&sm.Hs[st][step][jl], bytes ? hs + (size_t)step * 4 * a.d : a.S, bytes);
        }
        if (w == 0) {
            const float *src = a.bnd_in + (size_t)(ti.ticket - (unsigned)a.n_groups) * 4 * 32 + 3 * 32 + jl;
            const bool bnd = ti.chunk > 0 && SLSTM_PIN(src, a.bnd_in, ext_tiles(a));
            cp_async4(&sm.hb[st][jl], bnd ? src : a.bnd_in, bnd ? 4 : 0);
        }
    }
}

SLSTM_DEVINL void seg_load(const GuessSmem &sm, int w, int f, Seg &x, bool head)
{
    x.A = sm.seg[0][f][w];
    x.mu = sm.seg[1][f][w];
    x.u = sm.seg[2][f][w];
    x.v = sm.seg[3][f][w];
    x.o = sm.seg[4][f][w];
    x.head = head;
}

SLSTM_DEVINL void seg_store(GuessSmem &sm, int w, int f, const Seg &x)
{
    sm.seg[0][f][w] = x.A;
    sm.seg[1][f][w] = x.mu;
    sm.seg[2][f][w] = x.u;
    sm.seg[3][f][w] = x.v;
    sm.seg[4][f][w] = x.o;
}

// The state after the run x entered from v (c, n, m, h).
SLSTM_DEVINL void seg_enter(const Seg &x, const float v[4], float out[4])
{
    if (x.head) {
        out[0] = x.u;
        out[1] = x.v;
        out[2] = x.mu;
    } else {
        out[0] = v[0];
        out[1] = v[1];
        out[2] = v[2];
        seg_apply(x.A, x.mu, x.u, x.v, out[2], out[0], out[1]);
    }
    out[3] = guess_h(x.o, out[0], out[1]);
}

// One guess stage's look-back state: per tile a flag word, the tile's run
// (5 x 32 floats: A, mu, u, v, o) and its published state (4 x 32 words).
struct GuessChain {
    unsigned *flags;
    float *runs;
    unsigned long long *incw;
};

SLSTM_DEVINL GuessChain guess_chain(const Args &a, int stage)
{
    const size_t n = (size_t)a.n_tiles;
    return GuessChain{a.flags + stage * n, a.agg + stage * n * 160, a.incw + stage * n * 128};
}

// The guess's look-back when the predecessor's state is not published yet
// (warp 0, lane = feature, chunk > 0): publishes this tile's run, then
// composes the runs of unfinished predecessors until it meets a published
// state.  Returns the state (c, n, m, h) entering the tile in v.
SLSTM_DEVINL void guess_lookback(const Args &a, const GuessChain &gc, const Seg &tile, unsigned ticket, int chunk,
                                 int grp, float v[4])
{
    const int lane = threadIdx.x & 31;
    if (SLSTM_IN(ticket, a.n_tiles)) {
        float *dst = gc.runs + (size_t)ticket * 160 + lane;
        dst[0] = tile.A;
        dst[32] = tile.mu;
        dst[64] = tile.u;
        dst[96] = tile.v;
        dst[128] = tile.o;
        __threadfence();
        __syncwarp();
        if (lane == 0) st_release(gc.flags + ticket, (a.epoch << 2) | FLAG_AGG | (tile.head ? FLAG_HEAD : 0u));
    }
    Seg M;            // composition of the runs met so far (latest last)
    bool have = false;
    int q = chunk - 1;
    const uint64_t t0 = globaltimer_ns();
    unsigned polls = 0;
    const CarryArgs ca{gc.flags, nullptr, gc.incw, a.error, a.epoch, a.wait_ns, a.n_groups, a.n_tiles};
    for (;;) {
        const unsigned tq = (unsigned)q * (unsigned)a.n_groups + (unsigned)grp;
        float w[4];
        if (__all_sync(0xffffffffu, read_inc_words(ca, tq, lane, w))) {
            if (have) seg_enter(M, w, v);
            else {
#pragma unroll
                for (int e = 0; e < 4; ++e) v[e] = w[e];
            }
            return;
        }
        const unsigned f = SLSTM_IN(tq, a.n_tiles) ? ld_acquire(gc.flags + tq) : 0u;
        if ((f >> 2) == a.epoch && (f & FLAG_AGG)) {
            const float *src = gc.runs + (size_t)tq * 160 + lane;
            Seg x;
            x.A = __ldcg(src);
            x.mu = __ldcg(src + 32);
            x.u = __ldcg(src + 64);
            x.v = __ldcg(src + 96);
            x.o = __ldcg(src + 128);
            x.head = (f & FLAG_HEAD) != 0u;
            if (have) seg_compose(M, x, M);
            else M = x;
            have = true;
            if (M.head) {
                // a sequence starts inside: the state is the run's own end
                seg_enter(M, v, v);
                return;
            }
            --q;   // chunk 0 never publishes a run, so q stays >= 0
            continue;
        }
        if (++polls > 16) __nanosleep(64);
        if (globaltimer_ns() - t0 > a.wait_ns) {
            // gave up: the error word says so, and a NaN state makes every
            // output that depends on it NaN
            atomicOr(a.error, 1u);
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = __int_as_float(0x7fc00000);
            return;
        }
    }
}

// The decoupled guess and its refinement sweeps, NS stages per tile in one
// launch.  Stage 0 is the decoupled guess (SWEEP false) or a sweep of the
// guess that S holds (SWEEP true: the gates see r h_{t-1} of S, read before
// this launch overwrites it and, at a tile's first step, from the previous
// launch's boundary buffer); every later stage is a sweep of the stage before
// it, whose h never leaves the CTA.  Stage s of a tile takes its entering
// state from stage s of the tile before (its own flags, runs and published
// states), so the stages pipeline across tiles like one scan each.  One
// launch over every tile; launch k of the solve (epoch k + 1, control slot
// k & 1).  Per stage:
//   walk A  each thread folds its 4 steps into a run;
//   scan    the 16 warp runs of each feature are scanned (inclusive) by a
//           Kogge-Stone scan over 16 lanes, two features per warp, so that
//           the tile's run and every warp's prefix are known without a
//           serial walk;
//   carry   warp 0 takes the state entering the tile (the predecessor's
//           published state, or the look-back) and publishes the tile's;
//   walk B  each warp enters its steps through its prefix and replays them;
//           the last stage writes S and the tile's last state for the next
//           launch.
template <int FORGET, int NS, bool SWEEP, bool TMA, bool VARLEN>
__global__ void __launch_bounds__(NW * 32, 1) guess_kernel(Args a, int k, const __grid_constant__ NewtonMaps maps)
{
    extern __shared__ unsigned char smem_raw[];
    GuessSmem &sm = *reinterpret_cast<GuessSmem *>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    NewtonSlot &slot = a.ctrl->slot[k & 1];
    constexpr bool ANY_SWEEP = SWEEP || NS > 1;

    if (threadIdx.x == 0) {
        sm.exit_flag = (int)*(volatile unsigned *)&a.ctrl->done;
        if (!sm.exit_flag) {
            decode_tile(a, atomicAdd(&slot.ticket, 1u), sm.info[0]);
            decode_tile(a, atomicAdd(&slot.ticket, 1u), sm.info[1]);
        }
    }
    if (TMA && threadIdx.x == 0) {
        mbar_init(&sm.bar[0], 1);
        mbar_init(&sm.bar[1], 1);
        mbar_init_fence();
    }
    __syncthreads();
    if (sm.exit_flag) return;

    const size_t d = (size_t)a.d;
    const int T = a.T;
    const unsigned G = (unsigned)a.n_groups;
    int ring = 0, st = 0;
    unsigned it = 0;
    bool tma_ok = true;
    if (TMA) {
        if (threadIdx.x == 0) guess_issue_load<SWEEP>(a, maps, sm, 0, sm.info[0]);
    } else {
        guess_prefetch<SWEEP>(a, sm, 0, sm.info[0]);
        cp_async_commit();
    }

    for (;;) {
        const TileInfo ti = sm.info[ring];
        if (ti.ticket >= (unsigned)a.n_tiles) break;
        const int rn = ring == 2 ? 0 : ring + 1;
        unsigned after = 0;
        if (threadIdx.x == 0) after = atomicAdd(&slot.ticket, 1u);
        if (TMA) {
            if (threadIdx.x == 32) guess_issue_load<SWEEP>(a, maps, sm, st ^ 1, sm.info[rn]);
            if (tma_ok && !mbar_wait(&sm.bar[st], (it >> 1) & 1u, TMA_WAIT_NS)) {
                atomicOr(a.error, 2u);
                (void)mbar_wait(&sm.bar[st], (it >> 1) & 1u, TMA_WAIT_NS);
                tma_ok = false;
            }
        } else {
            guess_prefetch<SWEEP>(a, sm, st ^ 1, sm.info[rn]);
            cp_async_commit();
            cp_async_wait_prev();
            __syncthreads();
        }

        const unsigned ticket = ti.ticket;
        const int chunk = ti.chunk;
        const bool jv = ti.j0 + lane < a.d;
        const size_t jj = jv ? (size_t)(ti.j0 + lane) : 0;
        const int t_seg = chunk * TT + warp * L;

        float rz = 0.f, ri = 0.f, rf = 0.f, ro = 0.f;
        if (ANY_SWEEP && jv && SLSTM_IN(3 * d + jj, 4 * d)) {
            rz = __ldg(a.R + jj);
            ri = __ldg(a.R + d + jj);
            rf = __ldg(a.R + 2 * d + jj);
            ro = __ldg(a.R + 3 * d + jj);
        }
        if (threadIdx.x == 0) {
            unsigned wh = 0u;
            if (VARLEN) {
#pragma unroll
                for (int w = 0; w < NW; ++w)
                    wh |= (((ti.mask >> (w * L)) & ((1ull << L) - 1ull)) != 0ull) ? (1u << w) : 0u;
            }
            sm.whead = wh;
        }

        float hs[L];   // h of this thread's steps in the stage before (sweeps)
        float sv[4];   // the state after this thread's last step in the current stage
#pragma unroll
        for (int i = 0; i < L; ++i) hs[i] = 0.f;

#pragma unroll 1
        for (int stage = 0; stage < NS; ++stage) {
            const bool sweep = stage > 0 || SWEEP;
            const GuessChain gc = guess_chain(a, stage);
            // the gates' h before this warp's first step: the stage before's
            // state at step t_seg - 1
            float hp = 0.f;
            if (sweep) {
                if (stage == 0) {
                    if (warp > 0) hp = sm.Hs[st][warp * L - 1][lane];
                    else if (chunk > 0) hp = sm.hb[st][lane];
                    else if (!VARLEN && a.s0h && jv && SLSTM_IN(((size_t)ti.b * 4 + 3) * d + jj, a.n_s0))
                        hp = __ldg(a.s0h + ((size_t)ti.b * 4 + 3) * d + jj);
                } else {
                    hp = warp > 0 ? sm.hlast[warp - 1][lane] : sm.cin[3][lane];
                }
            }

            // the predecessor's published state of this stage, read now so
            // that the load's latency hides behind walk A and the scan: lane
            // 15 of each half-warp, for the feature it carries below
            const int fc = 2 * warp + (lane >> 4);
            const bool carry_lane = (lane & 15) == 15;
            unsigned long long pw[4] = {0ull, 0ull, 0ull, 0ull};
            if (carry_lane && chunk > 0 && SLSTM_IN(ticket - G, a.n_tiles)) {
                const unsigned long long *src = gc.incw + (size_t)(ticket - G) * 4 * 32 + fc;
#pragma unroll
                for (int e = 0; e < 4; ++e) pw[e] = ld_relaxed_u64(src + e * 32);
            }

            // ---- walk A: this warp's run, lane = feature ----
            float gz[L], glf[L], go[L], gi[L];
            {
                Seg run;
#pragma unroll
                for (int i = 0; i < L; ++i) {
                    const int sl = warp * L + i;
                    const bool head = VARLEN && ((ti.mask >> sl) & 1ull);
                    if (sweep && head) {
                        // a sequence starts here: its previous h is its own s0's
                        float s0v[4];
                        head_state(a, t_seg + i, jj, jv, s0v);
                        hp = s0v[3];
                    }
                    float pz = sm.P[st][sl][0][lane], pi = sm.P[st][sl][1][lane], pf = sm.P[st][sl][2][lane],
                          po = sm.P[st][sl][3][lane];
                    if (sweep) {
                        pz = fmaf(rz, hp, pz);
                        pi = fmaf(ri, hp, pi);
                        pf = fmaf(rf, hp, pf);
                        po = fmaf(ro, hp, po);
                        hp = stage == 0 ? sm.Hs[st][sl][lane] : hs[i];
                    }
                    guess_gates<FORGET>(pz, pf, po, gz[i], glf[i], go[i]);
                    gi[i] = pi;
                    if (head) {
                        float s0v[4];
                        head_state(a, t_seg + i, jj, jv, s0v);
                        run.mu = s0v[2];
                        run.u = s0v[0];
                        run.v = s0v[1];
                        seg_apply(glf[i], gi[i], gz[i], 1.0f, run.mu, run.u, run.v);
                        run.head = true;
                    } else if (i == 0) {
                        run.A = glf[i];
                        run.mu = gi[i];
                        run.u = gz[i];
                        run.v = 1.0f;
                        run.head = false;
                    } else {
                        seg_apply(glf[i], gi[i], gz[i], 1.0f, run.mu, run.u, run.v);
                        run.A += glf[i];
                    }
                    run.o = go[i];
                }
                seg_store(sm, warp, lane, run);
            }
            __syncthreads();

            // ---- scan of the warp runs: lane (feature 2 warp + lane / 16, run lane % 16) ----
            const unsigned whead = VARLEN ? sm.whead : 0u;   // dense sequences: no run holds a start
            bool ok = true;   // this lane's carry found the predecessor's state
            float vo[4];      // carry lanes: the state after the tile
            {
                const int f = fc, w = lane & 15;
                Seg x;
                seg_load(sm, w, f, x, ((whead >> w) & 1u) != 0u);
#pragma unroll
                for (int off = 1; off < NW; off *= 2) {
                    // the composition keeps the later run's output gate, so
                    // the earlier run's is not moved; dense sequences hold no
                    // start, so no head flag is either
                    Seg y;
                    y.A = __shfl_up_sync(0xffffffffu, x.A, off, 16);
                    y.mu = __shfl_up_sync(0xffffffffu, x.mu, off, 16);
                    y.u = __shfl_up_sync(0xffffffffu, x.u, off, 16);
                    y.v = __shfl_up_sync(0xffffffffu, x.v, off, 16);
                    y.o = 0.0f;
                    y.head = VARLEN && __shfl_up_sync(0xffffffffu, x.head ? 1 : 0, off, 16) != 0;
                    if (w >= off) seg_compose(x, y, x);
                }
                seg_store(sm, w, f, x);
                // ---- carry (fast path): the last run lane holds the tile's
                // run; entered from the predecessor's state read above ----
                if (carry_lane) {
                    float v[4] = {0.f, 0.f, 0.f, 0.f};
                    if (chunk == 0) {
                        if (!VARLEN && a.s0 && ti.j0 + f < a.d &&
                            SLSTM_IN(((size_t)ti.b * 4 + 3) * d + ti.j0 + f, a.n_s0)) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) v[e] = __ldg(a.s0 + ((size_t)ti.b * 4 + e) * d + ti.j0 + f);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            ok = ok && ((unsigned)(pw[e] >> 32) == a.epoch);
                            v[e] = __uint_as_float((unsigned)pw[e]);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) sm.cin[e][f] = v[e];
                    seg_enter(x, v, vo);
                }
            }
            static_assert(NW == 16, "the carry lanes are the last of 16 run lanes");
            if (__syncthreads_and(ok)) {
                // every feature found its predecessor's state: publish
                if (carry_lane && SLSTM_IN(ticket, a.n_tiles)) {
                    unsigned long long *dst = gc.incw + (size_t)ticket * 4 * 32 + fc;
#pragma unroll
                    for (int e = 0; e < 4; ++e) st_relaxed_u64(dst + e * 32, inc_word(a.epoch, vo[e]));
                }
            } else {
                // ---- carry (look-back): warp 0, lane = feature; nothing was
                // published above, and cin is written again for every feature ----
                if (warp == 0) {
                    float v[4] = {0.f, 0.f, 0.f, 0.f};
                    Seg tile;
                    seg_load(sm, NW - 1, lane, tile, whead != 0u);
                    if (chunk == 0) {
                        if (!VARLEN && a.s0 && jv && SLSTM_IN(((size_t)ti.b * 4 + 3) * d + jj, a.n_s0)) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) v[e] = __ldg(a.s0 + ((size_t)ti.b * 4 + e) * d + jj);
                        }
                    } else {
                        const CarryArgs ca{gc.flags, nullptr, gc.incw, a.error, a.epoch, a.wait_ns, a.n_groups, a.n_tiles};
                        const bool got = read_inc_words(ca, ticket - G, lane, v);
                        if (!__all_sync(0xffffffffu, got))
                            guess_lookback(a, gc, tile, ticket, chunk, (int)(ticket - (unsigned)chunk * G), v);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) sm.cin[e][lane] = v[e];
                    float vt[4];
                    seg_enter(tile, v, vt);
                    unsigned long long *dst = gc.incw + (size_t)ticket * 4 * 32 + lane;
                    if (SLSTM_IN(ticket, a.n_tiles)) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) st_relaxed_u64(dst + e * 32, inc_word(a.epoch, vt[e]));
                    }
                }
                __syncthreads();
            }

            // ---- walk B: enter this warp's steps through the prefix before it ----
            {
                float cv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) cv[e] = sm.cin[e][lane];
                if (warp == 0) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) sv[e] = cv[e];
                } else {
                    // whether the prefix of runs 0 .. warp - 1 holds a sequence start
                    const bool ph = (whead & ((1u << warp) - 1u)) != 0u;
                    Seg x;
                    seg_load(sm, warp - 1, lane, x, ph);
                    seg_enter(x, cv, sv);
                }
            }
            const bool last = stage == NS - 1;
            if (last && TMA) {
                if (lane == 0) bulk_wait_read_all();
                __syncwarp();
            }
            float *srow = a.S + ti.off + (size_t)warp * L * 4 * d + lane;
#pragma unroll
            for (int i = 0; i < L; ++i) {
                const int sl = warp * L + i;
                if (VARLEN && ((ti.mask >> sl) & 1ull)) head_state(a, t_seg + i, jj, jv, sv);
                seg_apply(glf[i], gi[i], gz[i], 1.0f, sv[2], sv[0], sv[1]);
                sv[3] = guess_h(go[i], sv[0], sv[1]);
                hs[i] = sv[3];
                if (last) {
                    const bool wr = jv && (t_seg + i < T);
                    if (TMA) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) sm.O[sl][e][lane] = sv[e];
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (wr && SLSTM_PIN(srow + (size_t)i * 4 * d + e * d, a.S, ext_ps(a)))
                                srow[(size_t)i * 4 * d + e * d] = sv[e];
                    }
                }
            }
            if (!last) {
                // the stage's h at this warp's last step, for the next warp's first gates
                sm.hlast[warp][lane] = sv[3];
                __syncthreads();
            }
        }
        if (TMA) {
            tma_store_fence();
            __syncwarp();
            if (lane == 0 && t_seg < T) {
                tma_store_3d(&maps.Sw, &sm.O[warp * L][0][0], ti.j0, t_seg * 4, ti.b);
                bulk_commit();
            }
        }
        // state at the tile's last step, read by the next launch
        if (warp == NW - 1 && t_seg + L - 1 < T) {
            float *dst = a.bnd_out + (size_t)ticket * 4 * 32;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (SLSTM_PIN(dst + e * 32 + lane, a.bnd_out, ext_tiles(a))) dst[e * 32 + lane] = sv[e];
        }
        if (threadIdx.x == 0) decode_tile(a, after, sm.info[rn == 2 ? 0 : rn + 1]);
        __syncthreads();   // this stage is free for the loads of the tile after next
        ring = rn;
        st ^= 1;
        ++it;
    }
    if (TMA) {
        if (lane == 0) bulk_wait_all();
    } else {
        cp_async_wait_all();
    }
    // the CTA that finishes the launch last clears the other control slot
    // for launch k + 1; the guess itself (k = 0) also marks the guess's
    // residual as not recorded (the first iteration records it)
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(&slot.finished, 1u) == gridDim.x - 1u) {
            NewtonSlot &nx = a.ctrl->slot[(k + 1) & 1];
            nx.ticket = 0u;
            nx.finished = 0u;
            nx.maxF_raw = 0u;
            nx.maxF_scaled = 0u;
            nx.failed = 0u;
            if (k == 0 && a.stats) {
                a.stats->init_max_abs_F = -1.0f;
                a.stats->init_max_scaled_F = -1.0f;
            }
            __threadfence();
        }
    }
}

// Caller-given guess: the state at the last step of every tile that has a
// successor, in the boundary layout the first Newton iteration reads
// ([tile][slot][32 features]).
__global__ void gather_boundaries(Args a)
{
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)a.n_tiles * 128) return;
    const unsigned tile = (unsigned)(idx >> 7);
    const int e = (int)((idx >> 5) & 3), lane = (int)(idx & 31);
    const unsigned chunk = tile / (unsigned)a.n_groups;
    const unsigned grp = tile - chunk * (unsigned)a.n_groups;
    const unsigned b = grp / (unsigned)a.groups_per_row;
    const int j = (int)(grp - b * (unsigned)a.groups_per_row) * 32 + lane;
    const long long t = (long long)chunk * TT + TT - 1;
    float v = 0.0f;
    const size_t src = (((size_t)b * a.T + (size_t)t) * 4 + e) * (size_t)a.d + j;
    if (t < a.T && j < a.d && SLSTM_IN(src, ext_ps(a))) v = a.S[src];
    if (SLSTM_IN(idx, ext_tiles(a))) a.bnd_out[idx] = v;
}

// TMA: tiles move by TMA (loads by TMA_THREAD into an mbarrier-guarded
// stage, stores per warp from the stage walk B wrote); otherwise by cp.async
// and plain stores.
// VARLEN: packed ragged sequences (B = 1); at a head step the previous state is
// the sequence's s0 and the Jacobian is zero, which makes the scan segmented.
// GRS: the first iteration from the decoupled guess also records the
// guess's residual (tolerance mode).
// One iteration (launch k of the solve) over every tile; newton_iter runs one
// per launch, newton_iter_loop several in one launch.  The TMA stages'
// mbarriers are initialised once per launch (bars_ready false: this body does
// it) and never again, since re-initialising a live mbarrier is not allowed;
// tiles_done, the tiles this CTA has taken in earlier bodies of the launch,
// carries their phases from one body to the next.
template <int FORGET, bool FIRST, bool RESID, bool TMA, bool VARLEN, int MODE, bool GRS>
SLSTM_DEVINL void newton_iter_body(const Args &a, int k, const NewtonMaps &maps, unsigned &tiles_done,
                                   bool &bars_ready)
{
    extern __shared__ unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    NewtonSlot &slot = a.ctrl->slot[k & 1];

    if (threadIdx.x == 0) {
        sm.exit_flag = (int)*(volatile unsigned *)&a.ctrl->done;
        if (!sm.exit_flag) {
            // AGG tiles are independent: a static order needs no counter
            decode_tile(a, MODE == MODE_AGG ? blockIdx.x : atomicAdd(&slot.ticket, 1u), sm.info[0]);
            decode_tile(a, MODE == MODE_AGG ? blockIdx.x + gridDim.x : atomicAdd(&slot.ticket, 1u), sm.info[1]);
        }
    }
    if (TMA && !bars_ready && threadIdx.x == TMA_THREAD) {
        mbar_init(&sm.bar[0], 1);
        mbar_init(&sm.bar[1], 1);
        mbar_init_fence();
    }
    bars_ready = true;
    __syncthreads();
    if (sm.exit_flag) return;

    const size_t d = (size_t)a.d;
    const int T = a.T;
    const unsigned G = (unsigned)a.n_groups;
    const size_t toff = prefetch_offset(a);
    const bool chain_warp = warp >= CHAIN0;
    float mx_raw = 0.f, mx_sc = 0.f;
    // the first iteration from the decoupled guess records the guess's
    // residual, which walk A forms anyway (r = f - S_old = -F)
    constexpr bool grs = GRS && MODE != MODE_AGG && !FIRST;
    float g_raw = 0.f, g_sc = 0.f;
    // Once a residual of this iteration fails the stopping test the solve
    // goes on whatever the others are: later tiles then only check that their
    // new states are finite (so that a non-finite iterate still stops the
    // solve at once).  The last allowed iteration, and every one with the
    // exact history, evaluates its whole residual; so do the cp.async path
    // (rows that are not 16-byte aligned) and packed sequences, whose
    // registers have no room for the second copy of walk B.
    const bool may_skip = TMA && !VARLEN && RESID && !a.exact_hist && (k + 1 - a.k0 < a.max_iters);

    unsigned it = tiles_done;   // tiles done by this CTA in the launch; stage it & 1, TMA phase (it >> 1) & 1
    const unsigned it0 = it;
    int ring = 0, st = (int)(it & 1u);
    bool tma_ok = true;    // false after a TMA wait expired: no further waits
    if (TMA) {
        if (threadIdx.x == TMA_THREAD) issue_tile_load(a, maps, sm, st, sm.info[0], !FIRST);
    } else {
        prefetch_tile(a, sm, st, sm.info[0], toff, !FIRST);
        cp_async_commit();
    }

    for (;;) {
        const TileInfo ti = sm.info[ring];
        if (ti.ticket >= (unsigned)a.n_tiles) break;
        const int rn = ring == 2 ? 0 : ring + 1;
        // tickets run two tiles ahead: fetch the one after the next now,
        // decode it into the ring at the end of this tile
        unsigned after = 0;
        if (threadIdx.x == 0) {
            after = MODE == MODE_AGG ? blockIdx.x + (it - it0 + 2u) * gridDim.x : atomicAdd(&slot.ticket, 1u);
            if (may_skip) sm.resid_skip = (int)*(volatile unsigned *)&slot.failed;
        }
        if (TMA) {
            // the other stage is free (every warp passed the barrier that
            // ends the previous tile): start the next tile's loads a whole
            // tile ahead, then wait for the current tile's boxes
            if (lane == 0 && warp >= TMA_WARP0 && warp < TMA_WARP0 + 4)
                issue_tile_load_part(a, maps, sm, st ^ 1, sm.info[rn], !FIRST, warp - TMA_WARP0);
            if (tma_ok && !mbar_wait(&sm.bar[st], (it >> 1) & 1u, TMA_WAIT_NS)) {
                atomicOr(a.error, 2u);
                (void)mbar_wait(&sm.bar[st], (it >> 1) & 1u, TMA_WAIT_NS);
                tma_ok = false;
            }
        } else {
            prefetch_tile(a, sm, st ^ 1, sm.info[rn], toff, !FIRST);
            cp_async_commit();
            cp_async_wait_prev();   // the current tile's copies have landed
            __syncthreads();
        }

        const unsigned ticket = ti.ticket;
        const int chunk = ti.chunk;
        const bool jv = ti.j0 + lane < a.d;
        const size_t jj = jv ? (size_t)(ti.j0 + lane) : 0;
        const int t_seg = chunk * TT + warp * L;

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
        // old state just before this warp's segment
        float sp[4] = {0.f, 0.f, 0.f, 0.f};
        if (t_seg == 0) {
            if (!VARLEN && a.s0 && jv && SLSTM_IN(((size_t)ti.b * 4 + 3) * d + jj, a.n_s0)) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sp[e] = __ldg(a.s0 + ((size_t)ti.b * 4 + e) * d + jj);
            }
        } else if (!FIRST) {
            if (warp == 0) {
                if (TMA) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) sp[e] = sm.bnd[st][e][lane];
                } else {
                    const float *src = a.bnd_in + (size_t)(ticket - G) * 4 * 32;
                    if (SLSTM_RANGE(src, a.bnd_in, ext_tiles(a), 128)) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) sp[e] = src[e * 32 + lane];
                    }
                }
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) sp[e] = sm.S[st][warp * L - 1][e][lane];
            }
        }

        // looks at the predecessor's inclusive prefix (chain lanes): before
        // and halfway through walk A, so that both loads' latency is hidden;
        // the second is read only when the first found nothing
        const bool look = MODE == MODE_FUSED && chain_warp && chunk > 0 && SLSTM_IN(ticket - G, a.n_tiles);
        const unsigned long long *predw = a.incw + chain_word(ticket - G, warp, lane);
        unsigned long long w1 = 0ull, w2 = 0ull;
        if (look) w1 = ld_relaxed_u64(predw);

        // ---- walk A ----
        // Jc[i] keeps J_t and f(S_{t-1}, P_t) of step i for walk B.  Steps past
        // T (only in a group's last tile) run on zero-filled rows; nothing
        // downstream of them is stored or published.
        Cell Jc[L];
        AffP agg;
        {
            float curS[4] = {sp[0], sp[1], sp[2], sp[3]};
#pragma unroll
            for (int i = 0; i < L; ++i) {
                if (i == L / 2 && look) w2 = ld_relaxed_u64(predw);
                const int sl = warp * L + i;
                float so[4] = {0.f, 0.f, 0.f, 0.f};
                if (!FIRST) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) so[e] = sm.S[st][sl][e][lane];
                }
                const bool head = VARLEN && ((ti.mask >> sl) & 1ull);
                if (head) head_state(a, t_seg + i, jj, jv, curS);
                cell_eval<FORGET, true>(curS[0], curS[1], curS[2], curS[3], sm.P[st][sl][0][lane],
                                        sm.P[st][sl][1][lane], sm.P[st][sl][2][lane], sm.P[st][sl][3][lane], rz, ri,
                                        rf, ro, Jc[i]);
                if (head) cell_zero_jac(Jc[i]);
                const float r[4] = {Jc[i].c - so[0], Jc[i].n - so[1], Jc[i].m - so[2], Jc[i].h - so[3]};
                if (grs) {
                    const bool valid = jv && (t_seg + i < T);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float af = valid ? fabsf(r[e]) : 0.0f;
                        g_raw = fmax_nan(g_raw, af);
                        g_sc = fmax_nan(g_sc, __fdividef(af, 1.0f + fabsf(so[e])));
                    }
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) curS[e] = so[e];
                // a head starts the warp's map afresh: select, never multiply
                // what came before by its zero Jacobian; in the aggregate
                // pass, steps past T (the last tile only) are left out, so
                // that the tile's map is the map of its steps (a time
                // slice's map composes it)
                const bool valid = MODE != MODE_AGG || t_seg + i < T;
                if (!valid) {
                    if (i == 0) affp_identity(agg);
                } else if (i == 0 || head) {
                    affp_from_cell<false>(agg, Jc[i], r);
                } else {
                    fold_p<false>(agg, Jc[i], r);
                }
            }
        }
        maps_store(sm.maps.m, warp, lane, agg);

        // warps whose steps contain a sequence start (packed sequences)
        unsigned whead = 0u;
        if (VARLEN) {
#pragma unroll
            for (int w = 0; w < NW; ++w) whead |= (((ti.mask >> (w * L)) & ((1ull << L) - 1ull)) != 0ull) ? (1u << w) : 0u;
        }
        if constexpr (MODE == MODE_AGG) {
            // the tile's aggregate map: a tree over the warp maps (at step h,
            // warp w composes slot (2w+2)h - 1 with slot (2w+1)h - 1 into the
            // former; a part that holds a sequence start ignores what enters
            // it and is kept as it is)
#pragma unroll
            for (int h = 1; h < NW; h *= 2) {
                __syncthreads();
                if (warp < NW / (2 * h)) {
                    const int hi = (2 * warp + 2) * h - 1, lo = (2 * warp + 1) * h - 1;
                    const bool hhead = VARLEN && (((whead >> ((2 * warp + 1) * h)) & ((1u << h) - 1u)) != 0u);
                    Aff x, y;
                    maps_load(sm.maps.m, hi, lane, x);
                    if (!hhead) {
                        maps_load(sm.maps.m, lo, lane, y);
                        aff_compose(x, y, x);
                        maps_store(sm.maps.m, hi, lane, x);
                    }
                }
            }
            __syncthreads();
            if (warp == 0) {
                Aff x;
                maps_load(sm.maps.m, NW - 1, lane, x);
                float *dst = a.agg + (size_t)ticket * 20 * 32 + lane;
                if (SLSTM_IN(ticket, a.n_tiles)) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) dst[e * 32] = x.a[e];
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[(16 + e) * 32] = x.b[e];
                    if (lane == 0) a.flags[ticket] = whead ? 1u : 0u;
                }
            }
        } else {

            // ---- carry ----
            float c = 0.f;   // chunk 0: the iterate before t = 0 is fixed, no correction enters
            bool ok = true;
            if (MODE == MODE_APPLY && chain_warp && SLSTM_IN(chain_word(ticket, warp, lane), ext_tiles(a)))
                c = a.cin_buf[chain_word(ticket, warp, lane)];
            if (look) {
                if ((unsigned)(w1 >> 32) == a.epoch) {
                    c = __uint_as_float((unsigned)w1);
                } else {
                    ok = (unsigned)(w2 >> 32) == a.epoch;
                    c = __uint_as_float((unsigned)w2);
                }
            }
            const bool withhold = (k == a.k0) && ((int)ticket == a.fault_ticket);
            const bool fast = __syncthreads_and(ok);
            if (chain_warp) {
                if (fast) {
                    c = carry_chain4<NW>(sm.maps.m, sm.maps.cin, c, warp, lane, whead, CHAIN0);
                    if (MODE == MODE_FUSED && !withhold && SLSTM_IN(chain_word(ticket, warp, lane), ext_tiles(a)))
                        st_relaxed_u64(a.incw + chain_word(ticket, warp, lane), inc_word(a.epoch, c));
                    named_bar_sync(CHAIN_BAR, 4 * 32);
                } else {
                    if (warp == CHAIN0) {
                        const CarryArgs ca{a.flags, a.agg, a.incw, a.error, a.epoch, a.wait_ns, a.n_groups, a.n_tiles};
                        tile_carry_fallback<NW>(ca, sm.maps.m, sm.maps.cin, ticket, chunk,
                                                (int)(ticket - (unsigned)chunk * G), withhold, whead);
                    }
                    named_bar_sync(CHAIN_BAR, 4 * 32);
    #pragma unroll 1
                    for (int w = 0; w < CHAIN0; ++w) named_bar_arrive(1 + w, 5 * 32);
                }
            } else {
                named_bar_sync(1 + warp, 5 * 32);   // the carry entering this warp is stored
            }

            // ---- walk B ----
            // this warp's store of the previous tile has read its rows of O
            if (TMA) {
                if (lane == 0) bulk_wait_read_all();
                __syncwarp();
            }
            float dl[4];
    #pragma unroll
            for (int e = 0; e < 4; ++e) dl[e] = sm.maps.cin[warp][e][sw(e, lane)];
            float snp[4];
    #pragma unroll
            for (int e = 0; e < 4; ++e) snp[e] = sp[e] + dl[e];
            // row pointer of this lane's first step; lanes past d and steps past T
            // write nothing
            float *srow = a.S + ti.off + (size_t)warp * L * 4 * d + lane;
            // the steps, with (FULL) or without the residual of the new iterate
            auto walk_b = [&](auto full_tag) {
                constexpr bool FULL = decltype(full_tag)::value;
    #pragma unroll
                for (int i = 0; i < L; ++i) {
                    const int sl = warp * L + i;
                    const bool wr = jv && (t_seg + i < T);
                    if (VARLEN && ((ti.mask >> sl) & 1ull)) {
                        // a sequence starts here: nothing from before enters it
    #pragma unroll
                        for (int e = 0; e < 4; ++e) dl[e] = 0.0f;
                    }
                    // S_new_t = f_t + J_t delta_{t-1};  delta_t = S_new_t - S_old_t
                    const float f4[4] = {Jc[i].c, Jc[i].n, Jc[i].m, Jc[i].h};
                    float sn[4];
                    jac_mul_add(Jc[i], dl, f4, sn);
    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float so = FIRST ? 0.f : sm.S[st][sl][e][lane];
                        dl[e] = sn[e] - so;
                    }
                    if (TMA) {
                        // rows past T and features past d fall outside the tensor and
                        // are not stored
    #pragma unroll
                        for (int e = 0; e < 4; ++e) sm.O[sl][e][lane] = sn[e];
                    } else {
    #pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (wr && SLSTM_PIN(srow + (size_t)i * 4 * d + e * d, a.S, ext_ps(a)))
                                srow[(size_t)i * 4 * d + e * d] = sn[e];
                    }
                    if (FULL) {
                        if (VARLEN && ((ti.mask >> sl) & 1ull)) head_state(a, t_seg + i, jj, jv, snp);
                        Cell f;
                        cell_eval<FORGET, false>(snp[0], snp[1], snp[2], snp[3], sm.P[st][sl][0][lane],
                                                 sm.P[st][sl][1][lane], sm.P[st][sl][2][lane], sm.P[st][sl][3][lane],
                                                 rz, ri, rf, ro, f);
                        const float F[4] = {sn[0] - f.c, sn[1] - f.n, sn[2] - f.m, sn[3] - f.h};
    #pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float af = wr ? fabsf(F[e]) : 0.0f;
                            const float sc = __fdividef(af, 1.0f + fabsf(sn[e]));
                            mx_raw = fmax_nan(mx_raw, af);
                            mx_sc = fmax_nan(mx_sc, sc);
                        }
                    } else if (RESID && i == L - 1) {
                        // only whether the new states are finite: a non-finite
                        // value travels down the lane to the thread's last
                        // step (dense sequences: nothing resets the lane)
                        const bool fin = (fabsf(sn[0]) <= FLT_MAX) && (fabsf(sn[1]) <= FLT_MAX) &&
                                         (fabsf(sn[2]) <= FLT_MAX) && (fabsf(sn[3]) <= FLT_MAX);
                        if (jv && !fin) {
                            mx_raw = __int_as_float(0x7fc00000);
                            mx_sc = mx_raw;
                        }
                    }
    #pragma unroll
                    for (int e = 0; e < 4; ++e) snp[e] = sn[e];
                }
            };
            if (RESID && (!may_skip || !sm.resid_skip)) walk_b(std::true_type{});
            else walk_b(std::false_type{});
            if (TMA) {
                tma_store_fence();
                __syncwarp();
                if (lane == 0 && t_seg < T) {
                    tma_store_3d(&maps.Sw, &sm.O[warp * L][0][0], ti.j0, t_seg * 4, ti.b);
                    bulk_commit();
                }
            }
            // state at the tile's last step, for the next launch's successor tile
            if (warp == NW - 1 && t_seg + L - 1 < T) {
                float *dst = a.bnd_out + (size_t)ticket * 4 * 32;
                // (a self-test of the checked build can shorten the extent by one)
    #pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (SLSTM_PIN(dst + e * 32 + lane, a.bnd_out, ext_tiles(a) - a.check_plant))
                        dst[e * 32 + lane] = snp[e];
            }
            // a failure of the test is announced to the tiles after it (until
            // this CTA has seen the announcement)
            if (may_skip && !sm.resid_skip &&
                __any_sync(0xffffffffu, (a.resid_raw ? mx_raw : mx_sc) > a.tol) && lane == 0)
                atomicExch(&slot.failed, 1u);

        }
        // the tile after the next one (read two tiles from now), decoded where
        // warp 0 would otherwise wait for the chain warps
        if (threadIdx.x == 0) decode_tile(a, after, sm.info[rn == 2 ? 0 : rn + 1]);

        __syncthreads();   // this stage is free for the loads of the tile after next
        ring = rn;
        st ^= 1;
        ++it;
    }
    if (TMA) {
        if (lane == 0) bulk_wait_all();
    } else {
        cp_async_wait_all();
    }
    tiles_done = it;
    if constexpr (MODE == MODE_AGG) return;   // the iteration itself is the APPLY launch

    if (RESID) {
        mx_raw = warp_max(mx_raw);
        mx_sc = warp_max(mx_sc);
        if (lane == 0) {
            sm.red[0][warp] = mx_raw;
            sm.red[1][warp] = mx_sc;
        }
    }
    if (grs) {
        g_raw = warp_max(g_raw);
        g_sc = warp_max(g_sc);
        if (lane == 0) {
            atomic_max_nonneg(&a.ctrl->init_raw, g_raw);
            atomic_max_nonneg(&a.ctrl->init_scaled, g_sc);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (RESID) {
            float r0 = sm.red[0][0], r1 = sm.red[1][0];
            for (int w = 1; w < NW; ++w) {
                r0 = (__float_as_uint(sm.red[0][w]) > __float_as_uint(r0)) ? sm.red[0][w] : r0;
                r1 = (__float_as_uint(sm.red[1][w]) > __float_as_uint(r1)) ? sm.red[1][w] : r1;
            }
            atomic_max_nonneg(&slot.maxF_raw, r0);
            atomic_max_nonneg(&slot.maxF_scaled, r1);
        }
        __threadfence();
        const unsigned fin = atomicAdd(&slot.finished, 1u);
        if (fin == gridDim.x - 1u) {
            __threadfence();
            finalize(a, k, RESID);
        }
    }
}

template <int FORGET, bool FIRST, bool RESID, bool TMA, bool VARLEN, int MODE, bool GRS>
__global__ void __launch_bounds__(NW * 32, 16 / NW) newton_iter(Args a, int k, const __grid_constant__ NewtonMaps maps)
{
    unsigned tiles = 0;
    bool bars = false;
    newton_iter_body<FORGET, FIRST, RESID, TMA, VARLEN, MODE, GRS>(a, k, maps, tiles, bars);
}

// Every CTA of the launch arrives at the counter, which then reaches `target`
// (arrivals accumulate over the launch's barriers); true once it has, false
// when the wait ran out (bit 4 of the error word, the stats record's error set
// to SLSTM_ERR_TIMEOUT and the solve marked done).  The launch must be
// cooperative, so that every CTA is resident.
SLSTM_DEVINL bool grid_barrier(const Args &a, unsigned target)
{
    bool ok = true;
    // this CTA's TMA stores of S (async proxy, waited for) ordered before the
    // arrival, and the TMA loads of the next iteration after the barrier
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();   // this CTA's writes of the iteration (and the finaliser's) before the arrival
        atomicAdd(&a.ctrl->gbar, 1u);
        const uint64_t t0 = globaltimer_ns();
        unsigned polls = 0;
        while (ld_acquire(&a.ctrl->gbar) < target) {
            if (++polls > 8) __nanosleep(128);
            if (globaltimer_ns() - t0 > a.wait_ns) {
                atomicOr(a.error, 4u);
                if (a.stats) atomicExch(&a.stats->error, (int)SLSTM_ERR_TIMEOUT);
                atomicExch(&a.ctrl->done, 1u);
                ok = false;
                break;
            }
        }
    }
    const bool all = !__syncthreads_or(!ok);
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return all;
}

// Launches k_begin .. k_end - 1 of a tolerance-mode solve with the fused
// carry, in one cooperative launch: each iteration is newton_iter_body, and a
// grid-wide barrier between two iterations stands in for the launch
// boundary (the iteration's finaliser has reset the next control slot and
// decided whether the solve is done).  The loop ends as soon as the
// stopping rule has, so a converged solve costs one short launch for the
// rest of its iteration cap.  debug_fault 3: CTA 0 leaves before the first
// barrier, whose wait then runs out in every other CTA.
template <int FORGET, bool TMA, bool VARLEN>
__global__ void __launch_bounds__(NW * 32, 16 / NW)
    newton_iter_loop(Args base, int k_begin, int k_end, const __grid_constant__ NewtonMaps maps)
{
    unsigned tiles = 0;   // this CTA's tiles so far: the TMA stages' phases
    bool bars = false;
    for (int k = k_begin; k < k_end; ++k) {
        if (k > k_begin) {
            if (base.loop_fault && blockIdx.x == 0) return;
            if (!grid_barrier(base, (unsigned)(k - k_begin) * gridDim.x)) return;
            if (*(volatile unsigned *)&base.ctrl->done) return;
        }
        newton_iter_body<FORGET, false, true, TMA, VARLEN, MODE_FUSED, false>(launch_args(base, k), k, maps, tiles,
                                                                              bars);
    }
}

template <int FORGET, bool FIRST, bool RESID, bool TMA, bool VARLEN, int MODE, bool GRS = false>
cudaError_t launch_one(const Args &a, const NewtonMaps &m, int k, int sms, cudaStream_t st)
{
    auto kern = newton_iter<FORGET, FIRST, RESID, TMA, VARLEN, MODE, GRS>;
    static int blocks_per_sm = 0;
    if (blocks_per_sm == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, kern, NW * 32, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (blocks_per_sm < 1) blocks_per_sm = 1;
    }
    const int grid = min(a.n_tiles, sms * blocks_per_sm);
    kern<<<grid, NW * 32, SMEM_BYTES, st>>>(a, k, m);
    return cudaGetLastError();
}

// Launches k_begin .. k_end - 1 as one cooperative newton_iter_loop launch
// (every CTA resident, which its grid barriers need).
template <int FORGET, bool TMA, bool VARLEN>
cudaError_t launch_loop(const Args &a, const NewtonMaps &m, int k_begin, int k_end, int sms, cudaStream_t st)
{
    auto kern = newton_iter_loop<FORGET, TMA, VARLEN>;
    static int blocks_per_sm = 0;
    if (blocks_per_sm == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        int b = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, NW * 32, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (b < 1) return cudaErrorInvalidConfiguration;
        blocks_per_sm = b;
    }
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3((unsigned)min(a.n_tiles, sms * blocks_per_sm), 1, 1);
    cfg.blockDim = dim3(NW * 32, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a, k_begin, k_end, m);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// Whether newton_iter_loop can run on `st`: the device takes cooperative
// launches and the stream is not being captured into a graph (a captured
// call keeps one launch per iteration).
bool device_loop_ok(cudaStream_t st)
{
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    if (cs != cudaStreamCaptureStatusNone) return false;
    static int coop = -1;
    if (coop < 0) {
        int dev = 0, v = 0;
        coop = (cudaGetDevice(&dev) == cudaSuccess &&
                cudaDeviceGetAttribute(&v, cudaDevAttrCooperativeLaunch, dev) == cudaSuccess && v != 0)
                   ? 1
                   : 0;
    }
    return coop == 1;
}

template <int FORGET, bool TMA, bool VARLEN, int MODE>
cudaError_t launch_pass(const Args &a, const NewtonMaps &m, int k, bool resid, int sms, cudaStream_t st)
{
    if (k == 0)
        return resid ? launch_one<FORGET, true, true, TMA, VARLEN, MODE>(a, m, k, sms, st)
                     : launch_one<FORGET, true, false, TMA, VARLEN, MODE>(a, m, k, sms, st);
    if (MODE != MODE_AGG && resid && a.guess_tested && k == a.k0)
        return launch_one<FORGET, false, true, TMA, VARLEN, MODE, true>(a, m, k, sms, st);
    return resid ? launch_one<FORGET, false, true, TMA, VARLEN, MODE>(a, m, k, sms, st)
                 : launch_one<FORGET, false, false, TMA, VARLEN, MODE>(a, m, k, sms, st);
}

template <int FORGET, int NS, bool SWEEP, bool TMA, bool VARLEN>
cudaError_t launch_guess_ns(const Args &a, const NewtonMaps &m, int k, int sms, cudaStream_t st)
{
    auto kern = guess_kernel<FORGET, NS, SWEEP, TMA, VARLEN>;
    static bool ready = false;
    if (!ready) {
        const cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GUESS_SMEM_BYTES);
        if (e != cudaSuccess) return e;
        ready = true;
    }
    kern<<<min(a.n_tiles, sms), NW * 32, GUESS_SMEM_BYTES, st>>>(a, k, m);
    return cudaGetLastError();
}

// One guess launch of a single stage (the decoupled guess, or a sweep of S).
template <int FORGET, bool SWEEP, bool TMA, bool VARLEN>
cudaError_t launch_guess(const Args &a, const NewtonMaps &m, int k, int sms, cudaStream_t st)
{
    return launch_guess_ns<FORGET, 1, SWEEP, TMA, VARLEN>(a, m, k, sms, st);
}


// Guess launches of a solve with `sweeps` refinement sweeps: launch 0 runs
// the decoupled guess and the first GUESS_STAGES - 1 sweeps tile by tile;
// any further sweep is a launch of its own (1, 2, ...).
// The caller's optional timing events (slstm_newton_config.events): the next
// one is recorded before each launch of work and after the last.
struct LaunchEvents {
    int n;
    void *const *ev;
    int next;
    cudaError_t record(cudaStream_t st)
    {
        const int i = next++;
        if (i >= n || ev[i] == nullptr) return cudaSuccess;
        return cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st);
    }
    // after the last launch: this and every remaining event mark the end
    cudaError_t finish(cudaStream_t st)
    {
        cudaError_t e = cudaSuccess;
        while (e == cudaSuccess && next < n) e = record(st);
        return e == cudaSuccess ? record(st) : e;
    }
};

inline int guess_launches(int sweeps) { return 1 + (sweeps > GUESS_STAGES - 1 ? sweeps - (GUESS_STAGES - 1) : 0); }

template <int FORGET, bool TMA, bool VARLEN>
cudaError_t launch_guess_all(const Args &base, const NewtonMaps &m, int sweeps, int sms, LaunchEvents &le,
                             cudaStream_t st)
{
    const int fused = 1 + (sweeps < GUESS_STAGES - 1 ? sweeps : GUESS_STAGES - 1);
    const Args a0 = launch_args(base, 0);
    cudaError_t e = le.record(st);
    if (e != cudaSuccess) return e;
    switch (fused) {
    case 1: e = launch_guess_ns<FORGET, 1, false, TMA, VARLEN>(a0, m, 0, sms, st); break;
    case 2: e = launch_guess_ns<FORGET, 2, false, TMA, VARLEN>(a0, m, 0, sms, st); break;
    case 3: e = launch_guess_ns<FORGET, 3, false, TMA, VARLEN>(a0, m, 0, sms, st); break;
    default: e = launch_guess_ns<FORGET, 4, false, TMA, VARLEN>(a0, m, 0, sms, st); break;
    }
    const int n = guess_launches(sweeps);
    for (int k = 1; k < n && e == cudaSuccess; ++k) {
        if ((e = le.record(st)) != cudaSuccess) return e;
        e = launch_guess<FORGET, true, TMA, VARLEN>(launch_args(base, k), m, k, sms, st);
    }
    return e;
}

// The launches of one solve: the initial guess (decoupled: the guess kernel
// and its sweeps; given: the boundary gather) as launches 0 .. k0 - 1, then
// Newton iterations k = k0 .. k0 + max_iters - 1.
template <int FORGET, bool TMA, bool VARLEN>
cudaError_t launch_iters(const Args &base, const NewtonMaps &m, int max_iters, bool fixed, bool two_pass, int sms,
                         int init, LaunchEvents &le, cudaStream_t st)
{
    if (init == SLSTM_INIT_DECOUPLED) {
        const cudaError_t e = launch_guess_all<FORGET, TMA, VARLEN>(base, m, base.guess_sweeps, sms, le, st);
        if (e != cudaSuccess) return e;
    } else if (init == SLSTM_INIT_GIVEN) {
        const long long n = (long long)base.n_tiles * 128;
        cudaError_t e = le.record(st);
        if (e != cudaSuccess) return e;
        gather_boundaries<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(base);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // in tolerance mode with the fused carry, the iterations from loop_from
    // on run inside one cooperative launch that stops with the solve
    const int k_end = base.k0 + max_iters;
    const int loop_at = (!fixed && !two_pass && base.loop_from > 0 && base.loop_from < max_iters && device_loop_ok(st))
                            ? base.k0 + base.loop_from
                            : k_end;
    for (int k = base.k0; k < loop_at; ++k) {
        const Args a = launch_args(base, k);
        const bool resid = !fixed || (k + 1 - base.k0 == max_iters);
        cudaError_t e = le.record(st);
        if (e != cudaSuccess) return e;
        if (two_pass) {
            if ((e = launch_pass<FORGET, TMA, VARLEN, MODE_AGG>(a, m, k, false, sms, st)) != cudaSuccess) return e;
            const int n_chunks = a.n_tiles / a.n_groups;
            const TileScanArgs sa{a.agg, a.flags, a.blk_agg, a.blk_head, a.blk_cin, a.cin_buf, &a.ctrl->done,
                              a.n_groups, n_chunks, scan_blocks(n_chunks)};
            if ((e = launch_tile_scan(sa, st)) != cudaSuccess) return e;
            e = launch_pass<FORGET, TMA, VARLEN, MODE_APPLY>(a, m, k, resid, sms, st);
        } else {
            e = launch_pass<FORGET, TMA, VARLEN, MODE_FUSED>(a, m, k, resid, sms, st);
        }
        if (e != cudaSuccess) return e;
    }
    if (loop_at < k_end) {
        cudaError_t e = le.record(st);
        if (e != cudaSuccess) return e;
        if ((e = launch_loop<FORGET, TMA, VARLEN>(base, m, loop_at, k_end, sms, st)) != cudaSuccess) return e;
    }
    return le.finish(st);
}

struct Layout {
    size_t ctrl, flags, incw, agg, bnd0, bnd1, cin, blk_agg, blk_head, blk_cin, total;
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
    l.flags = take(sizeof(unsigned) * (size_t)l.n_tiles * GUESS_STAGES);
    l.incw = take(sizeof(unsigned long long) * 4 * 32 * (size_t)l.n_tiles * GUESS_STAGES);
    l.agg = take(sizeof(float) * 20 * 32 * (size_t)l.n_tiles);
    l.bnd0 = take(sizeof(float) * 4 * 32 * (size_t)l.n_tiles);
    l.bnd1 = take(sizeof(float) * 4 * 32 * (size_t)l.n_tiles);
    l.cin = take(sizeof(float) * 4 * 32 * (size_t)l.n_tiles);
    const size_t nblk = (size_t)l.n_groups * scan_blocks(l.n_chunks);
    l.blk_agg = take(sizeof(float) * 20 * 32 * nblk);
    l.blk_head = take(sizeof(unsigned) * nblk);
    l.blk_cin = take(sizeof(float) * 4 * 32 * nblk);
    l.total = off;
    return l;
}

int sm_count()
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

template <int FORGET, bool TMA>
cudaError_t launch_iters_any(const Args &a, const NewtonMaps &m, int max_iters, bool fixed, bool two_pass, int sms,
                             bool varlen, int init, LaunchEvents &le, cudaStream_t st)
{
    return varlen ? launch_iters<FORGET, TMA, true>(a, m, max_iters, fixed, two_pass, sms, init, le, st)
                  : launch_iters<FORGET, TMA, false>(a, m, max_iters, fixed, two_pass, sms, init, le, st);
}

}  // namespace

size_t newton_workspace_bytes(int B, int T, int d) { return layout(B, T, d).total; }

namespace {

// Arguments, tensor maps and cleared control state of one call.
cudaError_t prepare(const float *P, const float *R, const float *s0, float *S, const slstm_newton_config &cfg,
                    slstm_newton_stats *stats, int B, int T, int d, void *ws, cudaStream_t st, const Varlen *vl,
                    Args &a, NewtonMaps &m, bool &tma, bool &two_pass)
{
    const Layout l = layout(B, T, d);
    char *base = static_cast<char *>(ws);
    a.P = P;
    a.R = R;
    a.s0 = s0;
    a.s0h = s0;
    a.S = S;
    a.ctrl = reinterpret_cast<NewtonCtrl *>(base + l.ctrl);
    a.flags = reinterpret_cast<unsigned *>(base + l.flags);
    a.agg = reinterpret_cast<float *>(base + l.agg);
    a.incw = reinterpret_cast<unsigned long long *>(base + l.incw);
    a.bnd_in = reinterpret_cast<float *>(base + l.bnd0);
    a.bnd_out = reinterpret_cast<float *>(base + l.bnd1);
    a.cin_buf = reinterpret_cast<float *>(base + l.cin);
    a.blk_agg = reinterpret_cast<float *>(base + l.blk_agg);
    a.blk_head = reinterpret_cast<unsigned *>(base + l.blk_head);
    a.blk_cin = reinterpret_cast<float *>(base + l.blk_cin);
    a.stats = stats;
    a.error = &a.ctrl->error;
    a.epoch = 1;
    a.wait_ns = (unsigned long long)(cfg.wait_limit_us > 0 ? cfg.wait_limit_us : 2000000) * 1000ull;
    a.B = B;
    a.T = T;
    a.d = d;
    a.groups_per_row = l.groups_per_row;
    a.n_groups = l.n_groups;
    a.div_groups = make_fastdiv((unsigned)l.n_groups);
    a.div_gpr = make_fastdiv((unsigned)l.groups_per_row);
    a.n_tiles = l.n_tiles;
    a.max_iters = cfg.max_iters;
    a.fixed = cfg.fixed_iters ? 1 : 0;
    a.tol = cfg.tol;
    a.guess_sweeps = cfg.guess_sweeps;
    a.k0 = cfg.init == SLSTM_INIT_ZERO ? 0 : (cfg.init == SLSTM_INIT_DECOUPLED ? guess_launches(cfg.guess_sweeps) : 1);
    a.resid_raw = cfg.residual_mode == SLSTM_RESIDUAL_RAW ? 1 : 0;
    a.exact_hist = cfg.history == SLSTM_HISTORY_EXACT ? 1 : 0;
    a.guess_tested = (cfg.init == SLSTM_INIT_DECOUPLED && !a.fixed) ? 1 : 0;
    a.vec16 = ((d & 3) == 0 && (reinterpret_cast<uintptr_t>(P) & 15) == 0 &&
               (reinterpret_cast<uintptr_t>(S) & 15) == 0) ? 1 : 0;
    // fault injection: the first tile of chunk 1 withholds its publications,
    // so the first tile of chunk 2 has nothing to wait for
    a.fault_ticket = (cfg.debug_fault == 1 && l.n_chunks >= 3) ? l.n_groups : -1;
    a.check_plant = cfg.debug_fault == 2 ? 1 : 0;
    a.loop_fault = cfg.debug_fault == 3 ? 1 : 0;
    a.loop_from = cfg.loop_from < 0 ? 0 : (cfg.loop_from == 0 ? SLSTM_DEFAULT_LOOP_FROM : cfg.loop_from);
    a.n_s0 = (long long)(vl ? vl->n_seq : B) * 4 * d;

    // control block, aggregate flags and the epoch tags of the inclusive
    // prefixes start cleared on every call
    cudaError_t e = cudaMemsetAsync(base + l.ctrl, 0, l.agg - l.ctrl, st);
    if (e == cudaSuccess && stats) e = cudaMemsetAsync(stats, 0, sizeof(slstm_newton_stats), st);
    if (e != cudaSuccess) return e;
    a.vmask = nullptr;
    a.vseq = nullptr;
    if (vl) {
        // malformed offsets mark the call done before any iteration runs
        if ((e = varlen_build(*vl, T, stats, &a.ctrl->done, st)) != cudaSuccess) return e;
        a.vmask = vl->mask;
        a.vseq = vl->seq;
    }
    const int sms = sm_count();
    // TMA moves the tiles when the rows are 16-byte aligned and every row
    // coordinate fits a signed 32-bit box coordinate
    memset(&m, 0, sizeof(m));
    const uint64_t rows = 4 * (uint64_t)T, bstride = rows * (uint64_t)d;
    tma = a.vec16 && (reinterpret_cast<uintptr_t>(R) & 15) == 0 && rows < (1ull << 31) &&
          make_map_f32_3d(&m.P, P, d, rows, B, d, bstride, 32, TT * 4) &&
          make_map_f32_3d(&m.S, S, d, rows, B, d, bstride, 32, TT * 4) &&
          make_map_f32_3d(&m.Sw, S, d, rows, B, d, bstride, 32, L * 4) &&
          make_map_f32_4d(&m.H, S, d, 4, T, B, d, 4 * (uint64_t)d, bstride, 32, TT);
    // With few feature groups and a long time axis, most tiles of a fused
    // launch would wait for their predecessor: take the two passes instead.
    // Fault injection acts on the fused launch's publications.
    two_pass = cfg.carry_mode == SLSTM_CARRY_TWO_PASS ||
               (cfg.carry_mode == SLSTM_CARRY_AUTO && cfg.debug_fault == 0 &&
                prefer_two_pass(l.n_groups, (long long)l.n_chunks * TT, sms));
    return cudaSuccess;
}

}  // namespace

cudaError_t newton_forward(const float *P, const float *R, const float *s0, float *S,
                           const slstm_newton_config &cfg, slstm_newton_stats *stats, int B, int T,
                           int d, void *ws, cudaStream_t st, const Varlen *vl)
{
    Args a;
    NewtonMaps m;
    bool tma = false, two_pass = false;
    cudaError_t e = prepare(P, R, s0, S, cfg, stats, B, T, d, ws, st, vl, a, m, tma, two_pass);
    if (e != cudaSuccess) return e;
    const int sms = sm_count();
    const bool v = vl != nullptr;
    const int init = cfg.init;
    LaunchEvents le{cfg.n_events, cfg.events, 0};
    if (cfg.forget == SLSTM_FORGET_EXP)
        return tma ? launch_iters_any<SLSTM_FORGET_EXP, true>(a, m, cfg.max_iters, a.fixed, two_pass, sms, v, init, le,
                                                              st)
                   : launch_iters_any<SLSTM_FORGET_EXP, false>(a, m, cfg.max_iters, a.fixed, two_pass, sms, v, init,
                                                               le, st);
    return tma ? launch_iters_any<SLSTM_FORGET_SIGMOID, true>(a, m, cfg.max_iters, a.fixed, two_pass, sms, v, init,
                                                              le, st)
               : launch_iters_any<SLSTM_FORGET_SIGMOID, false>(a, m, cfg.max_iters, a.fixed, two_pass, sms, v, init,
                                                               le, st);
}

cudaError_t newton_guess_prepare(const float *P, const float *s0, float *S, const slstm_newton_config &cfg,
                                 slstm_newton_stats *stats, int B, int T, int d, void *ws, cudaStream_t st,
                                 NewtonCtrl **ctrl)
{
    Args a;
    NewtonMaps m;
    bool tma = false, two_pass = false;
    cudaError_t e = prepare(P, nullptr, s0, S, cfg, stats, B, T, d, ws, st, nullptr, a, m, tma, two_pass);
    if (e != cudaSuccess) return e;
    *ctrl = a.ctrl;
    if (cfg.init != SLSTM_INIT_DECOUPLED) return cudaSuccess;
    const int sms = sm_count();
    const Args a0 = launch_args(a, 0);
    if (cfg.forget == SLSTM_FORGET_EXP)
        return tma ? launch_guess<SLSTM_FORGET_EXP, false, true, false>(a0, m, 0, sms, st)
                   : launch_guess<SLSTM_FORGET_EXP, false, false, false>(a0, m, 0, sms, st);
    return tma ? launch_guess<SLSTM_FORGET_SIGMOID, false, true, false>(a0, m, 0, sms, st)
               : launch_guess<SLSTM_FORGET_SIGMOID, false, false, false>(a0, m, 0, sms, st);
}


// ---------------------------------------------------------------------------
// Time context parallel ("sLSTM in this library", section "Tensor parallel":
// context parallel splits time).  Rank r of n holds the steps
// [t_r, t_r + T_r) of every sequence.  Every scan of the solve becomes: each
// rank composes its slice into one map (a run of the guess's monoid, or the
// affine map of a Newton iteration's linear solve), the maps are exchanged
// (all-gather, by the caller), and each rank enters its slice through the
// composition of the maps of the ranks before it.
// ---------------------------------------------------------------------------
namespace {

// The run of one tile of a guess (SWEEP: of a sweep, the gates seeing the
// previous guess's h), one CTA per tile, warp w folding steps 4w .. 4w + 3
// (steps past T are left out); warp 0 composes the 16 warp runs into
// agg[tile] rows 0..4 and flags[tile] bit 0 (the tile is empty: never).
template <int FORGET, bool SWEEP>
__global__ void __launch_bounds__(NW * 32) cp_tile_run_kernel(Args a)
{
    __shared__ float runs[NW][5][32];
    __shared__ int nonempty[NW];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned ticket = blockIdx.x;
    TileInfo ti;
    decode_tile(a, ticket, ti);
    const size_t d = (size_t)a.d;
    const bool jv = ti.j0 + lane < a.d;
    const size_t jj = jv ? (size_t)(ti.j0 + lane) : 0;
    const int t_seg = ti.chunk * TT + warp * L;
    float rz = 0.f, ri = 0.f, rf = 0.f, ro = 0.f, hp = 0.f;
    if (SWEEP && jv && SLSTM_IN(3 * d + jj, 4 * d)) {
        rz = __ldg(a.R + jj);
        ri = __ldg(a.R + d + jj);
        rf = __ldg(a.R + 2 * d + jj);
        ro = __ldg(a.R + 3 * d + jj);
        const int tp = t_seg - 1;
        if (tp >= 0 && tp < a.T && SLSTM_IN((((size_t)ti.b * a.T + tp) * 4 + 3) * d + jj, ext_ps(a)))
            hp = __ldg(a.S + (((size_t)ti.b * a.T + tp) * 4 + 3) * d + jj);
        else if (tp < 0 && a.s0h && SLSTM_IN(((size_t)ti.b * 4 + 3) * d + jj, a.n_s0))
            hp = __ldg(a.s0h + ((size_t)ti.b * 4 + 3) * d + jj);
    }
    Seg run;
    int n = 0;
#pragma unroll
    for (int i = 0; i < L; ++i) {
        const int t = t_seg + i;
        if (t >= a.T) break;
        const size_t row = ((size_t)ti.b * a.T + t) * 4;
        float p[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) p[g] = (jv && SLSTM_IN((row + g) * d + jj, ext_ps(a))) ? __ldg(a.P + (row + g) * d + jj) : 0.0f;
        if (SWEEP) {
            p[0] = fmaf(rz, hp, p[0]);
            p[1] = fmaf(ri, hp, p[1]);
            p[2] = fmaf(rf, hp, p[2]);
            p[3] = fmaf(ro, hp, p[3]);
            hp = (jv && SLSTM_IN((row + 3) * d + jj, ext_ps(a))) ? __ldg(a.S + (row + 3) * d + jj) : 0.0f;
        }
        float z, lf, o;
        guess_gates<FORGET>(p[0], p[2], p[3], z, lf, o);
        if (n == 0) {
            run.A = lf;
            run.mu = p[1];
            run.u = z;
            run.v = 1.0f;
        } else {
            seg_apply(lf, p[1], z, 1.0f, run.mu, run.u, run.v);
            run.A += lf;
        }
        run.o = o;
        ++n;
    }
    runs[warp][0][lane] = run.A;
    runs[warp][1][lane] = run.mu;
    runs[warp][2][lane] = run.u;
    runs[warp][3][lane] = run.v;
    runs[warp][4][lane] = run.o;
    if (lane == 0) nonempty[warp] = n > 0;
    __syncthreads();
    if (warp == 0) {
        Seg tile;
        tile.head = false;
        for (int w = 0; w < NW; ++w) {
            if (!nonempty[w]) break;
            Seg x;
            x.A = runs[w][0][lane];
            x.mu = runs[w][1][lane];
            x.u = runs[w][2][lane];
            x.v = runs[w][3][lane];
            x.o = runs[w][4][lane];
            x.head = false;
            if (w == 0) tile = x;
            else seg_compose(x, tile, tile);
        }
        float *dst = a.agg + (size_t)ticket * 20 * 32 + lane;
        if (SLSTM_IN(ticket, a.n_tiles)) {
            dst[0] = tile.A;
            dst[32] = tile.mu;
            dst[64] = tile.u;
            dst[96] = tile.v;
            dst[128] = tile.o;
        }
    }
}

// One warp per feature group: the tiles' runs composed in time order into
// the slice's run, out (B, 5, d) with entries (A, mu, u, v, o).
__global__ void __launch_bounds__(256) cp_slice_run_kernel(Args a, int n_chunks, float *out)
{
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (g >= a.n_groups) return;
    const int b = g / a.groups_per_row, j = (g - b * a.groups_per_row) * 32 + lane;
    Seg acc;
    for (int c = 0; c < n_chunks; ++c) {
        const float *src = a.agg + ((size_t)c * a.n_groups + g) * 20 * 32 + lane;
        Seg x;
        x.A = src[0];
        x.mu = src[32];
        x.u = src[64];
        x.v = src[96];
        x.o = src[128];
        x.head = false;
        if (c == 0) acc = x;
        else seg_compose(x, acc, acc);
    }
    if (j < a.d) {
        const float e5[5] = {acc.A, acc.mu, acc.u, acc.v, acc.o};
#pragma unroll
        for (int e = 0; e < 5; ++e) out[((size_t)b * 5 + e) * a.d + j] = e5[e];
    }
}

// Thread per (b, j): the state entering rank `rank`'s slice, s0 (or zero)
// carried through the runs (n, B, 5, d) of ranks 0 .. rank - 1.
__global__ void __launch_bounds__(256) cp_enter_runs_kernel(const float *runs, int rank, const float *s0, int B, int d,
                                                            float *out)
{
    const long long q = (long long)blockIdx.x * 256 + threadIdx.x;
    if (q >= (long long)B * d) return;
    const int b = (int)(q / d), j = (int)(q - (long long)b * d);
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = s0 ? s0[((size_t)b * 4 + e) * d + j] : 0.0f;
    for (int r = 0; r < rank; ++r) {
        const float *x = runs + (((size_t)r * B + b) * 5) * d + j;
        Seg s;
        s.A = x[0];
        s.mu = x[d];
        s.u = x[2 * d];
        s.v = x[3 * d];
        s.o = x[4 * d];
        s.head = false;
        seg_enter(s, v, v);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) out[((size_t)b * 4 + e) * d + j] = v[e];
}

// One warp per feature group: the block aggregates of the two-pass scan
// (scan_block_agg) composed in time order into the slice's affine map, out
// (B, 20, d): A row-major (16), then the offset (4).
__global__ void __launch_bounds__(256) cp_slice_map_kernel(const float *blk_agg, int n_groups, int n_blk, int gpr, int d,
                                                           float *out)
{
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (g >= n_groups) return;
    const int b = g / gpr, j = (g - b * gpr) * 32 + lane;
    Aff acc, x;
    load_agg(blk_agg + (size_t)g * n_blk * 640, lane, acc);
    for (int k = 1; k < n_blk; ++k) {
        load_agg(blk_agg + ((size_t)g * n_blk + k) * 640, lane, x);
        aff_compose(x, acc, acc);
    }
    if (j < d) {
#pragma unroll
        for (int e = 0; e < 16; ++e) out[((size_t)b * 20 + e) * d + j] = acc.a[e];
#pragma unroll
        for (int e = 0; e < 4; ++e) out[((size_t)b * 20 + 16 + e) * d + j] = acc.b[e];
    }
}

// Thread per (b, j): the Newton correction entering rank `rank`'s slice, 0
// carried through the maps (n, B, 20, d) of ranks 0 .. rank - 1.
__global__ void __launch_bounds__(256) cp_enter_maps_kernel(const float *maps, int rank, int B, int d, float *out)
{
    const long long q = (long long)blockIdx.x * 256 + threadIdx.x;
    if (q >= (long long)B * d) return;
    const int b = (int)(q / d), j = (int)(q - (long long)b * d);
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    for (int r = 0; r < rank; ++r) {
        const float *x = maps + (((size_t)r * B + b) * 20) * d + j;
        Aff m;
#pragma unroll
        for (int e = 0; e < 16; ++e) m.a[e] = x[(size_t)e * d];
#pragma unroll
        for (int e = 0; e < 4; ++e) m.b[e] = x[(size_t)(16 + e) * d];
        aff_apply(m, v, v);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) out[((size_t)b * 4 + e) * d + j] = v[e];
}

struct CpLayout {
    size_t newton, enter, total;
};

CpLayout cp_layout(int B, int T, int d)
{
    CpLayout c;
    c.newton = 0;
    c.enter = (newton_workspace_bytes(B, T, d) + 255) & ~(size_t)255;
    c.total = c.enter + (((size_t)B * 4 * d * 4 + 255) & ~(size_t)255);
    return c;
}

slstm_newton_config cp_config(int forget, const slstm_newton_config *cfg)
{
    slstm_newton_config c;
    memset(&c, 0, sizeof(c));
    if (cfg) c = *cfg;
    c.forget = forget;
    c.max_iters = 1;
    c.fixed_iters = 0;
    c.init = SLSTM_INIT_GIVEN;
    c.guess_sweeps = 0;
    c.carry_mode = SLSTM_CARRY_TWO_PASS;
    c.debug_fault = 0;
    c.n_events = 0;
    c.events = nullptr;
    return c;
}

template <int FORGET>
cudaError_t cp_run_launch(const Args &a, bool sweep, cudaStream_t st)
{
    if (sweep) cp_tile_run_kernel<FORGET, true><<<a.n_tiles, NW * 32, 0, st>>>(a);
    else cp_tile_run_kernel<FORGET, false><<<a.n_tiles, NW * 32, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t cp_workspace_bytes(int B, int T, int d) { return cp_layout(B, T, d).total; }

cudaError_t cp_guess_run(const float *P, const float *R, const float *s_before, const float *S, bool sweep, int forget,
                         float *run_out, int B, int T, int d, void *ws, cudaStream_t st)
{
    const slstm_newton_config cfg = cp_config(forget, nullptr);
    Args a;
    NewtonMaps m;
    bool tma = false, two_pass = false;
    cudaError_t e = prepare(P, R, nullptr, const_cast<float *>(S), cfg, nullptr, B, T, d, ws, st, nullptr, a, m,
                            tma, two_pass);
    if (e != cudaSuccess) return e;
    a.s0h = s_before;
    e = forget == SLSTM_FORGET_EXP ? cp_run_launch<SLSTM_FORGET_EXP>(a, sweep, st)
                                   : cp_run_launch<SLSTM_FORGET_SIGMOID>(a, sweep, st);
    if (e != cudaSuccess) return e;
    const int n_chunks = a.n_tiles / a.n_groups;
    cp_slice_run_kernel<<<(a.n_groups + 7) / 8, 256, 0, st>>>(a, n_chunks, run_out);
    return cudaGetLastError();
}

cudaError_t cp_guess_apply(const float *P, const float *R, const float *s0, const float *s_before,
                           const float *runs, int rank, float *S, bool sweep, int forget, int B, int T, int d,
                           void *ws, cudaStream_t st)
{
    const CpLayout cl = cp_layout(B, T, d);
    float *enter = reinterpret_cast<float *>(static_cast<char *>(ws) + cl.enter);
    const long long nbd = (long long)B * d;
    cp_enter_runs_kernel<<<(unsigned)((nbd + 255) / 256), 256, 0, st>>>(runs, rank, s0, B, d, enter);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    slstm_newton_config cfg = cp_config(forget, nullptr);
    cfg.init = SLSTM_INIT_DECOUPLED;
    Args a;
    NewtonMaps m;
    bool tma = false, two_pass = false;
    if ((e = prepare(P, R, enter, S, cfg, nullptr, B, T, d, ws, st, nullptr, a, m, tma, two_pass)) != cudaSuccess)
        return e;
    a.s0h = s_before;
    const int sms = sm_count();
    if (!sweep) {
        const Args a0 = launch_args(a, 0);
        if (forget == SLSTM_FORGET_EXP)
            return tma ? launch_guess<SLSTM_FORGET_EXP, false, true, false>(a0, m, 0, sms, st)
                       : launch_guess<SLSTM_FORGET_EXP, false, false, false>(a0, m, 0, sms, st);
        return tma ? launch_guess<SLSTM_FORGET_SIGMOID, false, true, false>(a0, m, 0, sms, st)
                   : launch_guess<SLSTM_FORGET_SIGMOID, false, false, false>(a0, m, 0, sms, st);
    }
    // a sweep reads the previous guess's h at every tile's first step from
    // the boundary buffer: gather it from S first (launch 0), then sweep as
    // launch 1
    const long long n = (long long)a.n_tiles * 128;
    gather_boundaries<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(launch_args(a, 0));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const Args a1 = launch_args(a, 1);
    if (forget == SLSTM_FORGET_EXP)
        return tma ? launch_guess<SLSTM_FORGET_EXP, true, true, false>(a1, m, 1, sms, st)
                   : launch_guess<SLSTM_FORGET_EXP, true, false, false>(a1, m, 1, sms, st);
    return tma ? launch_guess<SLSTM_FORGET_SIGMOID, true, true, false>(a1, m, 1, sms, st)
               : launch_guess<SLSTM_FORGET_SIGMOID, true, false, false>(a1, m, 1, sms, st);
}

cudaError_t cp_newton_map(const float *P, const float *R, const float *s_before, const float *S, int forget,
                          float *map_out, int B, int T, int d, void *ws, cudaStream_t st)
{
    const slstm_newton_config cfg = cp_config(forget, nullptr);
    Args a;
    NewtonMaps m;
    bool tma = false, two_pass = false;
    slstm_newton_stats *no_stats = nullptr;
    cudaError_t e = prepare(P, R, s_before, const_cast<float *>(S), cfg, no_stats, B, T, d, ws, st, nullptr, a, m,
                            tma, two_pass);
    if (e != cudaSuccess) return e;
    // the iterate's state at every tile's last step (launch 0), then the
    // aggregate pass of iteration 1 and the block aggregates
    const long long n = (long long)a.n_tiles * 128;
    gather_boundaries<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(launch_args(a, 0));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int sms = sm_count();
    const Args a1 = launch_args(a, 1);
    if (forget == SLSTM_FORGET_EXP)
        e = tma ? launch_one<SLSTM_FORGET_EXP, false, false, true, false, MODE_AGG>(a1, m, 1, sms, st)
                : launch_one<SLSTM_FORGET_EXP, false, false, false, false, MODE_AGG>(a1, m, 1, sms, st);
    else
        e = tma ? launch_one<SLSTM_FORGET_SIGMOID, false, false, true, false, MODE_AGG>(a1, m, 1, sms, st)
                : launch_one<SLSTM_FORGET_SIGMOID, false, false, false, false, MODE_AGG>(a1, m, 1, sms, st);
    if (e != cudaSuccess) return e;
    const int n_chunks = a.n_tiles / a.n_groups;
    TileScanArgs sa{a1.agg, a1.flags, a1.blk_agg, a1.blk_head, a1.blk_cin, a1.cin_buf, nullptr,
                    a.n_groups, n_chunks, scan_blocks(n_chunks)};
    const long long nw = (long long)sa.n_groups * sa.n_blk;
    scan_block_agg<<<(unsigned)((nw + 7) / 8), 256, 0, st>>>(sa);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    cp_slice_map_kernel<<<(a.n_groups + 7) / 8, 256, 0, st>>>(a.blk_agg, a.n_groups, sa.n_blk, a.groups_per_row, d,
                                                              map_out);
    return cudaGetLastError();
}

cudaError_t cp_newton_apply(const float *P, const float *R, const float *s_before, const float *maps, int rank,
                            float *S, const slstm_newton_config &user, slstm_newton_stats *stats, int B, int T, int d,
                            void *ws, cudaStream_t st)
{
    const CpLayout cl = cp_layout(B, T, d);
    float *enter = reinterpret_cast<float *>(static_cast<char *>(ws) + cl.enter);
    const long long nbd = (long long)B * d;
    cp_enter_maps_kernel<<<(unsigned)((nbd + 255) / 256), 256, 0, st>>>(maps, rank, B, d, enter);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const slstm_newton_config cfg = cp_config(user.forget, &user);
    Args a;
    NewtonMaps m;
    bool tma = false, two_pass = false;
    if ((e = prepare(P, R, s_before, S, cfg, stats, B, T, d, ws, st, nullptr, a, m, tma, two_pass)) != cudaSuccess)
        return e;
    // the tile aggregates, block aggregates and boundary states of
    // cp_newton_map are still in the workspace; the carries start from the
    // correction entering the slice
    const int n_chunks = a.n_tiles / a.n_groups;
    const Args a1 = launch_args(a, 1);
    TileScanArgs sa{a1.agg, a1.flags, a1.blk_agg, a1.blk_head, a1.blk_cin, a1.cin_buf, &a1.ctrl->done,
                    a.n_groups, n_chunks, scan_blocks(n_chunks)};
    sa.cin0 = enter;
    sa.gpr = a.groups_per_row;
    sa.d = d;
    scan_block_carry<<<(sa.n_groups + 7) / 8, 256, 0, st>>>(sa);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const long long nw = (long long)sa.n_groups * sa.n_blk;
    scan_tile_carry<<<(unsigned)((nw + 7) / 8), 256, 0, st>>>(sa);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int sms = sm_count();
    if (user.forget == SLSTM_FORGET_EXP)
        return tma ? launch_one<SLSTM_FORGET_EXP, false, true, true, false, MODE_APPLY>(a1, m, 1, sms, st)
                   : launch_one<SLSTM_FORGET_EXP, false, true, false, false, MODE_APPLY>(a1, m, 1, sms, st);
    return tma ? launch_one<SLSTM_FORGET_SIGMOID, false, true, true, false, MODE_APPLY>(a1, m, 1, sms, st)
               : launch_one<SLSTM_FORGET_SIGMOID, false, true, false, false, MODE_APPLY>(a1, m, 1, sms, st);
}

}  // namespace slstm
