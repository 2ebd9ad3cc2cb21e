// Carry hand-off between the tiles of a blocked scan of 4x4 affine maps
// (a block-bidiagonal solve) with a decoupled look-back.
//
// A tile is 32 features x (NW warps x L steps).  Each warp folds its own L
// steps into one affine map per feature (lane = feature) and stores it in
// shared memory.  The carry entering the tile is the inclusive prefix of the
// tile before it in the same feature group (ticket - n_groups); from it the
// carry entering every warp follows by applying the warp maps in order, and
// the last of these values is the tile's own inclusive prefix, which it
// publishes for its successor.
//
// Publication.  An inclusive prefix (4 values per feature) is published as
// 64-bit words (value bits | epoch << 32), so a reader validates and reads it
// with one load per word and the writer needs no fence.  The epoch tags are
// cleared at the start of every call and each launch of the call has its own
// epoch.  A tile whose predecessor has not published yet publishes its own
// aggregate (gated by a per-tile flag word) and looks back past unfinished
// tiles, composing their aggregates until it meets a published prefix.
//
// Progress.  Tiles take tickets from a global counter in the order CTAs ask
// for them, tile (chunk c, group g) has ticket c * n_groups + g, and a CTA
// only waits on lower tickets, each held by a running CTA as its current
// tile: every wait ends.  Waits are also bounded in time; on expiry the tile
// records an error and continues with a NaN carry, so that the outputs that
// depend on it are NaN rather than silently wrong.
//
// Two layouts of the per-warp maps are supported.  The plain one,
// s_agg[w][20][32] (entry-major), is walked by warp 0 alone.  TileMaps stores
// the maps column-major with XOR-swizzled rows so that four warps can walk
// them at once with one (feature, row) pair per lane (carry_chain4): the
// carry's serial dependence over the NW maps then costs one 4-term dot
// product per map and lane instead of a 4x4 matrix-vector product.
#pragma once

#include "checked.cuh"
#include "common.cuh"

namespace slstm {

struct CarryArgs {
    unsigned *flags;              // [n_tiles] aggregate-published flags
    float *agg;                   // [n_tiles][20][32] published aggregates
    unsigned long long *incw;     // [n_tiles][4][32] inclusive prefixes (value bits | epoch << 32)
    unsigned *error;              // set to nonzero when a wait expires
    unsigned epoch;               // nonzero, unique per launch since the tags were cleared
    unsigned long long wait_ns;   // bound of one wait
    int n_groups;                 // feature groups (tiles per chunk)
    int n_tiles;                  // tiles of the launch (extent of the per-tile words; checked build)
};

SLSTM_DEVINL unsigned long long ld_relaxed_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

SLSTM_DEVINL void st_relaxed_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

SLSTM_DEVINL unsigned long long inc_word(unsigned epoch, float v)
{
    return ((unsigned long long)epoch << 32) | __float_as_uint(v);
}

// This lane's part (feature `lane`, 4 slots) of tile tq's inclusive prefix,
// if published in this launch.
SLSTM_DEVINL bool read_inc_words(const CarryArgs &ca, unsigned tq, int lane, float v[4])
{
    if (!SLSTM_IN(tq, ca.n_tiles)) {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = 0.0f;
        return false;
    }
    const unsigned long long *src = ca.incw + (size_t)tq * 4 * 32 + lane;
    bool ok = true;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const unsigned long long w = ld_relaxed_u64(src + e * 32);
        ok = ok && ((unsigned)(w >> 32) == ca.epoch);
        v[e] = __uint_as_float((unsigned)w);
    }
    return ok;
}

// ---- plain layout -----------------------------------------------------------
SLSTM_DEVINL void load_aff_smem(float (*s_agg)[20][32], int w, int lane, Aff &x)
{
#pragma unroll
    for (int e = 0; e < 16; ++e) x.a[e] = s_agg[w][e][lane];
#pragma unroll
    for (int e = 0; e < 4; ++e) x.b[e] = s_agg[w][16 + e][lane];
}

SLSTM_DEVINL void store_aff_smem(float (*s_agg)[20][32], int w, int lane, const Aff &x)
{
#pragma unroll
    for (int e = 0; e < 16; ++e) s_agg[w][e][lane] = x.a[e];
#pragma unroll
    for (int e = 0; e < 4; ++e) s_agg[w][16 + e][lane] = x.b[e];
}

// ---- look-back (warp 0, lane = feature) -------------------------------------
// Segment heads.  Bit w of `whead` marks a warp map that starts a new segment
// (packed sequences): it ignores what enters it, so applying or composing it
// selects its own map instead of multiplying by its zero matrix (a zero
// matrix times a non-finite carry would not give zero).  A tile aggregate
// that contains a head is published with FLAG_HEAD, and a look-back that
// meets one stops there: its offset is that tile's inclusive prefix.
constexpr unsigned FLAG_HEAD = 2u;

// The predecessor has not published its prefix: publish this tile's
// aggregate (composed from the warp maps that load(w, x) returns, in
// processing order) unless `withhold`, then walk back over earlier tiles of
// the group.  Returns this lane's carry entering the tile in `carry`.
template <int NW, class LoadMap>
SLSTM_DEVINL void tile_lookback(const CarryArgs &ca, LoadMap load, unsigned ticket, int chunk, int grp,
                                bool withhold, float carry[4], unsigned whead = 0u)
{
    const int lane = threadIdx.x & 31;
    Aff tile;
    load(0, tile);
    for (int w = 1; w < NW; ++w) {
        Aff x;
        load(w, x);
        if ((whead >> w) & 1u) tile = x;
        else aff_compose(x, tile, tile);
    }
    if (!withhold && SLSTM_IN(ticket, ca.n_tiles)) {
        float *dst = ca.agg + (size_t)ticket * 20 * 32;
#pragma unroll
        for (int e = 0; e < 16; ++e) dst[e * 32 + lane] = tile.a[e];
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[(16 + e) * 32 + lane] = tile.b[e];
        __threadfence();
        __syncwarp();
        // with a head inside, successors need not look past this tile (the
        // warps before the head still take the carry found below)
        if (lane == 0) st_release(ca.flags + ticket, (ca.epoch << 2) | FLAG_AGG | (whead ? FLAG_HEAD : 0u));
    }
    Aff M;  // composition of the aggregates met so far (latest first)
    aff_identity(M);
    int q = chunk - 1;
    const uint64_t t0 = globaltimer_ns();
    unsigned polls = 0;
    for (;;) {
        const unsigned tq = (unsigned)q * (unsigned)ca.n_groups + (unsigned)grp;
        float v[4];
        const bool got = read_inc_words(ca, tq, lane, v);
        if (__all_sync(0xffffffffu, got)) {
            aff_apply(M, v, carry);
            return;
        }
        const unsigned f = SLSTM_IN(tq, ca.n_tiles) ? ld_acquire(ca.flags + tq) : 0u;
        if ((f >> 2) == ca.epoch && (f & FLAG_AGG)) {
            Aff x;
            const float *src = ca.agg + (size_t)tq * 20 * 32;
#pragma unroll
            for (int e = 0; e < 16; ++e) x.a[e] = __ldcg(src + e * 32 + lane);
#pragma unroll
            for (int e = 0; e < 4; ++e) x.b[e] = __ldcg(src + (16 + e) * 32 + lane);
            if (f & FLAG_HEAD) {
                // that tile's prefix is its offset
                aff_apply(M, x.b, carry);
                return;
            }
            aff_compose(M, x, M);
            --q;   // chunk 0 never publishes an aggregate, so q stays >= 0
            continue;
        }
        if (++polls > 16) __nanosleep(64);
        if (globaltimer_ns() - t0 > ca.wait_ns) {
            // gave up: the error word says so, and a NaN carry makes every
            // output that depends on the missing prefix NaN
            atomicOr(ca.error, 1u);
#pragma unroll
            for (int e = 0; e < 4; ++e) carry[e] = __int_as_float(0x7fc00000);
            return;
        }
    }
}

// Warp 0, lane = feature: v_{w+1} = A_w v_w + b_w through the tile from
// `carry`; put(w, v_w) stores the carry entering warp w; the final value, the
// tile's inclusive prefix, is published unless `withhold`.
template <int NW, class LoadMap, class PutCarry>
SLSTM_DEVINL void carry_serial(const CarryArgs &ca, LoadMap load, PutCarry put, unsigned ticket, bool withhold,
                               const float carry[4], unsigned whead = 0u)
{
    const int lane = threadIdx.x & 31;
    // the next warp's map is loaded while the current one is applied
    float v[4] = {carry[0], carry[1], carry[2], carry[3]};
    Aff x;
    load(0, x);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        // the next map is read before the store, which loads may not pass
        Aff xn;
        if (w + 1 < NW) load(w + 1, xn);
        put(w, v);
        if ((whead >> w) & 1u) {
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = x.b[e];
        } else {
            aff_apply(x, v, v);
        }
        if (w + 1 < NW) x = xn;
    }
    if (!withhold && SLSTM_IN(ticket, ca.n_tiles)) {
        unsigned long long *dst = ca.incw + (size_t)ticket * 4 * 32 + lane;
#pragma unroll
        for (int e = 0; e < 4; ++e) st_relaxed_u64(dst + e * 32, inc_word(ca.epoch, v[e]));
    }
}

// Warp 0 only, plain layout.  Writes the carry entering every warp to
// s_cin[w] and publishes the tile's inclusive prefix.  `first` enters chunk
// 0; `withhold` suppresses this tile's publications (fault injection).
// `pre_ok` / `pre`: the predecessor's prefix as read earlier by the caller
// (to overlap the load's latency with other work); it is read again here
// when that read was early.
template <int NW>
SLSTM_DEVINL void tile_carry_serial(const CarryArgs &ca, float (*s_agg)[20][32], float (*s_cin)[4][32],
                                    unsigned ticket, int chunk, int grp, const float first[4], bool withhold,
                                    bool pre_ok = false, const float *pre = nullptr)
{
    const int lane = threadIdx.x & 31;
    auto load = [&](int w, Aff &x) { load_aff_smem(s_agg, w, lane, x); };
    float carry[4] = {first[0], first[1], first[2], first[3]};
    if (chunk > 0) {
        bool ok = pre_ok && (pre != nullptr);
        if (ok) {
#pragma unroll
            for (int e = 0; e < 4; ++e) carry[e] = pre[e];
        }
        if (!__all_sync(0xffffffffu, ok)) ok = read_inc_words(ca, ticket - (unsigned)ca.n_groups, lane, carry);
        if (!__all_sync(0xffffffffu, ok)) tile_lookback<NW>(ca, load, ticket, chunk, grp, withhold, carry);
    }
    carry_serial<NW>(
        ca, load,
        [&](int w, const float v[4]) {
#pragma unroll
            for (int e = 0; e < 4; ++e) s_cin[w][e][lane] = v[e];
        },
        ticket, withhold, carry);
}

// ---- packed fold ---------------------------------------------------------
// A fold's running aggregate with its matrix columns paired, so that the
// 4x4 products run on the packed fp32x2 pipe (__ffma2_rn / __fmul2_rn, two
// lanes of the same scalar operation per instruction).  Each packed lane
// performs exactly the scalar jac_mul / jacT_mul sequence.
struct AffP {
    float2 a01[4];   // row r: (A[r][0], A[r][1])
    float2 a23[4];   // row r: (A[r][2], A[r][3])
    float b[4];
};

SLSTM_DEVINL float2 dup2(float v) { return make_float2(v, v); }

// Columns x_k <- J x_k for a pair of columns (rows in x[0..3]).
SLSTM_DEVINL void jac_mul_p(const float2 j[11], float2 x[4])
{
    // j: fp, jcm, jch, jnm, jnh, beta, dmh, jhc, jhn, jhm, jhh
    const float2 y0 = __ffma2_rn(j[0], x[0], __ffma2_rn(j[1], x[2], __fmul2_rn(j[2], x[3])));
    const float2 y1 = __ffma2_rn(j[0], x[1], __ffma2_rn(j[3], x[2], __fmul2_rn(j[4], x[3])));
    const float2 y2 = __ffma2_rn(j[5], x[2], __fmul2_rn(j[6], x[3]));
    const float2 y3 = __ffma2_rn(j[7], x[0], __ffma2_rn(j[8], x[1], __ffma2_rn(j[9], x[2], __fmul2_rn(j[10], x[3]))));
    x[0] = y0;
    x[1] = y1;
    x[2] = y2;
    x[3] = y3;
}

// Columns x_k <- J^T x_k for a pair of columns.
SLSTM_DEVINL void jacT_mul_p(const float2 j[11], float2 x[4])
{
    const float2 y0 = __ffma2_rn(j[0], x[0], __fmul2_rn(j[7], x[3]));
    const float2 y1 = __ffma2_rn(j[0], x[1], __fmul2_rn(j[8], x[3]));
    const float2 y2 = __ffma2_rn(j[1], x[0], __ffma2_rn(j[3], x[1], __ffma2_rn(j[5], x[2], __fmul2_rn(j[9], x[3]))));
    const float2 y3 = __ffma2_rn(j[2], x[0], __ffma2_rn(j[4], x[1], __ffma2_rn(j[6], x[2], __fmul2_rn(j[10], x[3]))));
    x[0] = y0;
    x[1] = y1;
    x[2] = y2;
    x[3] = y3;
}

SLSTM_DEVINL void cell_pairs(const Cell &J, float2 j[11])
{
    j[0] = dup2(J.fp);
    j[1] = dup2(J.jcm);
    j[2] = dup2(J.jch);
    j[3] = dup2(J.jnm);
    j[4] = dup2(J.jnh);
    j[5] = dup2(J.beta);
    j[6] = dup2(J.dmh);
    j[7] = dup2(J.jhc);
    j[8] = dup2(J.jhn);
    j[9] = dup2(J.jhm);
    j[10] = dup2(J.jhh);
}

// agg <- (J, r) o agg (TRANS: J^T).
template <bool TRANS>
SLSTM_DEVINL void fold_p(AffP &agg, const Cell &J, const float r[4])
{
    float2 j[11];
    cell_pairs(J, j);
    float2 x[4] = {agg.a01[0], agg.a01[1], agg.a01[2], agg.a01[3]};
    if (TRANS) jacT_mul_p(j, x); else jac_mul_p(j, x);
#pragma unroll
    for (int i = 0; i < 4; ++i) agg.a01[i] = x[i];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = agg.a23[i];
    if (TRANS) jacT_mul_p(j, x); else jac_mul_p(j, x);
#pragma unroll
    for (int i = 0; i < 4; ++i) agg.a23[i] = x[i];
    if (TRANS) {
        jacT_mul(J, agg.b[0], agg.b[1], agg.b[2], agg.b[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) agg.b[e] += r[e];
    } else {
        const float b[4] = {agg.b[0], agg.b[1], agg.b[2], agg.b[3]};
        jac_mul_add(J, b, r, agg.b);
    }
}

SLSTM_DEVINL void affp_identity(AffP &x)
{
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        x.a01[r] = make_float2(r == 0 ? 1.f : 0.f, r == 1 ? 1.f : 0.f);
        x.a23[r] = make_float2(r == 2 ? 1.f : 0.f, r == 3 ? 1.f : 0.f);
        x.b[r] = 0.f;
    }
}

// The aggregate of a single step: (J, r) (TRANS: (J^T, r)).
template <bool TRANS>
SLSTM_DEVINL void affp_from_cell(AffP &x, const Cell &J, const float r[4])
{
    if (TRANS) {
        x.a01[0] = make_float2(J.fp, 0.f);   x.a23[0] = make_float2(0.f, J.jhc);
        x.a01[1] = make_float2(0.f, J.fp);   x.a23[1] = make_float2(0.f, J.jhn);
        x.a01[2] = make_float2(J.jcm, J.jnm); x.a23[2] = make_float2(J.beta, J.jhm);
        x.a01[3] = make_float2(J.jch, J.jnh); x.a23[3] = make_float2(J.dmh, J.jhh);
    } else {
        x.a01[0] = make_float2(J.fp, 0.f);   x.a23[0] = make_float2(J.jcm, J.jch);
        x.a01[1] = make_float2(0.f, J.fp);   x.a23[1] = make_float2(J.jnm, J.jnh);
        x.a01[2] = make_float2(0.f, 0.f);    x.a23[2] = make_float2(J.beta, J.dmh);
        x.a01[3] = make_float2(J.jhc, J.jhn); x.a23[3] = make_float2(J.jhm, J.jhh);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) x.b[e] = r[e];
}

// ---- chain layout -------------------------------------------------------------
// Row length of TileMaps.  Feature f of row r sits at position f ^ (8 r)
// (sw(r, f)): a row written by 32 feature lanes is a permutation of 32 banks,
// and the 32 (row, feature) pairs a chain warp reads (8 features x 4 rows)
// also fall in 32 distinct banks.
constexpr int MAP_LD = 32;
SLSTM_DEVINL int sw(int r, int f) { return f ^ (r << 3); }

// Per-warp maps of a tile, [warp][column k, k = 4: offset b][row][feature],
// and the carries entering the warps, [warp][slot][feature].
typedef float MapArr[5][4][MAP_LD];
typedef float CinArr[4][MAP_LD];

template <int NW>
struct TileMaps {
    MapArr m[NW];
    CinArr cin[NW];
};

// Lane = feature.
SLSTM_DEVINL void maps_store(MapArr *m, int w, int lane, const Aff &x)
{
#pragma unroll
    for (int r = 0; r < 4; ++r) {
#pragma unroll
        for (int k = 0; k < 4; ++k) m[w][k][r][sw(r, lane)] = x.a[r * 4 + k];
        m[w][4][r][sw(r, lane)] = x.b[r];
    }
}

SLSTM_DEVINL void maps_store(MapArr *m, int w, int lane, const AffP &x)
{
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        m[w][0][r][sw(r, lane)] = x.a01[r].x;
        m[w][1][r][sw(r, lane)] = x.a01[r].y;
        m[w][2][r][sw(r, lane)] = x.a23[r].x;
        m[w][3][r][sw(r, lane)] = x.a23[r].y;
        m[w][4][r][sw(r, lane)] = x.b[r];
    }
}

SLSTM_DEVINL void maps_load(const MapArr *m, int w, int lane, Aff &x)
{
#pragma unroll
    for (int r = 0; r < 4; ++r) {
#pragma unroll
        for (int k = 0; k < 4; ++k) x.a[r * 4 + k] = m[w][k][r][sw(r, lane)];
        x.b[r] = m[w][4][r][sw(r, lane)];
    }
}

// Chain lanes: four warps with warp & 3 = 0 .. 3, lane (row = lane >> 3,
// feature = 8 * (warp & 3) + (lane & 7)).
SLSTM_DEVINL int chain_feature(int warp, int lane) { return ((warp & 3) << 3) | (lane & 7); }
SLSTM_DEVINL int chain_row(int lane) { return lane >> 3; }

// Word of tile tq's inclusive prefix that chain lane (warp, lane) owns.
SLSTM_DEVINL size_t chain_word(unsigned tq, int warp, int lane)
{
    return ((size_t)tq * 4 + chain_row(lane)) * 32 + chain_feature(warp, lane);
}

// Chain warps only.  c: this lane's component of the carry entering the
// tile.  Stores the carry entering every warp in cin and returns this
// lane's component of the tile's inclusive prefix.  The arithmetic (order of
// the fused multiply-adds) is that of aff_apply, so both walks give the same
// bits.
//
// release > 0: each chain warp arrives at named barrier 1 + w (160 threads:
// the 4 chain warps and warp w) once the carry entering warp w < release is
// stored, so that warp can go on while the chain walks the later maps.
template <int NW>
SLSTM_DEVINL float carry_chain4(const MapArr *m, CinArr *cin, float c, int warp, int lane, unsigned whead = 0u,
                                int release = 0)
{
    const int f = chain_feature(warp, lane);
    const int r = chain_row(lane);
    const int fs = sw(r, f);
    const int i8 = lane & 7;
    // the map entries are read two maps ahead, before the stores and barrier
    // arrivals of the current map, which the compiler may not move loads past
    float q[3][5];
    auto load = [&](int w, float *o) {
#pragma unroll
        for (int k = 0; k < 5; ++k) o[k] = m[w][k][r][fs];
    };
    load(0, q[0]);
    if (NW > 1) load(1, q[1]);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        if (w + 2 < NW) load(w + 2, q[(w + 2) % 3]);
        cin[w][r][fs] = c;
        if (w < release) named_bar_arrive(1 + w, 5 * 32);
        const float *a = q[w % 3];
        const float v0 = __shfl_sync(0xffffffffu, c, i8);
        const float v1 = __shfl_sync(0xffffffffu, c, 8 + i8);
        const float v2 = __shfl_sync(0xffffffffu, c, 16 + i8);
        const float v3 = __shfl_sync(0xffffffffu, c, 24 + i8);
        // two FMA chains of depth two joined by an add: one level less on
        // the chain's critical path than a single chain of four
        const float nc = fmaf(a[1], v1, fmaf(a[0], v0, a[4])) + fmaf(a[3], v3, a[2] * v2);
        c = ((whead >> w) & 1u) ? a[4] : nc;
    }
    return c;
}

// One warp only, chain layout, when some chain lane found no published
// predecessor prefix: reads it again, else looks back; then walks the maps
// serially (lane = feature).  chunk > 0.
template <int NW>
SLSTM_DEVINL void tile_carry_fallback(const CarryArgs &ca, const MapArr *m, CinArr *cin, unsigned ticket, int chunk,
                                      int grp, bool withhold, unsigned whead = 0u)
{
    const int lane = threadIdx.x & 31;
    auto load = [&](int w, Aff &x) { maps_load(m, w, lane, x); };
    float carry[4];
    const bool ok = read_inc_words(ca, ticket - (unsigned)ca.n_groups, lane, carry);
    if (!__all_sync(0xffffffffu, ok)) tile_lookback<NW>(ca, load, ticket, chunk, grp, withhold, carry, whead);
    carry_serial<NW>(
        ca, load,
        [&](int w, const float v[4]) {
#pragma unroll
            for (int e = 0; e < 4; ++e) cin[w][e][sw(e, lane)] = v[e];
        },
        ticket, withhold, carry, whead);
}

namespace {

// ---- two-pass carry ----------------------------------------------------------
// Between the two passes of a blocked scan: the carry entering every tile,
// from the aggregates of the tiles before it in its feature group (chunk 0
// gets none).  Tile aggregates are [tile][20][32] (entry-major, lane =
// feature; A row-major, then b), carries [tile][4][32].  A group's chunks are cut into blocks of SCAN_BLK: the
// aggregates of every block are composed (scan_block_agg), the blocks of a
// group are walked in order (scan_block_carry), and every block applies its
// aggregates from the carry entering it (scan_tile_carry).  One warp per
// (group, block), lane = feature; a tile with a sequence start passes on its
// offset whatever enters it.
constexpr int SCAN_BLK = 32;

SLSTM_DEVINL void load_agg(const float *src, int lane, Aff &x)
{
#pragma unroll
    for (int e = 0; e < 16; ++e) x.a[e] = __ldcg(src + e * 32 + lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) x.b[e] = __ldcg(src + (16 + e) * 32 + lane);
}

SLSTM_DEVINL void store_agg(float *dst, int lane, const Aff &x)
{
#pragma unroll
    for (int e = 0; e < 16; ++e) dst[e * 32 + lane] = x.a[e];
#pragma unroll
    for (int e = 0; e < 4; ++e) dst[(16 + e) * 32 + lane] = x.b[e];
}

struct TileScanArgs {
    const float *agg;          // [n_tiles][20][32] tile aggregates
    const unsigned *head;      // [n_tiles] nonzero: the tile holds a sequence start
    float *blk_agg;            // [n_groups][n_blk][20][32]
    unsigned *blk_head;        // [n_groups][n_blk]
    float *blk_cin;            // [n_groups][n_blk][4][32]
    float *cin;                // [n_tiles][4][32] the carry entering each tile
    const unsigned *done;      // nonzero: the call has finished (or null)
    int n_groups, n_chunks, n_blk;
    // the carry entering each group's first tile, (B, 4, d) with group g =
    // (b, features 32 (g % gpr) ..), or null for zero (time slices after the
    // first of a context-parallel solve)
    const float *cin0 = nullptr;
    int gpr = 1, d = 0;
};

// (group, block) per warp: the composition of the block's tile aggregates.
__global__ void __launch_bounds__(256) scan_block_agg(TileScanArgs s)
{
    if (s.done && *(volatile const unsigned *)s.done) return;
    const int lane = threadIdx.x & 31;
    const long long wid = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (wid >= (long long)s.n_groups * s.n_blk) return;
    const int g = (int)(wid / s.n_blk), k = (int)(wid % s.n_blk);
    const int c0 = k * SCAN_BLK, c1 = min(c0 + SCAN_BLK, s.n_chunks);
    const size_t G = (size_t)s.n_groups;
    Aff acc, x;
    load_agg(s.agg + ((size_t)c0 * G + g) * 640, lane, acc);
    bool hd = s.head[(size_t)c0 * G + g] != 0u;
    for (int c = c0 + 1; c < c1; ++c) {
        load_agg(s.agg + ((size_t)c * G + g) * 640, lane, x);
        if (s.head[(size_t)c * G + g] != 0u) {
            acc = x;   // starts afresh: ignores what came before
            hd = true;
        } else {
            aff_compose(x, acc, acc);
        }
    }
    store_agg(s.blk_agg + (size_t)wid * 640, lane, acc);
    if (lane == 0) s.blk_head[wid] = hd ? 1u : 0u;
}

// One warp per group: the carry entering each block.
__global__ void __launch_bounds__(256) scan_block_carry(TileScanArgs s)
{
    if (s.done && *(volatile const unsigned *)s.done) return;
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (g >= s.n_groups) return;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (s.cin0) {
        const int b = g / s.gpr, j = (g - b * s.gpr) * 32 + lane;
        if (j < s.d) {
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = s.cin0[((size_t)b * 4 + e) * s.d + j];
        }
    }
    Aff x;
    for (int k = 0; k < s.n_blk; ++k) {
        const size_t w = (size_t)g * s.n_blk + k;
#pragma unroll
        for (int e = 0; e < 4; ++e) s.blk_cin[w * 128 + e * 32 + lane] = v[e];
        if (k + 1 == s.n_blk) break;
        load_agg(s.blk_agg + w * 640, lane, x);
        if (s.blk_head[w] != 0u) {
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = x.b[e];
        } else {
            aff_apply(x, v, v);
        }
    }
}

// (group, block) per warp: the carry entering each tile of the block.
__global__ void __launch_bounds__(256) scan_tile_carry(TileScanArgs s)
{
    if (s.done && *(volatile const unsigned *)s.done) return;
    const int lane = threadIdx.x & 31;
    const long long wid = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (wid >= (long long)s.n_groups * s.n_blk) return;
    const int g = (int)(wid / s.n_blk), k = (int)(wid % s.n_blk);
    const int c0 = k * SCAN_BLK, c1 = min(c0 + SCAN_BLK, s.n_chunks);
    const size_t G = (size_t)s.n_groups;
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = s.blk_cin[(size_t)wid * 128 + e * 32 + lane];
    Aff x;
    for (int c = c0; c < c1; ++c) {
        const size_t t = (size_t)c * G + g;
#pragma unroll
        for (int e = 0; e < 4; ++e) s.cin[t * 128 + e * 32 + lane] = v[e];
        if (c + 1 == c1) break;
        load_agg(s.agg + t * 640, lane, x);
        if (s.head[t] != 0u) {
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = x.b[e];
        } else {
            aff_apply(x, v, v);
        }
    }
}

// The three scan launches on `st`.
inline cudaError_t launch_tile_scan(const TileScanArgs &s, cudaStream_t st)
{
    const long long nw = (long long)s.n_groups * s.n_blk;
    scan_block_agg<<<(unsigned)((nw + 7) / 8), 256, 0, st>>>(s);
    scan_block_carry<<<(s.n_groups + 7) / 8, 256, 0, st>>>(s);
    scan_tile_carry<<<(unsigned)((nw + 7) / 8), 256, 0, st>>>(s);
    return cudaGetLastError();
}

inline int scan_blocks(int n_chunks) { return (n_chunks + SCAN_BLK - 1) / SCAN_BLK; }

// Two passes pay off with few feature groups and a long time axis (measured
// on B200 for the Newton iteration: faster with 8-32 groups from 16 384 steps
// on, slower with 64 groups or 8192 steps).
inline bool prefer_two_pass(int n_groups, long long steps, int sms) { return 4 * n_groups <= sms && steps >= 16384; }

}  // namespace

// cp.async copies into shared memory (zero-fill beyond `bytes`).
SLSTM_DEVINL uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

SLSTM_DEVINL void cp_async16(void *dst, const void *src, int bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(bytes)
                 : "memory");
}

SLSTM_DEVINL void cp_async4(void *dst, const void *src, int bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(bytes)
                 : "memory");
}

SLSTM_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
SLSTM_DEVINL void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
SLSTM_DEVINL void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

}  // namespace slstm
