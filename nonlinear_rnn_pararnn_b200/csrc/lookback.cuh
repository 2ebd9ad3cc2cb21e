// Blocked scan of 4x4 affine maps across CTAs with a decoupled look-back.
//
// A "tile" is 32 features x (NW warps x L steps).  Inside a tile every warp
// folds its own L steps serially (one feature per lane).  The NW warp
// aggregates are turned into inclusive prefixes by a Kogge-Stone tree in
// shared memory (all warps work, log2 NW levels).  Warp 0 then publishes the
// tile aggregate, looks back over the tiles before it (same feature group,
// earlier in processing order) until it meets a published inclusive prefix,
// and publishes its own; every warp finally derives its incoming carry from
// the tile carry and its predecessor's prefix.
//
// Tiles take tickets from a global counter in the order CTAs start, and tile
// (chunk c, group g) has ticket c * n_groups + g, so a tile only ever waits
// on tiles that started before it: every wait ends.  Waits are bounded in
// time anyway; on expiry the tile records an error, continues with a zero
// carry and still publishes, so that no other tile waits on it.
//
// Global state per tile (ticket):  flag word, aggregate [20][32] and
// inclusive prefix [4][32] (feature-contiguous so that a warp moves 128-byte
// rows).
#pragma once

#include "common.cuh"

namespace slstm {

struct LookbackArgs {
    unsigned *flags;   // [n_tiles]
    float *agg;        // [n_tiles][20][32]
    float *inc;        // [n_tiles][4][32]
    unsigned *error;   // set to nonzero when a wait expires
    unsigned epoch;    // nonzero, unique per launch since the flags were cleared
    uint64_t wait_ns;  // bound of one wait
    int n_groups;      // feature groups (tiles per chunk)
};

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

// All threads of the CTA.  On entry s_agg[w] holds warp w's aggregate (in
// processing order) and `mine` the same value in registers; on exit s_agg[w]
// holds the inclusive prefix agg_w o ... o agg_0.  Ends with a barrier.
template <int NW>
SLSTM_DEVINL void tile_prefix_tree(float (*s_agg)[20][32], Aff &mine)
{
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < NW; off <<= 1) {
        Aff left;
        if (warp >= off) load_aff_smem(s_agg, warp - off, lane, left);
        __syncthreads();
        if (warp >= off) {
            aff_compose(mine, left, mine);
            store_aff_smem(s_agg, warp, lane, mine);
        }
        __syncthreads();
    }
}

// Warp 0 only, after tile_prefix_tree.  Publishes the tile aggregate
// (s_agg[NW-1]), looks back, publishes the inclusive prefix and writes the
// carry entering the tile to s_cin[0..3][lane].  `first_carry` is the value
// entering chunk 0.  `withhold` suppresses this tile's publications (fault
// injection).
template <int NW>
SLSTM_DEVINL void tile_lookback_warp0(float (*s_agg)[20][32], float (*s_cin)[32],
                                      const LookbackArgs &lb, unsigned ticket, int chunk,
                                      const float first_carry[4], bool withhold)
{
    const int lane = threadIdx.x & 31;
    Aff tile;
    load_aff_smem(s_agg, NW - 1, lane, tile);

    float carry[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) carry[e] = first_carry[e];

    if (chunk > 0) {
        if (!withhold) {
            float *dst = lb.agg + (size_t)ticket * 20 * 32;
#pragma unroll
            for (int e = 0; e < 16; ++e) dst[e * 32 + lane] = tile.a[e];
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[(16 + e) * 32 + lane] = tile.b[e];
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release(lb.flags + ticket, (lb.epoch << 2) | FLAG_AGG);
        }
        Aff M;  // composition of the aggregates met so far (latest first)
        aff_identity(M);
        int q = chunk - 1;
        bool expired = false;
        const unsigned grp = ticket % (unsigned)lb.n_groups;
        for (;;) {
            const unsigned tq = (unsigned)q * (unsigned)lb.n_groups + grp;
            unsigned st = 0;
            if (lane == 0) st = wait_flag(lb.flags + tq, lb.epoch, lb.wait_ns);
            st = __shfl_sync(0xffffffffu, st, 0);
            if (st == 0u) {
                expired = true;
#pragma unroll
                for (int e = 0; e < 4; ++e) carry[e] = 0.0f;
                break;
            }
            if (st == FLAG_INC) {
                float v[4];
                const float *src = lb.inc + (size_t)tq * 4 * 32;
#pragma unroll
                for (int e = 0; e < 4; ++e) v[e] = __ldcg(src + e * 32 + lane);
                aff_apply(M, v, carry);
                break;
            }
            Aff x;
            const float *src = lb.agg + (size_t)tq * 20 * 32;
#pragma unroll
            for (int e = 0; e < 16; ++e) x.a[e] = __ldcg(src + e * 32 + lane);
#pragma unroll
            for (int e = 0; e < 4; ++e) x.b[e] = __ldcg(src + (16 + e) * 32 + lane);
            aff_compose(M, x, M);
            --q;  // chunk 0 always publishes an inclusive prefix, so q stays >= 0
        }
        if (expired && lane == 0) atomicOr(lb.error, 1u);
    }

    if (!withhold) {
        float incv[4];
        aff_apply(tile, carry, incv);
        float *dst = lb.inc + (size_t)ticket * 4 * 32;
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e * 32 + lane] = incv[e];
        __threadfence();
        __syncwarp();
        if (lane == 0) st_release(lb.flags + ticket, (lb.epoch << 2) | FLAG_INC);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) s_cin[e][lane] = carry[e];
}

// Any warp, after the barrier that follows tile_lookback_warp0: the carry
// entering warp `warp` of the tile.
SLSTM_DEVINL void warp_carry(float (*s_agg)[20][32], float (*s_cin)[32], int warp, int lane,
                             float out[4])
{
    float cin[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) cin[e] = s_cin[e][lane];
    if (warp == 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) out[e] = cin[e];
        return;
    }
    Aff pre;
    load_aff_smem(s_agg, warp - 1, lane, pre);
    aff_apply(pre, cin, out);
}

// ---------------------------------------------------------------------------
// Carry hand-off used by the persistent kernels (Newton iteration, adjoint).
// A tile's inclusive prefix (4 values per feature) is published as 64-bit
// words (value bits | epoch << 32): a reader validates and reads it with one
// load per word and the writer needs no fence.  The epoch tags are cleared
// at the start of every call, and each launch of the call has its own epoch.
// A tile whose predecessor has not published yet publishes its aggregate
// (gated by the per-tile flag word) and looks back past unfinished tiles.
// ---------------------------------------------------------------------------
struct CarryArgs {
    unsigned *flags;              // [n_tiles]
    float *agg;                   // [n_tiles][20][32]
    unsigned long long *incw;     // [n_tiles][4][32]
    unsigned *error;
    unsigned epoch;
    unsigned long long wait_ns;
    int n_groups;
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

// This lane's part of tile tq's inclusive prefix, if published in this launch.
SLSTM_DEVINL bool read_inc_words(const CarryArgs &ca, unsigned tq, int lane, float v[4])
{
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

// Warp 0 only.  s_agg[w] holds warp w's own aggregate (in processing order).
// Writes the carry entering every warp to s_cin[w] and publishes the tile's
// inclusive prefix.  `first` enters chunk 0; `withhold` suppresses this
// tile's publications (fault injection).  In the common case (predecessor
// published) only 4-vectors move: v_{w+1} = A_w v_w + b_w; the 4x4 tile
// aggregate is formed only when it must be published.  `pre_ok` / `pre`: the
// predecessor's prefix as read earlier by the caller (to overlap the load's
// latency with other work); it is read again here when that read was early.
template <int NW>
SLSTM_DEVINL void tile_carry_serial(const CarryArgs &ca, float (*s_agg)[20][32], float (*s_cin)[4][32],
                                    unsigned ticket, int chunk, int grp, const float first[4], bool withhold,
                                    bool pre_ok = false, const float *pre = nullptr)
{
    const int lane = threadIdx.x & 31;
    float carry[4] = {first[0], first[1], first[2], first[3]};
    if (chunk > 0) {
        unsigned tq = ticket - (unsigned)ca.n_groups;
        float v[4];
        bool ok = pre_ok && (pre != nullptr);
        if (ok) {
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = pre[e];
        }
        if (!__all_sync(0xffffffffu, ok)) ok = read_inc_words(ca, tq, lane, v);
        if (__all_sync(0xffffffffu, ok)) {
#pragma unroll
            for (int e = 0; e < 4; ++e) carry[e] = v[e];
        } else {
            Aff tile;
            load_aff_smem(s_agg, 0, lane, tile);
            for (int w = 1; w < NW; ++w) {
                Aff x;
                load_aff_smem(s_agg, w, lane, x);
                aff_compose(x, tile, tile);
            }
            if (!withhold) {
                float *dst = ca.agg + (size_t)ticket * 20 * 32;
#pragma unroll
                for (int e = 0; e < 16; ++e) dst[e * 32 + lane] = tile.a[e];
#pragma unroll
                for (int e = 0; e < 4; ++e) dst[(16 + e) * 32 + lane] = tile.b[e];
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release(ca.flags + ticket, (ca.epoch << 2) | FLAG_AGG);
            }
            Aff M;
            aff_identity(M);
            int q = chunk - 1;
            const uint64_t t0 = globaltimer_ns();
            unsigned polls = 0;
            for (;;) {
                tq = (unsigned)q * (unsigned)ca.n_groups + (unsigned)grp;
                if (read_inc_words(ca, tq, lane, v)) {
                    aff_apply(M, v, carry);
                    break;
                }
                const unsigned f = ld_acquire(ca.flags + tq);
                if ((f >> 2) == ca.epoch && (f & 3u) == FLAG_AGG) {
                    Aff x;
                    const float *src = ca.agg + (size_t)tq * 20 * 32;
#pragma unroll
                    for (int e = 0; e < 16; ++e) x.a[e] = __ldcg(src + e * 32 + lane);
#pragma unroll
                    for (int e = 0; e < 4; ++e) x.b[e] = __ldcg(src + (16 + e) * 32 + lane);
                    aff_compose(M, x, M);
                    --q;   // chunk 0 never publishes an aggregate, so q stays >= 0
                    continue;
                }
                if (++polls > 16) __nanosleep(64);
                if (globaltimer_ns() - t0 > ca.wait_ns) {
                    atomicOr(ca.error, 1u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) carry[e] = 0.f;
                    break;
                }
            }
        }
    }
    // the next warp's map is loaded while the current one is applied
    float v[4] = {carry[0], carry[1], carry[2], carry[3]};
    Aff x;
    load_aff_smem(s_agg, 0, lane, x);
#pragma unroll
    for (int w = 0; w < NW; ++w) {
#pragma unroll
        for (int e = 0; e < 4; ++e) s_cin[w][e][lane] = v[e];
        Aff xn;
        if (w + 1 < NW) load_aff_smem(s_agg, w + 1, lane, xn);
        aff_apply(x, v, v);
        if (w + 1 < NW) x = xn;
    }
    if (!withhold) {
        unsigned long long *dst = ca.incw + (size_t)ticket * 4 * 32 + lane;
#pragma unroll
        for (int e = 0; e < 4; ++e)
            st_relaxed_u64(dst + e * 32, ((unsigned long long)ca.epoch << 32) | __float_as_uint(v[e]));
    }
}

// Value component e (slot order c, n, m, h) of a cell evaluation; e is a
// compile-time constant after unrolling.
SLSTM_DEVINL float cell_f(const Cell &c, int e) { return e == 0 ? c.c : (e == 1 ? c.n : (e == 2 ? c.m : c.h)); }

// Named CTA barriers for a producer warp handing a value to a consumer warp:
// the producer arrives, the consumer waits; `n` counts both warps' threads.
SLSTM_DEVINL void named_bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
SLSTM_DEVINL void named_bar_arrive(int id, int n) { asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory"); }

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

// Copy one row of 32 consecutive floats (src, 16-byte aligned when vec16)
// into shared memory; only `valid` leading floats are read, the rest become
// zero.  Called by 8 lanes (vec16: 16 bytes each) or 32 lanes (4 bytes each);
// `part` is the caller's index within that group.
SLSTM_DEVINL void copy_row32(float *dst, const float *src, int valid, bool vec16, int part)
{
    if (vec16) {
        const int f0 = 4 * part;
        const int bytes = valid > f0 ? 4 * min(4, valid - f0) : 0;
        cp_async16(dst + f0, bytes ? src + f0 : src, bytes);
    } else {
        const int bytes = valid > part ? 4 : 0;
        cp_async4(dst + part, bytes ? src + part : src, bytes);
    }
}

// Fold one step's map (J, r) into a running aggregate: agg <- (J, r) o agg.
SLSTM_DEVINL void fold_jac(Aff &agg, const Cell &J, const float r[4])
{
#pragma unroll
    for (int col = 0; col < 4; ++col)
        jac_mul(J, agg.a[col], agg.a[4 + col], agg.a[8 + col], agg.a[12 + col]);
    jac_mul(J, agg.b[0], agg.b[1], agg.b[2], agg.b[3]);
#pragma unroll
    for (int e = 0; e < 4; ++e) agg.b[e] += r[e];
}

// Same with the transposed Jacobian: agg <- (J^T, r) o agg.
SLSTM_DEVINL void fold_jacT(Aff &agg, const Cell &J, const float r[4])
{
#pragma unroll
    for (int col = 0; col < 4; ++col)
        jacT_mul(J, agg.a[col], agg.a[4 + col], agg.a[8 + col], agg.a[12 + col]);
    jacT_mul(J, agg.b[0], agg.b[1], agg.b[2], agg.b[3]);
#pragma unroll
    for (int e = 0; e < 4; ++e) agg.b[e] += r[e];
}

SLSTM_DEVINL void cell_identity(Cell &J)
{
    J.fp = 1.0f;
    J.jcm = J.jch = J.jnm = J.jnh = 0.0f;
    J.beta = 1.0f;
    J.dmh = 0.0f;
    J.jhc = J.jhn = J.jhm = 0.0f;
    J.jhh = 1.0f;
}

}  // namespace slstm
