// Shared device code for libslstm: the fp32 sLSTM cell with its Jacobian in
// registers, 4x4 affine-map algebra, and the bounded publish / look-back
// primitives of the blocked scans.
//
// The cell follows "xLSTM - a from-scratch, educational reimplementation"
// (section "Exponential gating + the stabilizer") and the summary "xLSTM:
// Extended Long Short-Term Memory" (section "Method", sLSTM step: gate order
// z, i, f, o and read-out h = o * c / n), with the diag mixing of "sLSTM in
// this library" (section "Cell": channelwise R of shape (4, d_h), a 4x4
// Jacobian per feature).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/slstm.h"

#define SLSTM_DEVINL __device__ __forceinline__

namespace slstm {

// ---------------------------------------------------------------------------
// Cell
// ---------------------------------------------------------------------------

// Value and Jacobian of one step s_t = f(s_{t-1}, P_t) for one feature.
// The Jacobian d s_t / d s_{t-1} has the sparsity pattern
//   [ fp   0    jcm  jch ]
//   [ 0    fp   jnm  jnh ]
//   [ 0    0    beta dmh ]
//   [ jhc  jhn  jhm  jhh ]
// (rows and columns in slot order c, n, m, h).
struct Cell {
    float c, n, m, h;
    float fp, jcm, jch, jnm, jnh, beta, dmh, jhc, jhn, jhm, jhh;
};

// The step's Jacobian set to zero: the step does not depend on the one before
// (the first step of a packed sequence).
SLSTM_DEVINL void cell_zero_jac(Cell &J)
{
    J.fp = J.jcm = J.jch = J.jnm = J.jnh = J.beta = J.dmh = J.jhc = J.jhn = J.jhm = J.jhh = 0.0f;
}

// Gate-space derivative G = d s_t / d a_t, nonzero pattern (columns z,i,f,o):
//   [ gcz gci gcf 0   ]
//   [ 0   gni gnf 0   ]
//   [ 0   gmi gmf 0   ]
//   [ ghz ghi ghf gho ]
struct CellG {
    float gcz, gci, gcf, gni, gnf, gmi, gmf, ghz, ghi, ghf, gho;
};

// The factors of G that the adjoint keeps for its second walk.  The gates see
// h_{t-1} only through the diagonal r (a_t = P_t + r h_{t-1}), so the h
// column of J is G r, and with
//   mu_c = lam_c + on lam_h,   mu_n = lam_n - ony lam_h,   X = gci mu_c + gni mu_n
// both products follow from eight numbers:
//   G^T lam = (gcz mu_c,  X + (1 - fb) lam_m,  dlf (fb lam_m - X),  gho lam_h)
//   J^T lam = (fp mu_c,   fp mu_n,             fb lam_m - X,        r . G^T lam)
// where on = o / n, ony = o c / n^2, dlf = d log f / d a_f, fb = 1 on the forget
// branch of the stabiliser's max and 0 on the input branch, and
// dlfs = fb ? dlf : -dlf carries fb in its sign bit.
struct CellB {
    float fp, gci, gni, on, ony, gcz, dlfs, gho;
};

// Transcendentals on the MUFU pipe through CUDA's fast intrinsics (__expf,
// __logf, __fdividef), combined by the identities
//   sigmoid(x) = 1 / (1 + e^{-x}),   tanh(x) = 1 - 2 / (1 + e^{2x}).
// Both stay finite for any x: e^{..} = inf gives 1/inf = 0.
SLSTM_DEVINL float sigmoid_fast(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
SLSTM_DEVINL float tanh_fast(float x) { return 1.0f - __fdividef(2.0f, 1.0f + __expf(2.0f * x)); }

// forget: SLSTM_FORGET_SIGMOID or SLSTM_FORGET_EXP.  WANT_J: fill the
// Jacobian fields.  WANT_G: fill *g.
template <int FORGET, bool WANT_J, bool WANT_G = false, bool WANT_B = false>
SLSTM_DEVINL void cell_eval(float c0, float n0, float m0, float h0, float pz, float pi, float pf,
                            float po, float rz, float ri, float rf, float ro, Cell &o,
                            CellG *g = nullptr, CellB *bq = nullptr)
{
    const float az = fmaf(rz, h0, pz);
    const float ai = fmaf(ri, h0, pi);
    const float af = fmaf(rf, h0, pf);
    const float ao = fmaf(ro, h0, po);
    const float z = tanh_fast(az);
    const float og = sigmoid_fast(ao);
    float lf, dlf;
    if (FORGET == SLSTM_FORGET_EXP) {
        lf = af;
        dlf = 1.0f;
    } else {
        // log sigmoid(af) = min(af, 0) - log1p(exp(-|af|)); its derivative
        // is sigmoid(-af).
        const float e = __expf(-fabsf(af));
        const float ope = 1.0f + e;
        lf = fminf(af, 0.0f) - __logf(ope);
        dlf = __fdividef(af >= 0.0f ? e : 1.0f, ope);
    }
    const float u = lf + m0;
    const bool fb = (u >= ai);  // forget branch of the max
    const float m = fb ? u : ai;
    const float e = __expf(-fabsf(u - ai));
    const float fp = fb ? 1.0f : e;  // exp(u - m)
    const float ip = fb ? e : 1.0f;  // exp(ai - m)
    const float c = fmaf(fp, c0, ip * z);
    const float n = fmaf(fp, n0, ip);
    const float inv_n = __fdividef(1.0f, n);
    const float y = c * inv_n;
    o.c = c;
    o.n = n;
    o.m = m;
    o.h = og * y;
    if (WANT_J || WANT_G || WANT_B) {
        const float on = og * inv_n;
        const float dz = 1.0f - z * z;
        if (WANT_B) {
            bq->fp = fp;
            bq->gci = fb ? ip * z : -fp * c0;
            bq->gni = fb ? ip : -fp * n0;
            bq->on = on;
            bq->ony = on * y;
            bq->gcz = ip * dz;
            bq->dlfs = fb ? dlf : -dlf;
            bq->gho = y * og * (1.0f - og);
        }
        if (WANT_J) {
            // d(log f') / d h0 - d(log i') / d h0 = dlf * rf - ri; only one of
            // the two is nonzero, selected by the branch of the max.
            const float d = fmaf(dlf, rf, -ri);
            const float jcm = fb ? -ip * z : fp * c0;
            const float jnm = fb ? -ip : fp * n0;
            const float q = ip * dz * rz;
            const float jch = fmaf(jcm, d, q);
            const float jnh = jnm * d;
            o.fp = fp;
            o.jcm = jcm;
            o.jch = jch;
            o.jnm = jnm;
            o.jnh = jnh;
            o.beta = fb ? 1.0f : 0.0f;
            o.dmh = fb ? dlf * rf : ri;
            o.jhc = on * fp;
            o.jhn = -o.jhc * y;
            o.jhm = on * fmaf(-y, jnm, jcm);
            o.jhh = fmaf(on, fmaf(-y, jnh, jch), y * og * (1.0f - og) * ro);
        }
        if (WANT_G) {
            // a_i moves m only on the input branch, a_f only on the forget branch.
            const float gci = fb ? ip * z : -fp * c0;
            const float gni = fb ? ip : -fp * n0;
            const float gcf = fb ? -ip * z * dlf : fp * c0 * dlf;
            const float gnf = fb ? -ip * dlf : fp * n0 * dlf;
            g->gcz = ip * dz;
            g->gci = gci;
            g->gcf = gcf;
            g->gni = gni;
            g->gnf = gnf;
            g->gmi = fb ? 0.0f : 1.0f;
            g->gmf = fb ? dlf : 0.0f;
            g->ghz = on * g->gcz;
            g->ghi = on * fmaf(-y, gni, gci);
            g->ghf = on * fmaf(-y, gnf, gcf);
            g->gho = y * og * (1.0f - og);
        }
    }
}

// ---------------------------------------------------------------------------
// Affine maps v -> A v + b on 4-vectors
// ---------------------------------------------------------------------------
struct Aff {
    float a[16];  // row-major
    float b[4];
};

SLSTM_DEVINL void aff_identity(Aff &x)
{
#pragma unroll
    for (int i = 0; i < 16; ++i) x.a[i] = (i % 5 == 0) ? 1.0f : 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) x.b[i] = 0.0f;
}

// out = second o first (apply `first`, then `second`).
SLSTM_DEVINL void aff_compose(const Aff &second, const Aff &first, Aff &out)
{
    Aff r;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float acc = 0.0f;
#pragma unroll
            for (int l = 0; l < 4; ++l) acc = fmaf(second.a[i * 4 + l], first.a[l * 4 + k], acc);
            r.a[i * 4 + k] = acc;
        }
        float acc = second.b[i];
#pragma unroll
        for (int l = 0; l < 4; ++l) acc = fmaf(second.a[i * 4 + l], first.b[l], acc);
        r.b[i] = acc;
    }
    out = r;
}

SLSTM_DEVINL void aff_apply(const Aff &m, const float v[4], float out[4])
{
    float r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float acc = m.b[i];
#pragma unroll
        for (int l = 0; l < 4; ++l) acc = fmaf(m.a[i * 4 + l], v[l], acc);
        r[i] = acc;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = r[i];
}

// x <- J x for the sparse cell Jacobian, x a column 4-vector.
SLSTM_DEVINL void jac_mul(const Cell &J, float &x0, float &x1, float &x2, float &x3)
{
    const float y0 = fmaf(J.fp, x0, fmaf(J.jcm, x2, J.jch * x3));
    const float y1 = fmaf(J.fp, x1, fmaf(J.jnm, x2, J.jnh * x3));
    const float y2 = fmaf(J.beta, x2, J.dmh * x3);
    const float y3 = fmaf(J.jhc, x0, fmaf(J.jhn, x1, fmaf(J.jhm, x2, J.jhh * x3)));
    x0 = y0;
    x1 = y1;
    x2 = y2;
    x3 = y3;
}

// y = J x + a for the sparse cell Jacobian, with a entering the innermost
// fused multiply-add of each row.
SLSTM_DEVINL void jac_mul_add(const Cell &J, const float x[4], const float a[4], float y[4])
{
    y[0] = fmaf(J.fp, x[0], fmaf(J.jcm, x[2], fmaf(J.jch, x[3], a[0])));
    y[1] = fmaf(J.fp, x[1], fmaf(J.jnm, x[2], fmaf(J.jnh, x[3], a[1])));
    y[2] = fmaf(J.beta, x[2], fmaf(J.dmh, x[3], a[2]));
    y[3] = fmaf(J.jhc, x[0], fmaf(J.jhn, x[1], fmaf(J.jhm, x[2], fmaf(J.jhh, x[3], a[3]))));
}

// x <- J^T x for the sparse cell Jacobian.
SLSTM_DEVINL void jacT_mul(const Cell &J, float &x0, float &x1, float &x2, float &x3)
{
    const float y0 = fmaf(J.fp, x0, J.jhc * x3);
    const float y1 = fmaf(J.fp, x1, J.jhn * x3);
    const float y2 = fmaf(J.jcm, x0, fmaf(J.jnm, x1, fmaf(J.beta, x2, J.jhm * x3)));
    const float y3 = fmaf(J.jch, x0, fmaf(J.jnh, x1, fmaf(J.dmh, x2, J.jhh * x3)));
    x0 = y0;
    x1 = y1;
    x2 = y2;
    x3 = y3;
}

// ---------------------------------------------------------------------------
// Look-back flag word of a tile: (epoch << 2) | FLAG_AGG once the tile's
// aggregate is published.  A fresh epoch per launch means stale words never
// match.
// ---------------------------------------------------------------------------
constexpr unsigned FLAG_AGG = 1u;

SLSTM_DEVINL unsigned ld_acquire(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

SLSTM_DEVINL void st_release(unsigned *p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

SLSTM_DEVINL uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Division by a divisor d >= 1 that is fixed for a launch, for dividends below
// 2^31: q = (n * M) >> (32 + s) with s = ceil(log2 d) and the round-up
// multiplier M = ceil(2^(32+s) / d) < 2^33 (Granlund and Montgomery,
// "Division by invariant integers using multiplication", 1994).  Turns the
// per-tile ticket decode into a multiply and a shift.
struct FastDiv {
    unsigned long long mul;
    unsigned shift;
    unsigned d;
};

inline FastDiv make_fastdiv(unsigned d)
{
    unsigned s = 0;
    while ((1ull << s) < d) ++s;
    FastDiv f;
    f.mul = ((1ull << (32 + s)) + d - 1) / d;
    f.shift = 32 + s;
    f.d = d;
    return f;
}

SLSTM_DEVINL unsigned fast_div(unsigned n, const FastDiv &f)
{
    return (unsigned)(((unsigned long long)n * f.mul) >> f.shift);
}

// Non-negative float max through its bit pattern (NaN sorts above +inf).
// Named CTA barriers (ids 1..15; id 0 is __syncthreads).  `count` threads,
// a multiple of 32, take part; whole warps call these.
SLSTM_DEVINL void named_bar_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

SLSTM_DEVINL void named_bar_arrive(int id, int count)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

SLSTM_DEVINL void atomic_max_nonneg(unsigned *slot, float v)
{
    atomicMax(slot, __float_as_uint(fabsf(v)));
}

// max(a, b), NaN when either is NaN (fmaxf would drop it): a non-finite
// residual stays visible through every reduction.
SLSTM_DEVINL float fmax_nan(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

SLSTM_DEVINL float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax_nan(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

}  // namespace slstm
