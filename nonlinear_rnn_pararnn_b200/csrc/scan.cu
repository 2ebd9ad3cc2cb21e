// scan_block4: associative scan of 4x4 affine maps over time, one independent
// recurrence per (batch row, feature) ("pararnn-torch structure", section
// "Naming": scan_block4 for the (B,T,4,4,d) layout; "sLSTM in this library",
// section "Packed sequences": the Newton inner solve is a scan on the (J, r)
// monoid).
//   forward:  y_t = A_t y_{t-1} + b_t,   y_{-1} = y0
//   reverse:  y_t = A_t^T y_{t+1} + b_t, y_T   = y0
// Blocked: each thread folds L steps of one feature serially, warps of a
// tile are combined in shared memory, tiles are chained by a decoupled
// look-back (lookback.cuh).  Composition in fp32.
#include "launchers.h"
#include "lookback.cuh"

namespace slstm {
namespace {

constexpr int NW = 8;
constexpr int L = 4;
constexpr int TT = NW * L;

struct ScanArgs {
    const float *A;
    const float *b;
    const float *y0;
    float *y;
    unsigned *ticket;
    LookbackArgs lb;
    int T, d, groups_per_row;
};

template <bool REVERSE>
SLSTM_DEVINL void load_step(const ScanArgs &a, size_t row, size_t jj, Aff &m)
{
    const size_t d = (size_t)a.d;
    const float *pa = a.A + row * 16 * d + jj;
    const float *pb = a.b + row * 4 * d + jj;
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float v = __ldg(pa + (r * 4 + c) * d);
            if (REVERSE)
                m.a[c * 4 + r] = v;
            else
                m.a[r * 4 + c] = v;
        }
#pragma unroll
    for (int e = 0; e < 4; ++e) m.b[e] = __ldg(pb + e * d);
}

template <bool REVERSE>
__global__ void __launch_bounds__(NW * 32, 2) scan_kernel(ScanArgs a)
{
    __shared__ float s_agg[NW][20][32];
    __shared__ float s_cin[4][32];
    __shared__ unsigned s_ticket;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) s_ticket = atomicAdd(a.ticket, 1u);
    __syncthreads();
    const unsigned ticket = s_ticket;
    const int G = a.lb.n_groups;
    const int chunk = (int)(ticket / (unsigned)G);
    const int grp = (int)(ticket % (unsigned)G);
    const int bb = grp / a.groups_per_row;
    const int j = (grp % a.groups_per_row) * 32 + lane;
    const bool jv = j < a.d;
    const size_t jj = jv ? (size_t)j : 0;
    const size_t d = (size_t)a.d;
    const int T = a.T;
    const int p_seg = chunk * TT + warp * L;
    const size_t row0 = (size_t)bb * T;

    Aff agg;
    aff_identity(agg);
#pragma unroll
    for (int i = 0; i < L; ++i) {
        const int p = p_seg + i;
        if (p < T && jv) {
            const int t = REVERSE ? T - 1 - p : p;
            Aff m;
            load_step<REVERSE>(a, row0 + t, jj, m);
            aff_compose(m, agg, agg);
        }
    }
    store_aff_smem(s_agg, warp, lane, agg);
    __syncthreads();
    tile_prefix_tree<NW>(s_agg, agg);
    if (warp == 0) {
        float first[4] = {0.f, 0.f, 0.f, 0.f};
        if (a.y0 && jv) {
#pragma unroll
            for (int e = 0; e < 4; ++e) first[e] = a.y0[((size_t)bb * 4 + e) * d + jj];
        }
        tile_lookback_warp0<NW>(s_agg, s_cin, a.lb, ticket, chunk, first, false);
    }
    __syncthreads();

    float v[4];
    warp_carry(s_agg, s_cin, warp, lane, v);
#pragma unroll
    for (int i = 0; i < L; ++i) {
        const int p = p_seg + i;
        if (p < T && jv) {
            const int t = REVERSE ? T - 1 - p : p;
            Aff m;
            load_step<REVERSE>(a, row0 + t, jj, m);
            aff_apply(m, v, v);
            float *py = a.y + (row0 + t) * 4 * d + jj;
#pragma unroll
            for (int e = 0; e < 4; ++e) py[e * d] = v[e];
        }
    }
}

struct Layout {
    size_t ticket, flags, agg, inc, total;
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
    l.ticket = take(256);
    l.flags = take(sizeof(unsigned) * (size_t)l.n_tiles);
    l.agg = take(sizeof(float) * 20 * 32 * (size_t)l.n_tiles);
    l.inc = take(sizeof(float) * 4 * 32 * (size_t)l.n_tiles);
    l.total = off;
    return l;
}

}  // namespace

size_t scan_workspace_bytes(int B, int T, int d) { return layout(B, T, d).total; }

cudaError_t scan_block4_launch(const float *A, const float *b, const float *y0, float *y, int B,
                               int T, int d, bool reverse, void *ws, cudaStream_t st)
{
    const Layout l = layout(B, T, d);
    char *base = static_cast<char *>(ws);
    ScanArgs a;
    a.A = A;
    a.b = b;
    a.y0 = y0;
    a.y = y;
    a.ticket = reinterpret_cast<unsigned *>(base + l.ticket);
    a.lb.flags = reinterpret_cast<unsigned *>(base + l.flags);
    a.lb.agg = reinterpret_cast<float *>(base + l.agg);
    a.lb.inc = reinterpret_cast<float *>(base + l.inc);
    a.lb.error = a.ticket + 1;
    a.lb.epoch = 1;
    a.lb.wait_ns = 2000000000ull;
    a.lb.n_groups = l.n_groups;
    a.T = T;
    a.d = d;
    a.groups_per_row = l.groups_per_row;
    // the ticket counter, the error word and every flag start at zero
    cudaError_t e = cudaMemsetAsync(base, 0, l.agg, st);
    if (e != cudaSuccess) return e;
    if (reverse)
        scan_kernel<true><<<l.n_tiles, NW * 32, 0, st>>>(a);
    else
        scan_kernel<false><<<l.n_tiles, NW * 32, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace slstm
