// scan_block4: associative scan of 4x4 affine maps over time, one independent
// recurrence per (batch row, feature) ("pararnn-torch structure", section
// "Naming": scan_block4 for the (B,T,4,4,d) layout; "sLSTM in this library",
// section "Packed sequences": the Newton inner solve is a scan on the (J, r)
// monoid).
//   forward:  y_t = A_t y_{t-1} + b_t,   y_{-1} = y0
//   reverse:  y_t = A_t^T y_{t+1} + b_t, y_T   = y0
// A tile is 32 features x 32 steps (in processing order), one CTA of 8 warps,
// 4 steps per thread.  Persistent CTAs stage the next tile's A and b (80
// bytes per element) in shared memory with cp.async while they scan the
// current one:
//   walk A   each thread folds its 4 maps (dense 4x4 compositions, fp32);
//   carry    the last four warps take the carry entering the tile from the
//            tile before it (its published prefix, read during walk A; the
//            decoupled look-back of lookback.cuh when it is missing) and walk
//            it through the warp maps, one (feature, slot) pair per lane,
//            releasing each other warp as soon as its carry is stored;
//   walk B   each thread applies its maps from its carry and writes y.
#define SLSTM_FILE_ID 3
#include "launchers.h"
#include "lookback.cuh"

namespace slstm {
namespace {

constexpr int NW = 8;
constexpr int L = 4;
constexpr int TT = NW * L;
constexpr int CHAIN0 = NW - 4;          // first chain warp
constexpr int CHAIN_BAR = CHAIN0 + 1;   // the chain warps' own barrier (ids 1 .. CHAIN0: per warp)

struct ScanArgs {
    const float *A;
    const float *b;
    const float *y0;
    float *y;
    unsigned *ticket;
    CarryArgs ca;
    int T, d, groups_per_row, n_tiles, vec16;
    int fault_ticket;   // this tile publishes nothing (host-requested fault injection), or -1
    long long n_b;      // elements of b and y (A has 4 n_b)
    FastDiv div_groups, div_gpr;   // by n_groups and by groups_per_row
};

struct ScanSmem {
    float A[2][TT][16][32];   // [stage][step in processing order][row*4+col][feature]
    float b[2][TT][4][32];
    TileMaps<NW> maps;
    unsigned tick[2];
};

template <bool REVERSE>
SLSTM_DEVINL int step_time(int T, int chunk, int step)
{
    const int p = chunk * TT + step;
    return REVERSE ? T - 1 - p : p;
}

// Copies of one tile's A and b rows into stage `st`; steps outside [0, T)
// and features past d arrive as zeros.
template <bool REVERSE>
SLSTM_DEVINL void scan_prefetch(const ScanArgs &a, ScanSmem &sm, int st, unsigned ticket)
{
    if (ticket >= (unsigned)a.n_tiles) return;
    const int G = a.ca.n_groups;
    const int chunk = (int)fast_div(ticket, a.div_groups);
    const int grp = (int)(ticket - (unsigned)chunk * (unsigned)G);
    const int bb = (int)fast_div((unsigned)grp, a.div_gpr);
    const int j0 = (grp - bb * a.groups_per_row) * 32;
    const int T = a.T;
    const size_t d = (size_t)a.d;
    const size_t row0 = (size_t)bb * T;
    if (a.vec16) {
        // thread (q, c): step q, 16-byte chunk c of each of the 20 rows
        const int c = threadIdx.x & 7, q = threadIdx.x >> 3;
        const int jj = j0 + 4 * c;
        const int t = step_time<REVERSE>(T, chunk, q);
        const int nb = 4 * min(4, a.d - jj);
        const int bytes = (jj < a.d && t >= 0 && t < T &&
                           SLSTM_IN((row0 + t) * 16 * d + jj + 15 * d + nb / 4 - 1, 4 * a.n_b) &&
                           SLSTM_IN((row0 + t) * 4 * d + jj + 3 * d + nb / 4 - 1, a.n_b)) ? nb : 0;
        const float *pa = bytes ? a.A + (row0 + t) * 16 * d + jj : a.A;
        const float *pb = bytes ? a.b + (row0 + t) * 4 * d + jj : a.b;
#pragma unroll
        for (int e = 0; e < 16; ++e) cp_async16(&sm.A[st][q][e][4 * c], bytes ? pa + e * d : a.A, bytes);
#pragma unroll
        for (int e = 0; e < 4; ++e) cp_async16(&sm.b[st][q][e][4 * c], bytes ? pb + e * d : a.b, bytes);
    } else {
        // 4-byte copies, lane = feature; warp w takes steps w, w+8, ...
        const int jl = threadIdx.x & 31, w = threadIdx.x >> 5;
        const bool fj = j0 + jl < a.d;
        for (int q = w; q < TT; q += NW) {
            const int t = step_time<REVERSE>(T, chunk, q);
            const int bytes = (fj && t >= 0 && t < T && SLSTM_IN((row0 + t) * 16 * d + j0 + jl + 15 * d, 4 * a.n_b) &&
                               SLSTM_IN((row0 + t) * 4 * d + j0 + jl + 3 * d, a.n_b)) ? 4 : 0;
            const float *pa = bytes ? a.A + (row0 + t) * 16 * d + j0 + jl : a.A;
            const float *pb = bytes ? a.b + (row0 + t) * 4 * d + j0 + jl : a.b;
#pragma unroll
            for (int e = 0; e < 16; ++e) cp_async4(&sm.A[st][q][e][jl], bytes ? pa + e * d : a.A, bytes);
#pragma unroll
            for (int e = 0; e < 4; ++e) cp_async4(&sm.b[st][q][e][jl], bytes ? pb + e * d : a.b, bytes);
        }
    }
}

// The map of one step from shared memory (transposed matrix in reverse mode).
template <bool REVERSE>
SLSTM_DEVINL void load_map(const ScanSmem &sm, int st, int q, int lane, Aff &m)
{
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float v = sm.A[st][q][r * 4 + c][lane];
            if (REVERSE)
                m.a[c * 4 + r] = v;
            else
                m.a[r * 4 + c] = v;
        }
#pragma unroll
    for (int e = 0; e < 4; ++e) m.b[e] = sm.b[st][q][e][lane];
}

template <bool REVERSE>
__global__ void __launch_bounds__(NW * 32, 1) scan_kernel(ScanArgs a)
{
    extern __shared__ float4 smem_f4[];
    ScanSmem &sm = *reinterpret_cast<ScanSmem *>(smem_f4);
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
    scan_prefetch<REVERSE>(a, sm, 0, cur);
    cp_async_commit();

    while (cur < (unsigned)a.n_tiles) {
        unsigned after = 0;
        if (threadIdx.x == 0) after = atomicAdd(a.ticket, 1u);
        scan_prefetch<REVERSE>(a, sm, st ^ 1, nxt);
        cp_async_commit();
        cp_async_wait_prev();
        __syncthreads();

        const unsigned ticket = cur;
        const int chunk = (int)fast_div(ticket, a.div_groups);
        const int grp = (int)(ticket - (unsigned)chunk * (unsigned)G);
        const int bb = (int)fast_div((unsigned)grp, a.div_gpr);
        const int j = (grp - bb * a.groups_per_row) * 32 + lane;
        const bool jv = j < a.d;
        const size_t jj = jv ? (size_t)j : 0;
        const size_t row0 = (size_t)bb * T;
        const bool chain_warp = warp >= CHAIN0;

        // the predecessor's inclusive prefix (chain lanes), looked at before
        // and halfway through walk A
        const bool look = chain_warp && chunk > 0 && SLSTM_IN(ticket - (unsigned)G, a.n_tiles);
        const unsigned long long *predw = a.ca.incw + chain_word(ticket - (unsigned)G, warp, lane);
        unsigned long long w1 = 0ull, w2 = 0ull;
        if (look) w1 = ld_relaxed_u64(predw);

        // ---- walk A ----
        // the thread's maps stay in registers for walk B (one CTA per SM
        // leaves the whole register file to its 256 threads); steps past T
        // (only in a group's last tile) are skipped
        Aff mp[L];
        Aff agg;
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int q = warp * L + i;
            const bool valid = chunk * TT + q < T;
            if (valid) load_map<REVERSE>(sm, st, q, lane, mp[i]);
            else aff_identity(mp[i]);
            if (i == 0) agg = mp[0];
            else if (valid) aff_compose(mp[i], agg, agg);
            if (i == L / 2 && look) w2 = ld_relaxed_u64(predw);
        }
        maps_store(sm.maps.m, warp, lane, agg);

        // ---- carry ----
        float c = 0.f;
        bool ok = true;
        if (chain_warp && chunk == 0 && a.y0) {
            // chunk 0: y0 enters (chain lane (row, feature))
            const int jf = (grp - bb * a.groups_per_row) * 32 + chain_feature(warp, lane);
            if (jf < a.d && SLSTM_IN(((size_t)bb * 4 + chain_row(lane)) * d + jf, a.n_b / T))
                c = __ldg(a.y0 + ((size_t)bb * 4 + chain_row(lane)) * d + jf);
        }
        if (look) {
            if ((unsigned)(w1 >> 32) == a.ca.epoch) {
                c = __uint_as_float((unsigned)w1);
            } else {
                ok = (unsigned)(w2 >> 32) == a.ca.epoch;
                c = __uint_as_float((unsigned)w2);
            }
        }
        const bool fast = __syncthreads_and(ok);
        const bool withhold = (int)ticket == a.fault_ticket;
        if (chain_warp) {
            if (fast) {
                c = carry_chain4<NW>(sm.maps.m, sm.maps.cin, c, warp, lane, 0u, CHAIN0);
                if (!withhold && SLSTM_IN(chain_word(ticket, warp, lane), (long long)a.n_tiles * 128))
                    st_relaxed_u64(a.ca.incw + chain_word(ticket, warp, lane), inc_word(a.ca.epoch, c));
                named_bar_sync(CHAIN_BAR, 4 * 32);
            } else {
                if (warp == CHAIN0)
                    tile_carry_fallback<NW>(a.ca, sm.maps.m, sm.maps.cin, ticket, chunk, grp, withhold);
                named_bar_sync(CHAIN_BAR, 4 * 32);
#pragma unroll 1
                for (int w = 0; w < CHAIN0; ++w) named_bar_arrive(1 + w, 5 * 32);
            }
        } else {
            named_bar_sync(1 + warp, 5 * 32);   // the carry entering this warp is stored
        }

        // ---- walk B ----
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = sm.maps.cin[warp][e][sw(e, lane)];
#pragma unroll
        for (int i = 0; i < L; ++i) {
            const int q = warp * L + i;
            if (chunk * TT + q < T) {
                const int t = step_time<REVERSE>(T, chunk, q);
                aff_apply(mp[i], v, v);
                float *py = a.y + (row0 + t) * 4 * d + jj;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (jv && SLSTM_PIN(py + e * d, a.y, a.n_b)) py[e * d] = v[e];
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

struct Layout {
    size_t ticket, flags, incw, agg, total;
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
    l.incw = take(sizeof(unsigned long long) * 4 * 32 * (size_t)l.n_tiles);
    l.agg = take(sizeof(float) * 20 * 32 * (size_t)l.n_tiles);
    l.total = off;
    return l;
}

int sm_count_scan()
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

template <bool REVERSE>
cudaError_t launch_scan(const ScanArgs &a, cudaStream_t st)
{
    auto kern = scan_kernel<REVERSE>;
    static int blocks_per_sm = 0;
    if (blocks_per_sm == 0) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(ScanSmem));
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, kern, NW * 32, sizeof(ScanSmem));
        if (e != cudaSuccess) return e;
        if (blocks_per_sm < 1) blocks_per_sm = 1;
    }
    const int grid = min(a.n_tiles, sm_count_scan() * blocks_per_sm);
    kern<<<grid, NW * 32, sizeof(ScanSmem), st>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t scan_workspace_bytes(int B, int T, int d) { return layout(B, T, d).total; }

cudaError_t scan_block4_launch(const float *A, const float *b, const float *y0, float *y, int B,
                               int T, int d, bool reverse, void *ws, cudaStream_t st, bool debug_withhold)
{
    const Layout l = layout(B, T, d);
    char *base = static_cast<char *>(ws);
    ScanArgs a;
    a.A = A;
    a.b = b;
    a.y0 = y0;
    a.y = y;
    a.ticket = reinterpret_cast<unsigned *>(base + l.ticket);
    a.ca.flags = reinterpret_cast<unsigned *>(base + l.flags);
    a.ca.agg = reinterpret_cast<float *>(base + l.agg);
    a.ca.incw = reinterpret_cast<unsigned long long *>(base + l.incw);
    a.ca.error = a.ticket + 1;
    a.ca.epoch = 1;
    // fault injection: the first tile of chunk 1 publishes nothing, so the
    // first tile of chunk 2 gives up after a short wait
    a.fault_ticket = (debug_withhold && l.n_chunks >= 3) ? l.n_groups : -1;
    a.ca.wait_ns = a.fault_ticket >= 0 ? 20000000ull : 2000000000ull;
    a.ca.n_groups = l.n_groups;
    a.ca.n_tiles = l.n_tiles;
    a.n_b = (long long)B * T * 4 * d;
    a.T = T;
    a.d = d;
    a.groups_per_row = l.groups_per_row;
    a.div_groups = make_fastdiv((unsigned)l.n_groups);
    a.div_gpr = make_fastdiv((unsigned)l.groups_per_row);
    a.n_tiles = l.n_tiles;
    a.vec16 = ((d & 3) == 0 && (reinterpret_cast<uintptr_t>(A) & 15) == 0 &&
               (reinterpret_cast<uintptr_t>(b) & 15) == 0) ? 1 : 0;
    // the ticket counter, the error word, every flag and the epoch tags of
    // the inclusive prefixes start at zero
    cudaError_t e = cudaMemsetAsync(base, 0, l.agg, st);
    if (e != cudaSuccess) return e;
    return reverse ? launch_scan<true>(a, st) : launch_scan<false>(a, st);
}

}  // namespace slstm
