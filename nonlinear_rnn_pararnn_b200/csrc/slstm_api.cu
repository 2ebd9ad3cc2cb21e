// extern "C" entry points of libslstm.so (declared in include/slstm.h).
// Host-side validation happens here, before anything is enqueued; the
// launchers in launchers.h do the work.
#include <stdint.h>

#include "block.h"
#include "checked.cuh"
#include "launchers.h"

using namespace slstm;

namespace {

constexpr long long kIndexLimit = (1LL << 31) - 1;

bool aligned16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned16_or_null(const void *p) { return p == nullptr || aligned16(p); }
bool aligned256(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// Element offsets are 64-bit everywhere; the limits keep B*T (a GEMM row
// count), grid sizes and tile tickets inside 32 bits.
bool sizes_ok(int B, int T, int d_a, int d_b)
{
    if (B < 1 || T < 1 || d_a < 1 || d_b < 1) return false;
    if (B > 65535 || d_a > (1 << 20) || d_b > (1 << 20)) return false;
    if ((long long)B * T > kIndexLimit) return false;
    const long long w = (d_a > d_b ? d_a : d_b);
    const long long tiles = (long long)B * ((T + 31) / 32) * ((w + 31) / 32);
    return tiles <= kIndexLimit;
}

// Packed sequences: n_seq sequences over total_T packed steps (one batch row).
bool varlen_sizes_ok(int n_seq, int total_T, int d_a, int d_b)
{
    return n_seq >= 1 && n_seq <= total_T && sizes_ok(1, total_T, d_a, d_b);
}

bool ws_ok(void *ws, size_t have, size_t need)
{
    if (need == 0) return true;
    return aligned256(ws) && have >= need;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SLSTM_OK : SLSTM_ERR_CUDA; }

// The Newton configuration fields every forward entry point checks.
bool config_ok(const slstm_newton_config &c)
{
    if (c.max_iters < (c.init == SLSTM_INIT_DECOUPLED ? 0 : 1) || c.max_iters > SLSTM_MAX_ITERS) return false;
    if (c.guess_sweeps < 0 || c.guess_sweeps > SLSTM_MAX_GUESS_SWEEPS) return false;
    if (c.forget != SLSTM_FORGET_SIGMOID && c.forget != SLSTM_FORGET_EXP) return false;
    if (!(c.tol >= 0.0f) || c.wait_limit_us < 0) return false;
    if (c.init < SLSTM_INIT_DECOUPLED || c.init > SLSTM_INIT_GIVEN) return false;
    if (c.residual_mode != SLSTM_RESIDUAL_SCALED && c.residual_mode != SLSTM_RESIDUAL_RAW) return false;
    if (c.n_events < 0 || (c.n_events > 0 && c.events == nullptr)) return false;
    if (c.history != SLSTM_HISTORY_BOUND && c.history != SLSTM_HISTORY_EXACT) return false;
    if (c.debug_fault < 0 || c.debug_fault > 3) return false;
    return c.carry_mode >= SLSTM_CARRY_AUTO && c.carry_mode <= SLSTM_CARRY_TWO_PASS;
}

// Head mixing: whole heads of 1..SLSTM_MAX_HEAD_DIM features, one warp per
// (batch row, head) on a one-dimensional grid.
bool head_ok(int d_h, int d_head, int B)
{
    if (d_head < 1 || d_head > SLSTM_MAX_HEAD_DIM || d_h % d_head != 0) return false;
    return (long long)B * (d_h / d_head) <= (1LL << 30);
}

// The trunk layer: K-major bf16 GEMMs over d_model (rows of 16 bytes) and a
// SwiGLU epilogue over blocks of 32 hidden features.
bool block_sizes_ok(int B, int T, int D, int F)
{
    return sizes_ok(B, T, D, F) && D % 8 == 0 && F % 32 == 0;
}

// The trunk backward's column sums (weight gradients of the norms) take the
// B*T rows 256 at a time on the grid's y axis (at most 65535 chunks).
constexpr long long kBlockBwdMaxRows = 65535LL * 256;

}  // namespace

namespace slstm {

namespace {
struct CheckUnit {
    CheckReader read;
    CheckClearer clear;
};
CheckUnit g_units[32];
int g_n_units = 0;
}  // namespace

int check_register(CheckReader r, CheckClearer c)
{
    if (g_n_units < 32) g_units[g_n_units++] = CheckUnit{r, c};
    return g_n_units;
}

}  // namespace slstm

extern "C" {

int slstm_check_enabled(void)
{
#ifdef SLSTM_CHECKED
    return 1;
#else
    return 0;
#endif
}

int slstm_check_status(long long *out)
{
    if (out == nullptr) return SLSTM_ERR_INVALID_ARG;
    for (int i = 0; i < 4; ++i) out[i] = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return SLSTM_ERR_CUDA;
    for (int u = 0; u < g_n_units; ++u) {
        CheckRecord r;
        if (g_units[u].read(&r) != cudaSuccess) return SLSTM_ERR_CUDA;
        if (r.count != 0ull && out[0] == 0) {
            out[1] = r.site;
            out[2] = r.index;
            out[3] = r.extent;
        }
        out[0] += (long long)r.count;
    }
    return SLSTM_OK;
}

int slstm_check_clear(void)
{
    if (cudaDeviceSynchronize() != cudaSuccess) return SLSTM_ERR_CUDA;
    for (int u = 0; u < g_n_units; ++u)
        if (g_units[u].clear() != cudaSuccess) return SLSTM_ERR_CUDA;
    return SLSTM_OK;
}

const char *slstm_check_site_file(int file_id)
{
    static const char *const names[] = {nullptr,         "newton.cu", "backward.cu", "scan.cu",  "sequential.cu",
                                        "varlen.cu",     "decode.cu", "head.cu",     "block.cu", "gemm_simt.cu",
                                        "scan_noalloc.cu"};
    if (file_id < 1 || file_id >= (int)(sizeof(names) / sizeof(names[0]))) return nullptr;
    return names[file_id];
}

const char *slstm_status_string(int status)
{
    switch (status) {
    case SLSTM_OK: return "SLSTM_OK";
    case SLSTM_ERR_INVALID_ARG: return "SLSTM_ERR_INVALID_ARG";
    case SLSTM_ERR_CUDA: return "SLSTM_ERR_CUDA";
    case SLSTM_ERR_DIVERGED: return "SLSTM_ERR_DIVERGED";
    case SLSTM_ERR_TIMEOUT: return "SLSTM_ERR_TIMEOUT";
    case SLSTM_ERR_UNSUPPORTED: return "SLSTM_ERR_UNSUPPORTED";
    default: return "SLSTM_UNKNOWN_STATUS";
    }
}

size_t slstm_workspace_size(int op, int B, int T, int d_in, int d_h)
{
    switch (op) {
    case SLSTM_OP_PREACT_GEMM:
        if (!sizes_ok(B, T, d_in, d_h)) return 0;
        return preact_workspace_bytes(B, T, d_in, d_h, SLSTM_BF16);
    case SLSTM_OP_NEWTON_FORWARD:
        if (!sizes_ok(B, T, d_h, d_h)) return 0;
        return newton_workspace_bytes(B, T, d_h);
    case SLSTM_OP_SCAN_BLOCK4:
        if (!sizes_ok(B, T, d_h, d_h)) return 0;
        return scan_workspace_bytes(B, T, d_h);
    case SLSTM_OP_NEWTON_BACKWARD:
        if (!sizes_ok(B, T, d_in, d_h)) return 0;
        return backward_workspace_bytes(B, T, d_in, d_h);
    case SLSTM_OP_NEWTON_FORWARD_VARLEN:
        if (!varlen_sizes_ok(B, T, d_h, d_h)) return 0;
        return varlen_table_bytes(T) + newton_workspace_bytes(1, T, d_h);
    case SLSTM_OP_NEWTON_BACKWARD_VARLEN:
        if (!varlen_sizes_ok(B, T, d_in, d_h)) return 0;
        return varlen_table_bytes(T) + backward_workspace_bytes(1, T, d_in, d_h);
    case SLSTM_OP_CONTEXT_PARALLEL:
        if (!sizes_ok(B, T, d_h, d_h)) return 0;
        return cp_workspace_bytes(B, T, d_h);
    case SLSTM_OP_NEWTON_BACKWARD_HEAD:
        if (!sizes_ok(B, T, d_in, d_h)) return 0;
        return head_backward_workspace_bytes(B, T, d_in, d_h, SLSTM_MAX_HEAD_DIM);
    default: return 0;
    }
}

int slstm_preact_gemm(const void *x, const void *Wx, int dtype, const float *bias, float *P, int B,
                      int T, int d_in, int d_h, void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (dtype != SLSTM_F32 && dtype != SLSTM_BF16) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, d_in, d_h)) return SLSTM_ERR_INVALID_ARG;
    if (dtype == SLSTM_BF16 && d_in % 8 != 0) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wx) || !aligned16(bias) || !aligned16(P)) return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, preact_workspace_bytes(B, T, d_in, d_h, dtype))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(preact_launch(x, Wx, dtype, bias, P, B, T, d_in, d_h, ws,
                                     static_cast<cudaStream_t>(stream)));
}

int slstm_set_gemm_tiles(int tiles) { return gemm_tc_set_tiles(tiles); }

int slstm_newton_forward(const float *P, const float *R, const float *s0, float *S,
                         const slstm_newton_config *cfg, slstm_newton_stats *stats, int B, int T,
                         int d_h, void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (cfg == nullptr) return SLSTM_ERR_INVALID_ARG;
    if (!config_ok(*cfg)) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, d_h, d_h)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(P) || !aligned16(R) || !aligned16_or_null(s0) || !aligned16(S) || !aligned16(stats))
        return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, newton_workspace_bytes(B, T, d_h))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(newton_forward(P, R, s0, S, *cfg, stats, B, T, d_h, ws,
                                      static_cast<cudaStream_t>(stream)));
}

int scan_block4(const float *A, const float *b, const float *y0, float *y, int B, int T, int d,
                int flags, void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if ((flags & ~(SLSTM_SCAN_REVERSE_T | SLSTM_SCAN_DEBUG_WITHHOLD)) != 0) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, d, d)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(b) || !aligned16_or_null(y0) || !aligned16(y)) return SLSTM_ERR_INVALID_ARG;
    if (y == A || y == b) return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, scan_workspace_bytes(B, T, d))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(scan_block4_launch(A, b, y0, y, B, T, d, (flags & SLSTM_SCAN_REVERSE_T) != 0, ws,
                                          static_cast<cudaStream_t>(stream),
                                          (flags & SLSTM_SCAN_DEBUG_WITHHOLD) != 0));
}

int slstm_cp_guess_run(const float *P, const float *R, const float *s_before, const float *S, int sweep, int forget,
                       float *run, int B, int T, int d_h, void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (forget != SLSTM_FORGET_SIGMOID && forget != SLSTM_FORGET_EXP) return SLSTM_ERR_INVALID_ARG;
    if (sweep != 0 && sweep != 1) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, d_h, d_h)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(P) || !aligned16(R) || !aligned16(run)) return SLSTM_ERR_INVALID_ARG;
    if (sweep && (!aligned16(S) || !aligned16_or_null(s_before))) return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, cp_workspace_bytes(B, T, d_h))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(cp_guess_run(P, R, s_before, S, sweep != 0, forget, run, B, T, d_h, ws,
                                    static_cast<cudaStream_t>(stream)));
}

int slstm_cp_guess_apply(const float *P, const float *R, const float *s0, const float *s_before, const float *runs,
                         int rank, float *S, int sweep, int forget, int B, int T, int d_h, void *ws, size_t ws_bytes,
                         slstm_stream_t stream)
{
    if (forget != SLSTM_FORGET_SIGMOID && forget != SLSTM_FORGET_EXP) return SLSTM_ERR_INVALID_ARG;
    if (sweep != 0 && sweep != 1) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, d_h, d_h) || rank < 0 || rank > 65535) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(P) || !aligned16(R) || !aligned16_or_null(s0) || !aligned16_or_null(s_before) || !aligned16(S))
        return SLSTM_ERR_INVALID_ARG;
    if (rank > 0 && !aligned16(runs)) return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, cp_workspace_bytes(B, T, d_h))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(cp_guess_apply(P, R, s0, s_before, runs, rank, S, sweep != 0, forget, B, T, d_h, ws,
                                      static_cast<cudaStream_t>(stream)));
}

int slstm_cp_newton_map(const float *P, const float *R, const float *s_before, const float *S, int forget, float *map,
                        int B, int T, int d_h, void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (forget != SLSTM_FORGET_SIGMOID && forget != SLSTM_FORGET_EXP) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, d_h, d_h)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(P) || !aligned16(R) || !aligned16_or_null(s_before) || !aligned16(S) || !aligned16(map))
        return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, cp_workspace_bytes(B, T, d_h))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(cp_newton_map(P, R, s_before, S, forget, map, B, T, d_h, ws, static_cast<cudaStream_t>(stream)));
}

int slstm_cp_newton_apply(const float *P, const float *R, const float *s_before, const float *maps, int rank,
                          float *S, const slstm_newton_config *cfg, slstm_newton_stats *stats, int B, int T, int d_h,
                          void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (cfg == nullptr || !config_ok(*cfg)) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, d_h, d_h) || rank < 0 || rank > 65535) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(P) || !aligned16(R) || !aligned16_or_null(s_before) || !aligned16(S) || !aligned16(stats))
        return SLSTM_ERR_INVALID_ARG;
    if (rank > 0 && !aligned16(maps)) return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, cp_workspace_bytes(B, T, d_h))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(cp_newton_apply(P, R, s_before, maps, rank, S, *cfg, stats, B, T, d_h, ws,
                                       static_cast<cudaStream_t>(stream)));
}

int slstm_sequential_step_head(const float *P, const float *R_head, const float *s0, float *S, int B, int T_steps,
                               int d_h, int d_head, int forget, slstm_stream_t stream)
{
    if (forget != SLSTM_FORGET_SIGMOID && forget != SLSTM_FORGET_EXP) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T_steps, d_h, d_h) || !head_ok(d_h, d_head, B)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(P) || !aligned16(R_head) || !aligned16_or_null(s0) || !aligned16(S)) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(head_sequential_launch(P, R_head, s0, S, B, T_steps, d_h, d_head, forget,
                                              static_cast<cudaStream_t>(stream)));
}

int slstm_newton_forward_head(const float *P, const float *R_head, const float *s0, float *S,
                              const slstm_newton_config *cfg, slstm_newton_stats *stats, int B, int T, int d_h,
                              int d_head, void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (cfg == nullptr || !config_ok(*cfg) || cfg->debug_fault != 0 || cfg->guess_sweeps != 0)
        return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, d_h, d_h) || !head_ok(d_h, d_head, B)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(P) || !aligned16(R_head) || !aligned16_or_null(s0) || !aligned16(S) || !aligned16(stats))
        return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, newton_workspace_bytes(B, T, d_h))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(head_newton_forward(P, R_head, s0, S, *cfg, stats, B, T, d_h, d_head, ws,
                                           static_cast<cudaStream_t>(stream)));
}

int slstm_newton_backward_head(const void *x, const void *Wx, int dtype, const float *P, const float *R_head,
                               const float *s0, const float *S, const float *dH, float *dx, float *dWx,
                               float *dR_head, float *db, float *ds0, int forget, int B, int T, int d_in, int d_h,
                               int d_head, void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (dtype != SLSTM_F32 && dtype != SLSTM_BF16) return SLSTM_ERR_INVALID_ARG;
    if (forget != SLSTM_FORGET_SIGMOID && forget != SLSTM_FORGET_EXP) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, d_in, d_h) || !head_ok(d_h, d_head, B)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wx) || !aligned16(P) || !aligned16(R_head) || !aligned16_or_null(s0) ||
        !aligned16(S) || !aligned16(dH) || !aligned16(dx) || !aligned16(dWx) || !aligned16(dR_head) ||
        !aligned16(db) || !aligned16_or_null(ds0))
        return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, head_backward_workspace_bytes(B, T, d_in, d_h, SLSTM_MAX_HEAD_DIM)))
        return SLSTM_ERR_INVALID_ARG;
    return cuda_status(head_backward_launch(x, Wx, dtype, P, R_head, s0, S, dH, dx, dWx, dR_head, db, ds0, forget,
                                            B, T, d_in, d_h, d_head, ws, static_cast<cudaStream_t>(stream)));
}

int slstm_sequential_step(const float *P, const float *R, const float *s0, float *S, int B,
                          int T_steps, int d_h, int forget, slstm_stream_t stream)
{
    if (forget != SLSTM_FORGET_SIGMOID && forget != SLSTM_FORGET_EXP) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T_steps, d_h, d_h)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(P) || !aligned16(R) || !aligned16_or_null(s0) || !aligned16(S)) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(sequential_launch(P, R, s0, S, B, T_steps, d_h, forget,
                                         static_cast<cudaStream_t>(stream)));
}

int slstm_decode_step(const void *x, const void *Wx, int dtype, const float *bias, const float *R,
                      const float *s_prev, float *s_next, int forget, int B, int d_in, int d_h,
                      slstm_stream_t stream)
{
    if (dtype != SLSTM_F32 && dtype != SLSTM_BF16) return SLSTM_ERR_INVALID_ARG;
    if (forget != SLSTM_FORGET_SIGMOID && forget != SLSTM_FORGET_EXP) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, 1, d_in, d_h)) return SLSTM_ERR_INVALID_ARG;
    if (d_in % (dtype == SLSTM_BF16 ? 8 : 4) != 0) return SLSTM_ERR_INVALID_ARG;   // 16-byte rows
    if (!aligned16(x) || !aligned16(Wx) || !aligned16(bias) || !aligned16(R) || !aligned16_or_null(s_prev) ||
        !aligned16(s_next))
        return SLSTM_ERR_INVALID_ARG;
    return cuda_status(decode_launch(x, Wx, dtype, bias, R, s_prev, s_next, forget, B, d_in, d_h,
                                     static_cast<cudaStream_t>(stream)));
}

int slstm_newton_backward(const void *x, const void *Wx, int dtype, const float *P, const float *R,
                          const float *s0, const float *S, const float *dH, float *dx, float *dWx,
                          float *dR, float *db, float *ds0, int forget, int B, int T, int d_in,
                          int d_h, void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (dtype != SLSTM_F32 && dtype != SLSTM_BF16) return SLSTM_ERR_INVALID_ARG;
    if (forget != SLSTM_FORGET_SIGMOID && forget != SLSTM_FORGET_EXP) return SLSTM_ERR_INVALID_ARG;
    if (!sizes_ok(B, T, d_in, d_h)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wx) || !aligned16(P) || !aligned16(R) || !aligned16_or_null(s0) ||
        !aligned16(S) || !aligned16(dH) || !aligned16(dx) || !aligned16(dWx) || !aligned16(dR) ||
        !aligned16(db) || !aligned16_or_null(ds0))
        return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, backward_workspace_bytes(B, T, d_in, d_h))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(backward_launch(x, Wx, dtype, P, R, s0, S, dH, dx, dWx, dR, db, ds0, forget, B, T,
                                       d_in, d_h, ws, static_cast<cudaStream_t>(stream)));
}

int slstm_newton_forward_varlen(const float *P, const float *R, const float *s0, const int *cu_seqlens, int n_seq,
                                float *S, const slstm_newton_config *cfg, slstm_newton_stats *stats, int total_T,
                                int d_h, void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (cfg == nullptr || cu_seqlens == nullptr) return SLSTM_ERR_INVALID_ARG;
    if (!config_ok(*cfg)) return SLSTM_ERR_INVALID_ARG;
    if (!varlen_sizes_ok(n_seq, total_T, d_h, d_h)) return SLSTM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(P) || !aligned16(R) || !aligned16_or_null(s0) || !aligned16(S) || !aligned16(stats))
        return SLSTM_ERR_INVALID_ARG;
    const size_t vt = varlen_table_bytes(total_T);
    if (!ws_ok(ws, ws_bytes, vt + newton_workspace_bytes(1, total_T, d_h))) return SLSTM_ERR_INVALID_ARG;
    const Varlen vl = varlen_layout(cu_seqlens, n_seq, total_T, ws);
    return cuda_status(newton_forward(P, R, s0, S, *cfg, stats, 1, total_T, d_h, static_cast<char *>(ws) + vt,
                                      static_cast<cudaStream_t>(stream), &vl));
}

int slstm_newton_backward_varlen(const void *x, const void *Wx, int dtype, const float *P, const float *R,
                                 const float *s0, const int *cu_seqlens, int n_seq, const float *S,
                                 const float *dH, float *dx, float *dWx, float *dR, float *db, float *ds0,
                                 int forget, int total_T, int d_in, int d_h, void *ws, size_t ws_bytes,
                                 slstm_stream_t stream)
{
    if (dtype != SLSTM_F32 && dtype != SLSTM_BF16) return SLSTM_ERR_INVALID_ARG;
    if (forget != SLSTM_FORGET_SIGMOID && forget != SLSTM_FORGET_EXP) return SLSTM_ERR_INVALID_ARG;
    if (cu_seqlens == nullptr || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return SLSTM_ERR_INVALID_ARG;
    if (!varlen_sizes_ok(n_seq, total_T, d_in, d_h)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(Wx) || !aligned16(P) || !aligned16(R) || !aligned16_or_null(s0) ||
        !aligned16(S) || !aligned16(dH) || !aligned16(dx) || !aligned16(dWx) || !aligned16(dR) ||
        !aligned16(db) || !aligned16_or_null(ds0))
        return SLSTM_ERR_INVALID_ARG;
    const size_t vt = varlen_table_bytes(total_T);
    if (!ws_ok(ws, ws_bytes, vt + backward_workspace_bytes(1, total_T, d_in, d_h))) return SLSTM_ERR_INVALID_ARG;
    const Varlen vl = varlen_layout(cu_seqlens, n_seq, total_T, ws);
    return cuda_status(backward_launch(x, Wx, dtype, P, R, s0, S, dH, dx, dWx, dR, db, ds0, forget, 1, total_T,
                                       d_in, d_h, static_cast<char *>(ws) + vt, static_cast<cudaStream_t>(stream),
                                       &vl));
}

size_t slstm_block_workspace_size(int B, int T, int d_model, int d_ff)
{
    if (!block_sizes_ok(B, T, d_model, d_ff)) return 0;
    return block_workspace_bytes(B, T, d_model, d_ff);
}

int slstm_block_forward(const float *x, const float *norm1_w, const void *Wx, const float *bias, const float *R,
                        const float *norm2_w, const void *W_gu, const void *W_down, float *y, float *S,
                        const slstm_newton_config *cfg, slstm_newton_stats *stats, int B, int T, int d_model,
                        int d_ff, float eps, void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (cfg == nullptr) return SLSTM_ERR_INVALID_ARG;
    if (!config_ok(*cfg)) return SLSTM_ERR_INVALID_ARG;
    if (!block_sizes_ok(B, T, d_model, d_ff)) return SLSTM_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !(eps < 1e30f)) return SLSTM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(norm1_w) || !aligned16(Wx) || !aligned16(bias) || !aligned16(R) ||
        !aligned16(norm2_w) || !aligned16(W_gu) || !aligned16(W_down) || !aligned16(y) || !aligned16(S) ||
        !aligned16(stats))
        return SLSTM_ERR_INVALID_ARG;
    const size_t M = (size_t)B * T;
    const char *yb = reinterpret_cast<const char *>(y), *sb = reinterpret_cast<const char *>(S);
    if (yb < sb + M * 16 * d_model && sb < yb + M * 4 * d_model) return SLSTM_ERR_INVALID_ARG;   // y overlaps S
    if (!ws_ok(ws, ws_bytes, block_workspace_bytes(B, T, d_model, d_ff))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(block_forward_launch(x, norm1_w, Wx, bias, R, norm2_w, W_gu, W_down, y, S, *cfg, stats, B, T,
                                            d_model, d_ff, eps, ws, static_cast<cudaStream_t>(stream)));
}

size_t slstm_block_backward_workspace_size(int B, int T, int d_model, int d_ff)
{
    if (!block_sizes_ok(B, T, d_model, d_ff)) return 0;
    return block_backward_workspace_bytes(B, T, d_model, d_ff);
}

int slstm_block_backward(const float *x, const float *norm1_w, const void *Wx, const float *bias, const float *R,
                         const float *norm2_w, const void *W_gu, const void *W_down, const float *S, const float *dY,
                         float *dx, float *dnorm1_w, float *dWx, float *dbias, float *dR, float *dnorm2_w,
                         float *dW_gu, float *dW_down, int forget, int B, int T, int d_model, int d_ff, float eps,
                         void *ws, size_t ws_bytes, slstm_stream_t stream)
{
    if (forget != SLSTM_FORGET_SIGMOID && forget != SLSTM_FORGET_EXP) return SLSTM_ERR_INVALID_ARG;
    if (!block_sizes_ok(B, T, d_model, d_ff)) return SLSTM_ERR_INVALID_ARG;
    if ((long long)B * T > kBlockBwdMaxRows) return SLSTM_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !(eps < 1e30f)) return SLSTM_ERR_INVALID_ARG;
    const void *ptrs[] = {x, norm1_w, Wx, bias, R, norm2_w, W_gu, W_down, S, dY,
                          dx, dnorm1_w, dWx, dbias, dR, dnorm2_w, dW_gu, dW_down};
    for (const void *p : ptrs)
        if (!aligned16(p)) return SLSTM_ERR_INVALID_ARG;
    if (!ws_ok(ws, ws_bytes, block_backward_workspace_bytes(B, T, d_model, d_ff))) return SLSTM_ERR_INVALID_ARG;
    return cuda_status(block_backward_launch(x, norm1_w, Wx, bias, R, norm2_w, W_gu, W_down, S, dY, dx, dnorm1_w, dWx,
                                             dbias, dR, dnorm2_w, dW_gu, dW_down, forget, B, T, d_model, d_ff, eps, ws,
                                             static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
