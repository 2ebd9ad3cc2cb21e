// Head flags of packed ragged sequences ("sLSTM in this library", "Packed
// sequences": FlashAttention-style exclusive-prefix offsets cu_seqlens, a
// head flag at each cu_seqlens[:-1]).  One thread per sequence marks the
// first step of each nonempty sequence in a bit mask (one word per 32 packed
// steps, the tile height of the Newton and adjoint kernels) and records the
// sequence index there.  Offsets are clamped into [0, total_T], so malformed
// input can never lead to an out-of-range access; it is reported instead.
#define SLSTM_FILE_ID 5
#include "checked.cuh"
#include "launchers.h"

namespace slstm {
namespace {

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

__global__ void varlen_table_kernel(const int *__restrict__ cu, int n_seq, int total_T, unsigned *mask, int *seq,
                                    unsigned *err, slstm_newton_stats *stats, unsigned *done)
{
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n_seq || !SLSTM_IN(k + 1, n_seq + 1)) return;
    int a = cu[k], b = cu[k + 1];
    const bool bad = a < 0 || b < a || b > total_T || (k == 0 && a != 0) || (k == n_seq - 1 && b != total_T);
    if (bad) {
        atomicOr(err, 1u);
        if (stats) stats->error = SLSTM_ERR_INVALID_ARG;
        if (done) atomicExch(done, 1u);
    }
    a = min(max(a, 0), total_T);
    b = min(max(b, 0), total_T);
    if (b > a && SLSTM_IN(a >> 5, (total_T + 31) / 32) && SLSTM_IN(a, total_T)) {
        atomicOr(&mask[a >> 5], 1u << (a & 31));
        seq[a] = k;
    }
}

}  // namespace

size_t varlen_table_bytes(int total_T)
{
    const size_t chunks = ((size_t)total_T + 31) / 32;
    return align256(4 * chunks) + align256(4 * (size_t)total_T) + 256;
}

Varlen varlen_layout(const int *cu, int n_seq, int total_T, void *ws)
{
    char *base = static_cast<char *>(ws);
    const size_t chunks = ((size_t)total_T + 31) / 32;
    Varlen v;
    v.cu = cu;
    v.n_seq = n_seq;
    v.mask = reinterpret_cast<unsigned *>(base);
    v.seq = reinterpret_cast<int *>(base + align256(4 * chunks));
    v.err = reinterpret_cast<unsigned *>(base + align256(4 * chunks) + align256(4 * (size_t)total_T));
    return v;
}

cudaError_t varlen_build(const Varlen &v, int total_T, slstm_newton_stats *stats, unsigned *done, cudaStream_t st)
{
    const size_t chunks = ((size_t)total_T + 31) / 32;
    cudaError_t e = cudaMemsetAsync(v.mask, 0, 4 * chunks, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(v.err, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return e;
    varlen_table_kernel<<<(v.n_seq + 255) / 256, 256, 0, st>>>(v.cu, v.n_seq, total_T, v.mask, v.seq, v.err, stats,
                                                              done);
    return cudaGetLastError();
}

}  // namespace slstm
