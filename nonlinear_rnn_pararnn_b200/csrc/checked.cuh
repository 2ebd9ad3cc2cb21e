// Bounds-checked debug build.  Compiled with -DSLSTM_CHECKED (libslstm_checked.so),
// a guarded global-memory access first tests its element index against the
// extent of its buffer; an index outside [0, extent) skips the access and is
// counted, and the first one is recorded (its site: source file and line, the
// index and the extent) in a device status record of the translation unit,
// which slstm_check_status() gathers.  No trap and no assert: the kernel goes
// on, so a violation is reported, never turned into a fault.  In the normal
// build a guard is the constant true and the record does not exist.
//
// A source that uses the guards defines SLSTM_FILE_ID (an index into the
// file names of slstm_api.cu) before including this header.
#pragma once

#include <cuda_runtime.h>

#ifndef SLSTM_FILE_ID
#define SLSTM_FILE_ID 0
#endif

namespace slstm {

struct CheckRecord {
    unsigned long long count;   // violations seen
    long long site;             // SLSTM_FILE_ID * 100000 + line of the first
    long long index, extent;
};

typedef cudaError_t (*CheckReader)(CheckRecord *out);
typedef cudaError_t (*CheckClearer)();
// Host side: every translation unit of the checked build registers its
// record's reader and clearer when the library is loaded.
int check_register(CheckReader r, CheckClearer c);

#ifdef SLSTM_CHECKED
namespace {
__device__ CheckRecord g_check;

__device__ __noinline__ void check_fail(long long i, long long n, long long site)
{
    if (atomicAdd(&g_check.count, 1ull) == 0ull) {
        g_check.site = site;
        g_check.index = i;
        g_check.extent = n;
    }
}

__device__ __forceinline__ bool check_in(long long i, long long n, long long site)
{
    if (i >= 0 && i < n) return true;
    check_fail(i, n, site);
    return false;
}

cudaError_t check_read(CheckRecord *out) { return cudaMemcpyFromSymbol(out, g_check, sizeof(CheckRecord)); }
cudaError_t check_clear()
{
    const CheckRecord z{0ull, 0, 0, 0};
    return cudaMemcpyToSymbol(g_check, &z, sizeof(z));
}
const int g_check_registered = check_register(check_read, check_clear);
}  // namespace
#define SLSTM_IN(i, n) ::slstm::check_in((long long)(i), (long long)(n), SLSTM_FILE_ID * 100000LL + __LINE__)
#else
#define SLSTM_IN(i, n) true
#endif

// The element at p lies in [base, base + n).
#define SLSTM_PIN(p, base, n) SLSTM_IN((p) - (base), (n))

}  // namespace slstm
