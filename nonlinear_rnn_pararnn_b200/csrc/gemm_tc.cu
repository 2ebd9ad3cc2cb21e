// bf16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM, fed by TMA):
//   C[m][n] = sum_k A[m][k] B[n][k] + bias[n]     (A, B bf16, K-major; C fp32)
// The input projection P = x W_x^T + b is this product with A = x (rows
// (b,t)), B = W_x (rows (g,j)) ("sLSTM in this library", section "API
// notes": W_x is a GEMM).
//
// Persistent CTAs (one per SM) walk 128 x 256 tiles of C (and split-K
// slices), n fastest so that the A rows of a tile row are reused from L2:
//   warp 0, one lane   TMA producer: A and B k-blocks (64 wide, 128-byte
//                      swizzle) into a 4-stage ring guarded by mbarriers;
//   warp 1, one lane   MMA issuer: tcgen05.mma (M=128, N=256, K=16) into one
//                      of two 256-column fp32 accumulators in TMEM, so that a
//                      tile's epilogue overlaps the next tile's main loop;
//   warps 2-5          epilogue: tcgen05.ld of their TMEM lane quarter, + bias,
//                      16-column slices staged in shared memory (four
//                      buffers) and written by TMA stores (plain stores when C
//                      rows are not 16-byte aligned).
// gemm_tc2_kernel is the same product on SM pairs (clusters of two CTAs,
// tcgen05 cta_group::2, 256 x 256 tiles), taken for long K where clusters of
// two can run; gemm_tc_kernel uses no clusters.  No multicast form anywhere.
// Every mbarrier wait is bounded in time; on expiry the CTA records an
// error, waits (bounded) for the loads and MMAs it issued, frees its TMEM and
// returns.
#include <cuda_bf16.h>
#include <string.h>

#include "block.h"
#include "launchers.h"
#include "tma.cuh"

namespace slstm {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr uint32_t A_STAGE = BM * BK * 2;   // 16 KB
constexpr uint32_t B_STAGE = BN * BK * 2;   // 32 KB
constexpr uint32_t STAGE_BYTES = A_STAGE + B_STAGE;
constexpr uint32_t TMEM_COLS = 2 * BN;      // two accumulators: one tile's epilogue overlaps the next one's MMAs
constexpr int EPI_COLS = 32;                // columns per TMEM load of the epilogue
constexpr int STORE_COLS = 16;              // columns per store box (64 bytes of fp32, 64-byte swizzle)
constexpr uint32_t STORE_BYTES = BM * STORE_COLS * 4;   // 8 KB
constexpr int STORE_BUFS = 4;               // staging buffers: up to three stores still reading
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STORE_BUFS * STORE_BYTES + 1024 + 256;
constexpr int THREADS = 192;                // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint64_t WAIT_NS = 1000000000ull;   // 1 s bound on any single wait

struct TcArgs {
    float *C;
    const float *bias;      // [N] or null
    int M, N, K;
    int a_parts;            // 1, or 2: C = (A0 + A1) B^T with A1 from the second map
    int kb_per_split;       // k-blocks of the virtual K (a_parts * ceil(K/64)) per split
    int m_tiles, n_tiles, n_work;   // work item w = (split, m tile, n tile), n fastest
    int tma_out;            // the epilogue stores through the C tensor map
    long long c_split;      // element offset between the C slices of the splits
    unsigned *error;
    int epi;                // GEMM_EPI_STORE, GEMM_EPI_SWIGLU or GEMM_EPI_RESIDUAL
    __nv_bfloat16 *Cb;      // GEMM_EPI_SWIGLU: the [M][N/2] bf16 product
    const float *res;       // GEMM_EPI_RESIDUAL: C = acc + res, res [M][N] (may be C)
};

// At most N of this thread's bulk store groups still read shared memory.
template <int N>
SLSTM_DEVINL void bulk_wait_read_n()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Named barrier with an OR reduction over `n` threads: every participant
// gets the same answer.
SLSTM_DEVINL bool bar_or(int id, int n, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n"
        " .reg .pred p, q;\n"
        " setp.ne.u32 p, %1, 0;\n"
        " bar.red.or.pred q, %2, %3, p;\n"
        " selp.u32 %0, 1, 0, q;\n"
        "}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0u;
}

SLSTM_DEVINL void bar_named(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// Shared-memory matrix descriptor of a K-major bf16 tile written by TMA with
// 128-byte swizzle: rows of 128 bytes, 8-row swizzle atoms 1024 bytes apart.
SLSTM_DEVINL uint64_t smem_desc_k_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);   // start address
    d |= (uint64_t)1u << 16;                     // leading byte offset (unused when swizzled)
    d |= (uint64_t)(1024u >> 4) << 32;           // stride byte offset: next 8-row atom
    d |= (uint64_t)1u << 46;                     // descriptor version for sm_100
    d |= (uint64_t)2u << 61;                     // 128-byte swizzle
    return d;
}

// Shared-memory matrix descriptor of an MN-major bf16 tile written by TMA as
// 64-element-wide boxes with 128-byte swizzle: each box is BK K-rows of 128
// bytes (one 64-element MN atom), boxes `atom_stride` bytes apart; 8-row K
// groups are 1024 bytes apart.
SLSTM_DEVINL uint64_t smem_desc_mn_sw128(uint32_t saddr, uint32_t atom_stride)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);        // start address
    d |= (uint64_t)((atom_stride >> 4) & 0x3FFFu) << 16;  // leading byte offset: next MN atom
    d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset: next 8-row K group
    d |= (uint64_t)1u << 46;                          // descriptor version for sm_100
    d |= (uint64_t)2u << 61;                          // 128-byte swizzle
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, M x N;
// a_mn / b_mn select MN-major (transposed) operands.
constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

SLSTM_DEVINL void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
        "}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

SLSTM_DEVINL void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

SLSTM_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
SLSTM_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
SLSTM_DEVINL void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// One 32-column chunk of an epilogue thread's TMEM lane (row `row` of the
// tile, v = its accumulator columns col0 .. col0 + 31): the SwiGLU product
// (which takes the next chunk too, advancing c and chunk), or the residual
// and bias added and the result stored, staged through BUFS 16-column
// shared-memory buffers in turn when C is written by TMA.
template <int BUFS>
SLSTM_DEVINL void epilogue_chunk(const TcArgs &g, const CUtensorMap *tmc, uint8_t *sE, float (&v)[32],
                                 uint32_t lane_addr, int &c, int &chunk, int m0, int row, int et, int col0, int z)
{
    if (g.epi == GEMM_EPI_SWIGLU) {
        // columns 64k .. 64k+31 are the gate of features 32k ..
        // 32k+31, columns 64k+32 .. 64k+63 their up projection:
        // write silu(gate) * up of the 32 features as bf16
        float u[32];
        tmem_ld32(lane_addr + (uint32_t)((c + 1) * EPI_COLS), u);
        ++c;
        ++chunk;
        const int grow = m0 + row;
        if (grow < g.M && col0 < g.N) {
            uint4 *dst = reinterpret_cast<uint4 *>(g.Cb + (size_t)grow * (g.N >> 1) + (col0 >> 1));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t w[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int i = 8 * j + 2 * h;
                    // silu(v) = v / (1 + e^-v); the fast divide returns 0 once
                    // the denominator passes 2^126, where silu is 0 to fp32 anyway
                    const float a0 = __fdividef(v[i], 1.0f + __expf(-v[i])) * u[i];
                    const float a1 = __fdividef(v[i + 1], 1.0f + __expf(-v[i + 1])) * u[i + 1];
                    const __nv_bfloat162 pr = __floats2bfloat162_rn(a0, a1);
                    w[h] = *reinterpret_cast<const uint32_t *>(&pr);
                }
                dst[j] = make_uint4(w[0], w[1], w[2], w[3]);
            }
        }
        return;
    }
    if (g.epi == GEMM_EPI_RESIDUAL) {
        const int grow = m0 + row;
        if (grow < g.M) {
            const float *src = g.res + (size_t)grow * g.N + col0;
            if ((g.N & 3) == 0 && col0 + 32 <= g.N) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 r4 = *reinterpret_cast<const float4 *>(src + 4 * j);
                    v[4 * j] += r4.x;
                    v[4 * j + 1] += r4.y;
                    v[4 * j + 2] += r4.z;
                    v[4 * j + 3] += r4.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (col0 + i < g.N) v[i] += src[i];
            }
        }
    }
    if (g.bias) {
        if ((g.N & 3) == 0 && col0 + 32 <= g.N && (reinterpret_cast<uintptr_t>(g.bias) & 15) == 0) {
            const float4 *b4 = reinterpret_cast<const float4 *>(g.bias + col0);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 bv = __ldg(b4 + j);
                v[4 * j] += bv.x;
                v[4 * j + 1] += bv.y;
                v[4 * j + 2] += bv.z;
                v[4 * j + 3] += bv.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += (col0 + i < g.N) ? __ldg(g.bias + col0 + i) : 0.0f;
        }
    }
    if (g.tma_out) {
        // two boxes of 16 columns, each staged in the next of the BUFS
        // buffers (row `row`, 16-byte piece j at piece j ^ ((row >> 1)
        // & 3): the tensor map's 64-byte swizzle) once the store that
        // last read that buffer is done with it
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            uint8_t *buf_e = sE + ((2 * chunk + hf) % BUFS) * STORE_BYTES;
            if (et == 0) bulk_wait_read_n<BUFS - 1>();
            bar_named(1, 128);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<float4 *>(buf_e + row * 64 + ((j ^ ((row >> 1) & 3)) << 4)) =
                    make_float4(v[16 * hf + 4 * j], v[16 * hf + 4 * j + 1], v[16 * hf + 4 * j + 2],
                                v[16 * hf + 4 * j + 3]);
            tma_store_fence();
            bar_named(1, 128);
            if (et == 0) {
                tma_store_3d(tmc, buf_e, col0 + STORE_COLS * hf, m0, z);
                bulk_commit();
            }
        }
    } else {
        const int grow = m0 + row;
        if (grow < g.M) {
            float *dst = g.C + (size_t)z * g.c_split + (size_t)grow * g.N + col0;
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (col0 + i < g.N) dst[i] = v[i];
        }
    }
}

// A_MN / B_MN: the operand is stored MN-major ([K][M] or [K][N], MN
// contiguous) instead of K-major; its tile is then loaded as 64-wide boxes.
//
// Persistent: CTA c takes work items c, c + gridDim.x, ...  Roles:
//   warp 0, one lane   TMA producer over every item's k-blocks (4-stage ring);
//   warp 1, one lane   MMA issuer; item i accumulates in TMEM columns
//                      [256 (i & 1), 256 (i & 1) + 256), handed to the
//                      epilogue by tcgen05.commit and back by an mbarrier;
//   warps 2-5          epilogue: TMEM lane quarter (warp & 3), + bias, then
//                      16-column slices staged in shared memory (64-byte
//                      swizzle) and written by TMA stores, four staging buffers.
template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tma2,
                   const __grid_constant__ CUtensorMap tmb, const __grid_constant__ CUtensorMap tmc, TcArgs g)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * A_STAGE;
    uint8_t *sE = smem + STAGES * STAGE_BYTES;   // 1024-aligned: the swizzle pattern is address based
    uint64_t *full = reinterpret_cast<uint64_t *>(sE + STORE_BUFS * STORE_BYTES);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;    // [2] accumulator ready
    uint64_t *tempty = tfull + 2;        // [2] accumulator drained (4 epilogue warps)
    uint64_t *fin = tempty + 2;          // every MMA issued has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + 1);
    __shared__ int s_abort;
    __shared__ int s_issued, s_consumed;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nk_part = (g.K + BK - 1) / BK;
    const int total_kb = g.a_parts * nk_part;
    const int per_split = g.m_tiles * g.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(fin, 1);
        mbar_init_fence();
        s_abort = 0;
        s_issued = 0;
        s_consumed = 0;
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer ----
            int gkb = 0;
            bool stop = false;
            for (int w = blockIdx.x; w < g.n_work && !stop; w += gridDim.x) {
                const int z = w / per_split;
                const int r = w - z * per_split;
                const int m0 = (r / g.n_tiles) * BM, n0 = (r % g.n_tiles) * BN;
                const int kb0 = z * g.kb_per_split;
                const int nkb = min(g.kb_per_split, total_kb - kb0);
                for (int kb = 0; kb < nkb; ++kb, ++gkb) {
                    const int s = gkb % STAGES;
                    const uint32_t ph = (uint32_t)(gkb / STAGES) & 1u;
                    if (*(volatile int *)&s_abort || !mbar_wait(&empty[s], ph ^ 1u, WAIT_NS)) {
                        s_abort = 1;
                        stop = true;
                        break;
                    }
                    const int vk = kb0 + kb;
                    const int part = vk / nk_part;
                    const int kk = vk - part * nk_part;
                    mbar_expect_tx(&full[s], STAGE_BYTES);
                    const CUtensorMap *am = part ? &tma2 : &tma;
                    if (A_MN) {
#pragma unroll
                        for (int i = 0; i < BM / 64; ++i)
                            tma_load_2d(sA + s * A_STAGE + i * (BK * 128), am, &full[s], m0 + 64 * i, kk * BK);
                    } else {
                        tma_load_2d(sA + s * A_STAGE, am, &full[s], kk * BK, m0);
                    }
                    if (B_MN) {
#pragma unroll
                        for (int i = 0; i < BN / 64; ++i)
                            tma_load_2d(sB + s * B_STAGE + i * (BK * 128), &tmb, &full[s], n0 + 64 * i, kk * BK);
                    } else {
                        tma_load_2d(sB + s * B_STAGE, &tmb, &full[s], kk * BK, n0);
                    }
                }
            }
            s_issued = gkb;
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer ----
            constexpr uint32_t idesc = idesc_bf16(BM, BN, A_MN, B_MN);
            constexpr uint64_t a_step = A_MN ? (2048u >> 4) : (32u >> 4);
            constexpr uint64_t b_step = B_MN ? (2048u >> 4) : (32u >> 4);
            int gkb = 0, lt = 0;
            bool stop = false;
            for (int w = blockIdx.x; w < g.n_work && !stop; w += gridDim.x, ++lt) {
                const int z = w / per_split;
                const int nkb = min(g.kb_per_split, total_kb - z * g.kb_per_split);
                const int buf = lt & 1;
                if (*(volatile int *)&s_abort || !mbar_wait(&tempty[buf], ((uint32_t)(lt >> 1) & 1u) ^ 1u, WAIT_NS)) {
                    s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(buf * BN);
                for (int kb = 0; kb < nkb; ++kb, ++gkb) {
                    const int s = gkb % STAGES;
                    const uint32_t ph = (uint32_t)(gkb / STAGES) & 1u;
                    if (*(volatile int *)&s_abort || !mbar_wait(&full[s], ph, WAIT_NS)) {
                        s_abort = 1;
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    // per MMA step of K = 16: K-major tiles advance 32 bytes along
                    // the swizzled row, MN-major tiles advance 16 K-rows (2048 bytes)
                    const uint64_t ad = A_MN ? smem_desc_mn_sw128(smem_u32(sA + s * A_STAGE), BK * 128)
                                             : smem_desc_k_sw128(smem_u32(sA + s * A_STAGE));
                    const uint64_t bd = B_MN ? smem_desc_mn_sw128(smem_u32(sB + s * B_STAGE), BK * 128)
                                             : smem_desc_k_sw128(smem_u32(sB + s * B_STAGE));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_bf16(acc, ad + a_step * k, bd + b_step * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                if (!stop) umma_commit(&tfull[buf]);
            }
            s_consumed = gkb;
            umma_commit(fin);   // fires when every MMA issued above has completed
        }
    } else {
        // ---- epilogue: warps 2-5, TMEM lane quarter q = warp & 3 ----
        const int q = warp & 3;
        const int et = threadIdx.x - 64;   // 0..127
        const int row = q * 32 + lane;     // row within the tile
        int lt = 0, chunk = 0;
        for (int w = blockIdx.x; w < g.n_work; w += gridDim.x, ++lt) {
            const int z = w / per_split;
            const int r = w - z * per_split;
            const int m0 = (r / g.n_tiles) * BM, n0 = (r % g.n_tiles) * BN;
            const int buf = lt & 1;
            const bool got = !*(volatile int *)&s_abort && mbar_wait(&tfull[buf], (uint32_t)(lt >> 1) & 1u, WAIT_NS);
            if (bar_or(1, 128, !got)) {
                s_abort = 1;
                break;
            }
            tc_fence_after();
            const uint32_t lane_addr = tmem + (uint32_t)(buf * BN) + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
            for (int c = 0; c < BN / EPI_COLS; ++c, ++chunk) {
                float v[32];
                tmem_ld32(lane_addr + (uint32_t)(c * EPI_COLS), v);
                const int col0 = n0 + c * EPI_COLS;
                epilogue_chunk<STORE_BUFS>(g, &tmc, sE, v, lane_addr, c, chunk, m0, row, et, col0, z);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
        }
        if (et == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && s_abort) {
        atomicOr(g.error, 1u);
        // loads issued but never consumed still land in this CTA's shared
        // memory, and issued MMAs still write TMEM: wait for both (bounded)
        for (int kb = s_consumed; kb < s_issued; ++kb)
            (void)mbar_wait(&full[kb % STAGES], (uint32_t)(kb / STAGES) & 1u, WAIT_NS);
    }
    if (threadIdx.x == 0) (void)mbar_wait(fin, 0u, WAIT_NS);
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// ---------------------------------------------------------------------------
// SM-pair tiles (tcgen05 cta_group::2).  A cluster of two CTAs on a pair of
// SMs computes a 256 x 256 tile of C with M = 256 MMAs issued by the even CTA
// (the leader): each CTA loads its own 128 rows of A and its own 128 rows of
// B (the two halves of the tile's N range) into its shared memory, the pair's
// tensor cores read both, and each CTA's TMEM holds the accumulator of its
// 128 rows x 256 columns.  Per CTA and k-block the ring holds 32 KB instead
// of 48 (the other half of B sits in the peer), so it is six stages deep
// (the single-SM kernel's is four) beside the same four staging buffers.
// Synchronisation, all through mbarriers:
//   full[s]    leader's: both CTAs' loads of stage s complete their bytes on
//              it (the leader arms it with both CTAs' byte counts);
//   empty[s]   each CTA's own: the leader's MMAs commit to both CTAs' copies
//              (two commits, no multicast form) once stage s is consumed;
//   tfull[b]   each CTA's own: accumulator b is ready (two commits);
//   tempty[b]  leader's: the eight epilogue warps of the pair arrive (four
//              remotely) once accumulator b is drained.
// No TMA load names another CTA's memory or another GPU's; no multicast.
// ---------------------------------------------------------------------------
constexpr int STAGES2 = 6;
constexpr int BNH = BN / 2;                               // rows of B per CTA
constexpr uint32_t B_HALF = BNH * BK * 2;                 // 16 KB
constexpr uint32_t STAGE2_BYTES = A_STAGE + B_HALF;       // 32 KB per CTA and stage
constexpr int STORE_BUFS2 = 4;                            // staging buffers: up to three stores still reading
constexpr int SMEM2_BYTES = STAGES2 * STAGE2_BYTES + STORE_BUFS2 * STORE_BYTES + 1024 + 256;
static_assert(SMEM2_BYTES <= 227 * 1024, "pair-tile shared memory");

SLSTM_DEVINL uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The shared::cluster address of the variable at shared::cta address `a` in
// the cluster's CTA `rank`.
SLSTM_DEVINL uint32_t cluster_addr(uint32_t a, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}

// Every thread of both CTAs of the cluster.
SLSTM_DEVINL void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

SLSTM_DEVINL void mbar_arrive_remote(uint32_t caddr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}

// mbar_wait with cluster-scope acquire (arrivals from the peer CTA).
SLSTM_DEVINL bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    auto try_once = [&]() {
        uint32_t ok;
        asm volatile(
            "{\n"
            " .reg .pred p;\n"
            " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
            " selp.u32 %0, 1, 0, p;\n"
            "}\n"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        return ok != 0u;
    };
    if (try_once()) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!try_once())
        if (globaltimer_ns() - t0 > limit_ns) return false;
    return true;
}

// A box of this GPU's tensor into this CTA's shared memory, its bytes
// completed on the pair's leader mbarrier at cluster address `bar`.
SLSTM_DEVINL void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t bar, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

SLSTM_DEVINL void umma2_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n"
        "}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// Arrive on the mbarrier at cluster address `bar` once every MMA this thread
// issued before has completed.
SLSTM_DEVINL void umma2_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Persistent clusters of two CTAs: cluster p takes work items p, p + the
// number of clusters, ...; item (split, m pair tile, n tile), n fastest.  In
// each CTA: warp 0 one lane loads (both CTAs), warp 1 one lane issues the MMAs
// (leader only), warps 2-5 drain this CTA's accumulator as in gemm_tc_kernel.
template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tma2,
                    const __grid_constant__ CUtensorMap tmb, const __grid_constant__ CUtensorMap tmc, TcArgs g)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES2 * A_STAGE;
    uint8_t *sE = smem + STAGES2 * STAGE2_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(sE + STORE_BUFS2 * STORE_BYTES);
    uint64_t *empty = full + STAGES2;
    uint64_t *tfull = empty + STAGES2;   // [2]
    uint64_t *tempty = tfull + 2;        // [2], the leader's
    uint64_t *fin = tempty + 2;          // the leader's: every MMA issued has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(fin + 1);
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0u;
    const int pair = (int)(blockIdx.x >> 1), n_pairs = (int)(gridDim.x >> 1);
    const int nk_part = (g.K + BK - 1) / BK;
    const int total_kb = g.a_parts * nk_part;
    const int per_split = g.m_tiles * g.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES2; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        mbar_init(fin, 1);
        mbar_init_fence();
        s_abort = 0;
    }
    if (warp == 0) {
        // the same warp of both CTAs allocates the pair's columns
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs' barriers are initialised and the columns allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---- loads (both CTAs): this CTA's A rows and its half of B ----
            int gkb = 0;
            bool stop = false;
            for (int w = pair; w < g.n_work && !stop; w += n_pairs) {
                const int z = w / per_split;
                const int r = w - z * per_split;
                const int m0 = (r / g.n_tiles) * (2 * BM) + (int)rank * BM;
                const int nb0 = (r % g.n_tiles) * BN + (int)rank * BNH;
                const int kb0 = z * g.kb_per_split;
                const int nkb = min(g.kb_per_split, total_kb - kb0);
                for (int kb = 0; kb < nkb; ++kb, ++gkb) {
                    const int s = gkb % STAGES2;
                    const uint32_t ph = (uint32_t)(gkb / STAGES2) & 1u;
                    if (*(volatile int *)&s_abort || !mbar_wait_cluster(&empty[s], ph ^ 1u, WAIT_NS)) {
                        s_abort = 1;
                        stop = true;
                        break;
                    }
                    const int vk = kb0 + kb;
                    const int part = vk / nk_part;
                    const int kk = vk - part * nk_part;
                    if (leader) mbar_expect_tx(&full[s], 2u * STAGE2_BYTES);
                    const uint32_t bar = cluster_addr(smem_u32(&full[s]), 0u);
                    const CUtensorMap *am = part ? &tma2 : &tma;
                    if (A_MN) {
#pragma unroll
                        for (int i = 0; i < BM / 64; ++i)
                            tma_load_2d_pair(sA + s * A_STAGE + i * (BK * 128), am, bar, m0 + 64 * i, kk * BK);
                    } else {
                        tma_load_2d_pair(sA + s * A_STAGE, am, bar, kk * BK, m0);
                    }
                    if (B_MN) {
#pragma unroll
                        for (int i = 0; i < BNH / 64; ++i)
                            tma_load_2d_pair(sB + s * B_HALF + i * (BK * 128), &tmb, bar, nb0 + 64 * i, kk * BK);
                    } else {
                        tma_load_2d_pair(sB + s * B_HALF, &tmb, bar, kk * BK, nb0);
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---- MMA issuer (leader): M = 256 over both CTAs' rows ----
            constexpr uint32_t idesc = idesc_bf16(2 * BM, BN, A_MN, B_MN);
            constexpr uint64_t a_step = A_MN ? (2048u >> 4) : (32u >> 4);
            constexpr uint64_t b_step = B_MN ? (2048u >> 4) : (32u >> 4);
            int gkb = 0, lt = 0;
            bool stop = false;
            for (int w = pair; w < g.n_work && !stop; w += n_pairs, ++lt) {
                const int z = w / per_split;
                const int nkb = min(g.kb_per_split, total_kb - z * g.kb_per_split);
                const int buf = lt & 1;
                if (*(volatile int *)&s_abort ||
                    !mbar_wait_cluster(&tempty[buf], ((uint32_t)(lt >> 1) & 1u) ^ 1u, WAIT_NS)) {
                    s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)(buf * BN);
                for (int kb = 0; kb < nkb; ++kb, ++gkb) {
                    const int s = gkb % STAGES2;
                    const uint32_t ph = (uint32_t)(gkb / STAGES2) & 1u;
                    if (*(volatile int *)&s_abort || !mbar_wait(&full[s], ph, WAIT_NS)) {
                        s_abort = 1;
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = A_MN ? smem_desc_mn_sw128(smem_u32(sA + s * A_STAGE), BK * 128)
                                             : smem_desc_k_sw128(smem_u32(sA + s * A_STAGE));
                    const uint64_t bd = B_MN ? smem_desc_mn_sw128(smem_u32(sB + s * B_HALF), BK * 128)
                                             : smem_desc_k_sw128(smem_u32(sB + s * B_HALF));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma2_bf16(acc, ad + a_step * k, bd + b_step * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
                    umma2_commit(cluster_addr(smem_u32(&empty[s]), 0u));
                    umma2_commit(cluster_addr(smem_u32(&empty[s]), 1u));
                }
                if (!stop) {
                    umma2_commit(cluster_addr(smem_u32(&tfull[buf]), 0u));
                    umma2_commit(cluster_addr(smem_u32(&tfull[buf]), 1u));
                }
            }
            umma2_commit(cluster_addr(smem_u32(fin), 0u));   // fires when every MMA above has completed
        }
    } else {
        // ---- epilogue: warps 2-5 of each CTA drain its 128 rows ----
        const int q = warp & 3;
        const int et = threadIdx.x - 64;   // 0..127
        const int row = q * 32 + lane;
        int lt = 0, chunk = 0;
        for (int w = pair; w < g.n_work; w += n_pairs, ++lt) {
            const int z = w / per_split;
            const int r = w - z * per_split;
            const int m0 = (r / g.n_tiles) * (2 * BM) + (int)rank * BM;
            const int n0 = (r % g.n_tiles) * BN;
            const int buf = lt & 1;
            const bool got =
                !*(volatile int *)&s_abort && mbar_wait_cluster(&tfull[buf], (uint32_t)(lt >> 1) & 1u, WAIT_NS);
            if (bar_or(1, 128, !got)) {
                s_abort = 1;
                break;
            }
            tc_fence_after();
            const uint32_t lane_addr = tmem + (uint32_t)(buf * BN) + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
            for (int c = 0; c < BN / EPI_COLS; ++c, ++chunk) {
                float v[32];
                tmem_ld32(lane_addr + (uint32_t)(c * EPI_COLS), v);
                const int col0 = n0 + c * EPI_COLS;
                epilogue_chunk<STORE_BUFS2>(g, &tmc, sE, v, lane_addr, c, chunk, m0, row, et, col0, z);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(cluster_addr(smem_u32(&tempty[buf]), 0u));
        }
        if (et == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && s_abort) {
        atomicOr(g.error, 1u);
        // copies and MMAs issued before the abort land within microseconds:
        // give them time before the pair's memory is released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000ull) __nanosleep(1000);
    }
    if (threadIdx.x == 0 && leader) (void)mbar_wait(fin, 0u, WAIT_NS);
    __syncthreads();
    cluster_sync_all();   // the leader's MMAs are done with both CTAs' memory
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// 2-D bf16 tensor of `rows` rows of `cols` contiguous elements (row stride
// ld elements), box of 64 contiguous elements x box_rows rows, 128-byte
// swizzle.  K-major operands: cols = K, rows = M or N.  MN-major operands:
// cols = M or N, rows = K.
bool make_map(CUtensorMap *map, const void *base, int rows, int cols, int ld, int box_rows)
{
    auto fn = tensor_map_encoder();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// fp32 C viewed as (N, M, splits), box 32 x 128 x 1, 128-byte swizzle: the
// epilogue's store boxes.  Rows past M and columns past N are not written.
bool make_c_map(CUtensorMap *map, float *C, int M, int N, int splits)
{
    auto fn = tensor_map_encoder();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)M, (cuuint64_t)splits};
    cuuint64_t strides[2] = {(cuuint64_t)N * 4, (cuuint64_t)M * N * 4};
    cuuint32_t box[3] = {(cuuint32_t)STORE_COLS, (cuuint32_t)BM, 1u};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, C, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int sm_count_tc()
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

// Tile shape in use (SLSTM_GEMM_TILES_*): SM-pair tiles (256 x 256 per
// cluster of two CTAs), single-SM tiles (128 x 256 per CTA), or pairs for
// plain-store products whose work items span at least PAIR_MIN_KB k-blocks.
// Measured on B200: a pair hands its two accumulators back to the MMA issuer
// only when both CTAs have drained them, so products whose epilogue's
// output stream sets the pace run faster on single SMs (the input
// projection, K = 1024: 0.474 against 0.503 ms; the trunk layer's forward,
// whose down projection reads and writes the fp32 residual: 6.21 against
// 6.35 ms with that GEMM on pairs), and those with long K on pairs (the
// gradient GEMMs: the cell's backward 2.81 -> 2.67 ms, the trunk layer's
// 12.20 -> 11.75 ms).
int g_tc_mode = SLSTM_GEMM_TILES_AUTO;
constexpr int PAIR_MIN_KB = 64;

// Clusters of two gemm_tc2_kernel CTAs that can be resident at once (0: none).
template <bool A_MN, bool B_MN>
int pair_clusters()
{
    static int n = -1;
    if (n < 0) {
        n = 0;
        auto kern = gemm_tc2_kernel<A_MN, B_MN>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2_BYTES) != cudaSuccess) {
            (void)cudaGetLastError();
            return n;
        }
        cudaLaunchConfig_t cfg;
        memset(&cfg, 0, sizeof(cfg));
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * 64, 1, 1);
        cfg.blockDim = dim3(THREADS, 1, 1);
        cfg.dynamicSmemBytes = SMEM2_BYTES;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int c = 0;
        if (cudaOccupancyMaxActiveClusters(&c, kern, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            c = 0;
        }
        n = c;
    }
    return n;
}

template <bool A_MN, bool B_MN>
cudaError_t launch_tc2(const CUtensorMap &ta, const CUtensorMap &ta2, const CUtensorMap &tb, const CUtensorMap &tc,
                       const TcArgs &g, int clusters, cudaStream_t st)
{
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * min(g.n_work, clusters), 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM2_BYTES;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<A_MN, B_MN>, ta, ta2, tb, tc, g);
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <bool A_MN, bool B_MN>
cudaError_t launch_tc(const CUtensorMap &ta, const CUtensorMap &ta2, const CUtensorMap &tb, const CUtensorMap &tc,
                      const TcArgs &g, cudaStream_t st)
{
    static bool attr_set = false;
    if (!attr_set) {
        const cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<A_MN, B_MN>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int grid = min(g.n_work, sm_count_tc());
    gemm_tc_kernel<A_MN, B_MN><<<grid, THREADS, SMEM_BYTES, st>>>(ta, ta2, tb, tc, g);
    return cudaGetLastError();
}

// B's tensor map for the tile shape, the tile counts, and the launch: SM-pair
// tiles when selected and clusters of two can run, else single-SM tiles.
template <bool A_MN, bool B_MN>
cudaError_t run_tc(const CUtensorMap &ta, const CUtensorMap &ta2, const void *Bm, int ldb, const CUtensorMap &tc,
                   TcArgs g, int splits, cudaStream_t st)
{
    g.n_tiles = (g.N + BN - 1) / BN;
    CUtensorMap tb;
    const bool pair = g_tc_mode == SLSTM_GEMM_TILES_PAIR ||
                      (g_tc_mode == SLSTM_GEMM_TILES_AUTO && g.epi == GEMM_EPI_STORE && g.kb_per_split >= PAIR_MIN_KB);
    const int clusters = pair ? pair_clusters<A_MN, B_MN>() : 0;
    const int rows = clusters > 0 ? 2 * BM : BM;
    // K-major B: boxes of this CTA's rows of the tile (half of BN on SM pairs)
    const bool ok = B_MN ? make_map(&tb, Bm, g.K, g.N, ldb, BK) : make_map(&tb, Bm, g.N, g.K, ldb, rows == BM ? BN : BNH);
    if (!ok) return cudaErrorInvalidValue;
    g.m_tiles = (g.M + rows - 1) / rows;
    g.n_work = g.m_tiles * g.n_tiles * splits;
    if (clusters > 0) return launch_tc2<A_MN, B_MN>(ta, ta2, tb, tc, g, clusters, st);
    return launch_tc<A_MN, B_MN>(ta, ta2, tb, tc, g, st);
}

}  // namespace

int gemm_tc_set_tiles(int tiles)
{
    if (tiles != SLSTM_GEMM_TILES_AUTO && tiles != SLSTM_GEMM_TILES_PAIR && tiles != SLSTM_GEMM_TILES_SINGLE) return -1;
    const int prev = g_tc_mode;
    g_tc_mode = tiles;
    return prev;
}

void gemm_tc_waves(int *tile_rows, int *units)
{
    // split-K products have long K: AUTO takes pairs for them
    const int clusters = g_tc_mode != SLSTM_GEMM_TILES_SINGLE ? pair_clusters<false, false>() : 0;
    *tile_rows = clusters > 0 ? 2 * BM : BM;
    *units = clusters > 0 ? clusters : sm_count_tc();
}

// C = (A0 [+ A1]) B^T (+ bias) with optional split-K into `splits` fp32
// slices C + z * M * N (the caller sums them).  A0, A1: [M][K] (a_mn = 0) or
// [K][M] (a_mn = 1) bf16 with row stride lda; B: [N][K] (b_mn = 0) or [K][N]
// (b_mn = 1) with row stride ldb.
cudaError_t gemm_tc_bf16_ex(const void *A0, const void *A1, int lda, bool a_mn, const void *Bm, int ldb, bool b_mn,
                            const float *bias, float *C, int M, int N, int K, int splits, unsigned *error,
                            cudaStream_t st)
{
    CUtensorMap ta, ta2;
    const bool ok_a = a_mn ? make_map(&ta, A0, K, M, lda, BK) : make_map(&ta, A0, M, K, lda, BM);
    if (!ok_a) return cudaErrorInvalidValue;
    if (A1 != nullptr) {
        const bool ok = a_mn ? make_map(&ta2, A1, K, M, lda, BK) : make_map(&ta2, A1, M, K, lda, BM);
        if (!ok) return cudaErrorInvalidValue;
    } else {
        ta2 = ta;
    }
    TcArgs g;
    memset(&g, 0, sizeof(g));   // epi = GEMM_EPI_STORE
    g.C = C;
    g.bias = bias;
    g.M = M;
    g.N = N;
    g.K = K;
    g.a_parts = A1 ? 2 : 1;
    const int total = g.a_parts * ((K + BK - 1) / BK);
    if (splits < 1) splits = 1;
    if (splits > total) splits = total;
    g.kb_per_split = (total + splits - 1) / splits;
    splits = (total + g.kb_per_split - 1) / g.kb_per_split;   // no empty split
    g.c_split = (long long)M * N;
    g.error = error;
    CUtensorMap tc;
    memset(&tc, 0, sizeof(tc));
    g.tma_out = ((N & 3) == 0 && (reinterpret_cast<uintptr_t>(C) & 15) == 0 && make_c_map(&tc, C, M, N, splits)) ? 1 : 0;
    if (a_mn)
        return b_mn ? run_tc<true, true>(ta, ta2, Bm, ldb, tc, g, splits, st)
                    : run_tc<true, false>(ta, ta2, Bm, ldb, tc, g, splits, st);
    return b_mn ? run_tc<false, true>(ta, ta2, Bm, ldb, tc, g, splits, st)
                : run_tc<false, false>(ta, ta2, Bm, ldb, tc, g, splits, st);
}

cudaError_t gemm_tc_bf16_epi(const void *A, const void *Bm, float *C, __nv_bfloat16 *Cb, const float *res, int M,
                             int N, int K, int epi, unsigned *error, cudaStream_t st)
{
    if (epi == GEMM_EPI_SWIGLU ? (Cb == nullptr || N % 64 != 0) : (C == nullptr || epi != GEMM_EPI_RESIDUAL ||
                                                                    res == nullptr))
        return cudaErrorInvalidValue;
    CUtensorMap ta;
    if (!make_map(&ta, A, M, K, K, BM)) return cudaErrorInvalidValue;
    TcArgs g;
    memset(&g, 0, sizeof(g));
    g.C = C;
    g.bias = nullptr;
    g.M = M;
    g.N = N;
    g.K = K;
    g.a_parts = 1;
    g.kb_per_split = (K + BK - 1) / BK;   // no split-K: the epilogue sees whole sums
    g.c_split = (long long)M * N;
    g.error = error;
    g.epi = epi;
    g.Cb = Cb;
    g.res = res;
    CUtensorMap tc;
    memset(&tc, 0, sizeof(tc));
    g.tma_out = (epi == GEMM_EPI_RESIDUAL && (N & 3) == 0 && (reinterpret_cast<uintptr_t>(C) & 15) == 0 &&
                 make_c_map(&tc, C, M, N, 1))
                    ? 1
                    : 0;
    return run_tc<false, false>(ta, ta, Bm, K, tc, g, 1, st);
}

int gemm_tc_splits(int M, int N, int K, int a_parts, int want)
{
    (void)M;
    (void)N;
    const int total = a_parts * ((K + BK - 1) / BK);
    if (want < 1) want = 1;
    if (want > total) want = total;
    const int per = (total + want - 1) / want;
    return (total + per - 1) / per;
}

cudaError_t gemm_tc_bf16(const void *A, const void *Bm, const float *bias, float *C, int M, int N, int K,
                         unsigned *error, cudaStream_t st)
{
    return gemm_tc_bf16_ex(A, nullptr, K, false, Bm, K, false, bias, C, M, N, K, 1, error, st);
}

}  // namespace slstm
