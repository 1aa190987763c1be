// k_down.cu -- the routed experts' bf16 down projection with the
// routing-weighted combine, for prefill-sized batches, on the fifth-generation
// tensor cores.  The experts' down projections stay bf16
// ("gemma4-26b-a4b-dflash-i8" README, table "Weights").
//
// For every pair (t, j) routed to expert e:
//     out[t][n] += w[t, j] * sum_i a(t, j)[i] * W_e[n][i],
// where a = gelu(gate) * up is held as three bf16 planes whose sum is its fp32
// value; the planes enter as a K three times as long (3 I) against the same
// weight columns, so the fp32 sums carry a's full precision.
//
// A tile is 128 weight rows of one expert (the MMA's M, tensor-memory lanes)
// by up to 160 of its pairs (the MMA's N: the tile's row count rounded up to
// 16, so a short tile costs only its own rows).  A weight step is 64 of the
// I: its weight box [128 rows][128 B] lands in a 3-slot ring and serves the
// three planes, whose activation boxes land in an 8-slot ring; each plane
// takes four MMAs (kind::f16, bf16 x bf16, K = 16, both operands from shared
// memory) into the tile's fp32 accumulator.  No scale changes along K, so the
// accumulator holds the whole sum and is read once per tile; two of them let
// the epilogue of one tile run under the MMAs of the next.
//
// The kernel is bound by the operand stream from L2 into shared memory, not
// by the tensor pipe, so it moves as few and as large boxes as it can: each
// weight box once for its three planes, and a tile's activation rows in one
// 128-row box plus 32-row boxes for what is left.  The 160-row cap (an
// expert's pairs at 2048 tokens x top-8 over 128 experts number about 128)
// keeps the activation slots small enough for eight of them.
//
// Warp roles: lane 0 of warp 0 issues the TMA loads, lane 0 of warp 1 the
// MMAs, warp 2 owns the tensor-memory allocation.  Warps 4..11 are the
// epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 (weight rows,
// i.e. output columns n) and one half of the tile's pairs, scales each pair's
// column by its routing weight and adds it into its token's output row; the
// 32 lanes add 32 consecutive floats, one coalesced reduction per pair and
// warp.  Reductions from different tiles meet in the same rows (a token's
// top-k pairs sit in different experts), so out must be zeroed beforehand
// and the fp32 sums' order varies from run to run.
//
// All waits are bounded; on a timeout the CTA sets QL_DEVERR_TIMEOUT and
// winds down without leaving tensor memory allocated, MMAs running or copies
// in flight.
#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

constexpr int DM = 128;                  // weight rows per tile (MMA M)
constexpr int DN = kDownTileRows;        // pairs per tile at most (MMA N <= 256)
constexpr int ACC_COLS = 256;            // tensor-memory columns between the two accumulators
constexpr int XBOX = 32;                 // activation rows per small TMA box
constexpr int XBIG = 128;                // activation rows per large TMA box
constexpr int A_BYTES = DM * 128;        // weight box, 16 KB
constexpr int B_BYTES = DN * 128;        // activation boxes, up to 20 KB
constexpr int WS = 3;                    // weight ring slots
constexpr int XS = 8;                    // activation ring slots
constexpr int NACC = 2;                  // accumulators [128 x DN]
constexpr uint32_t kTmemCols = 512;
constexpr int kEpiWarp0 = 4, kEpiWarps = 8;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int HALF = DN / 2;             // pairs per epilogue warp
constexpr int CW = 16;                   // columns per tensor-memory read
static_assert(NACC * ACC_COLS <= (int)kTmemCols && DN % 32 == 0 && DN <= ACC_COLS, "tile width");
static_assert(DN >= XBIG && (DN - XBIG) % XBOX == 0, "a large box and small ones cover any tile");
static_assert(B_BYTES % 1024 == 0 && A_BYTES % 1024 == 0 && (XBOX * 128) % 1024 == 0,
              "operand boxes stay 1024-byte aligned for the 128-byte swizzle");
constexpr int NBAT = (HALF + 31) / 32;  // 32-pair batches per epilogue warp
static_assert(HALF % CW == 0, "whole tensor-memory reads per warp");

// Shared memory (from a 1024-aligned base): [weight ring][activation ring][mbarriers][tmem address]
constexpr int X_OFF = WS * A_BYTES;
constexpr int BAR_OFF = X_OFF + XS * B_BYTES;
constexpr int B_WFULL = 0, B_WEMPTY = WS, B_XFULL = 2 * WS, B_XEMPTY = B_XFULL + XS, B_ACCF = B_XEMPTY + XS,
              B_ACCE = B_ACCF + NACC, B_DRAIN = B_ACCE + NACC, NBARS = B_DRAIN + 1;
constexpr int MISC_OFF = (BAR_OFF + 8 * NBARS + 15) / 16 * 16;
constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
    // K-major, 128-byte swizzle: 8-row atoms 1024 bytes apart (SBO), version 1.
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// kind::f16: D f32 (bits 4-5 = 1), A bf16 (bits 7-9 = 1), B bf16 (bits 10-12 = 1), both K-major,
// N >> 3 at bits 17-22, M >> 4 at bits 24-28.
__device__ __forceinline__ uint32_t idesc_bf16(int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(DM >> 4) << 24);
}
// D (+)= A * B^T, A and B from shared memory; acc_in = 0 overwrites D.
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc_in) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc_in));
}
__device__ __forceinline__ void commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t addr, float v[CW]) {
    uint32_t r[CW];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        "tcgen05.wait::ld.sync.aligned;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(addr)
        : "memory");
#pragma unroll
    for (int i = 0; i < CW; ++i) v[i] = __uint_as_float(r[i]);
}

struct DownArgs {
    CUtensorMap tmW;       // weights [E * N rows][2 I bytes], box [128 rows][128 B]
    CUtensorMap tmX;       // activation planes [rows_total][6 I bytes], box [32 rows][128 B]
    CUtensorMap tmXb;      // the same, box [128 rows][128 B]
    const MoeTile* tiles;  // the permute's tiles (at most DN rows each) and their count
    const int* n_tiles;
    const int32_t* perm;   // permuted row -> pair t * topk + j
    const float* wts;      // routing weight of each pair
    float* out;            // [T][N], zeroed before
    unsigned* err;
    int N, GW, topk;       // GW = I / 64 weight steps per tile
};

__global__ void __launch_bounds__(kThreads, 1) k_down_grouped(const __grid_constant__ DownArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const gb = smem_raw + (base - raw);
    auto bar = [&](int i) { return base + BAR_OFF + 8u * (uint32_t)i; };
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gb + MISC_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tiles = *a.n_tiles;
    const int GW = a.GW;

    if (threadIdx.x == 0) {
        for (int s = 0; s < WS; ++s) {
            mbar_init(bar(B_WFULL + s), 1);   // expect_tx
            mbar_init(bar(B_WEMPTY + s), 1);  // the MMA commit after the weight step's last plane
        }
        for (int s = 0; s < XS; ++s) {
            mbar_init(bar(B_XFULL + s), 1);   // expect_tx
            mbar_init(bar(B_XEMPTY + s), 1);  // the plane's MMA commit
        }
        for (int b = 0; b < NACC; ++b) {
            mbar_init(bar(B_ACCF + b), 1);          // the tile's last commit
            mbar_init(bar(B_ACCE + b), kEpiWarps);  // one arrive per epilogue warp
        }
        mbar_init(bar(B_DRAIN), 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long lim = wait_limit(a.err);
    bool dead = false;

    if (warp == 0 && lane == 0) {  // ---- producer ----
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmW) : "memory");
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmX) : "memory");
        asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmXb) : "memory");
        int wstep = 0, xstep = 0;
        for (int t = blockIdx.x; t < tiles && !dead; t += gridDim.x) {
            const MoeTile ti = a.tiles[t];
            // The tile's rows come in one 128-row box (from 96 rows on: large boxes stream faster than
            // small ones, worth the rows fetched past the tile) and 32-row boxes for the rest.
            const int big = ti.rows >= 96 ? 1 : 0;
            const int nb = (max(ti.rows - big * XBIG, 0) + XBOX - 1) / XBOX;
            const unsigned xbytes = (big * XBIG + nb * XBOX) * 128;
            const int wrow = ti.expert * a.N + ti.wb * DM;
            for (int w = 0; w < GW && !dead; ++w, ++wstep) {
                const int ws = wstep % WS;
                if (!mbar_wait(bar(B_WEMPTY + ws), ((wstep / WS) & 1) ^ 1, lim)) {
                    dead = true;
                    break;
                }
                mbar_expect_tx(bar(B_WFULL + ws), A_BYTES);
                tma_load_2d(base + ws * A_BYTES, &a.tmW, w * 128, wrow, bar(B_WFULL + ws));
                for (int pl = 0; pl < 3; ++pl, ++xstep) {  // plane pl: columns pl * I + 64 w
                    const int xs = xstep % XS;
                    if (!mbar_wait(bar(B_XEMPTY + xs), ((xstep / XS) & 1) ^ 1, lim)) {
                        dead = true;
                        break;
                    }
                    const uint32_t fb = bar(B_XFULL + xs), dst = base + X_OFF + xs * B_BYTES;
                    const int x = (pl * GW + w) * 128;
                    mbar_expect_tx(fb, xbytes);
                    if (big) tma_load_2d(dst, &a.tmXb, x, ti.row0, fb);
                    for (int b = 0; b < nb; ++b)
                        tma_load_2d(dst + (big * XBIG + b * XBOX) * 128, &a.tmX, x, ti.row0 + big * XBIG + b * XBOX,
                                    fb);
                }
            }
        }
        // Copies still in flight must land before the CTA's shared memory is released.
        for (int j = wstep > WS ? wstep - WS : 0; j < wstep; ++j)
            if (!mbar_wait(bar(B_WFULL + j % WS), (j / WS) & 1)) break;
        for (int j = xstep > XS ? xstep - XS : 0; j < xstep; ++j)
            if (!mbar_wait(bar(B_XFULL + j % XS), (j / XS) & 1)) break;
    } else if (warp == 1 && lane == 0) {  // ---- MMA issuer ----
        int wstep = 0, xstep = 0, tl = 0;
        for (int t = blockIdx.x; t < tiles && !dead; t += gridDim.x, ++tl) {
            const MoeTile ti = a.tiles[t];
            const int b = tl % NACC;
            if (!mbar_wait(bar(B_ACCE + b), ((tl / NACC) & 1) ^ 1, lim)) {  // the epilogue is done with it
                dead = true;
                break;
            }
            fence_after();
            const uint32_t idesc = idesc_bf16((ti.rows + 15) & ~15), d = tmem + b * ACC_COLS;
            for (int w = 0; w < GW && !dead; ++w, ++wstep) {
                const int ws = wstep % WS;
                if (!mbar_wait(bar(B_WFULL + ws), (wstep / WS) & 1, lim)) {
                    dead = true;
                    break;
                }
                const uint64_t ad = desc_sw128(base + ws * A_BYTES);
                for (int pl = 0; pl < 3; ++pl, ++xstep) {
                    const int xs = xstep % XS;
                    if (!mbar_wait(bar(B_XFULL + xs), (xstep / XS) & 1, lim)) {
                        dead = true;
                        break;
                    }
                    fence_after();
                    const uint64_t bd = desc_sw128(base + X_OFF + xs * B_BYTES);
#pragma unroll
                    for (int j = 0; j < 4; ++j)  // K = 16 bf16 = 32 bytes: +2 in the descriptor's address field
                        mma_ss(d, ad + 2 * j, bd + 2 * j, idesc, (w | pl | j) ? 1u : 0u);
                    commit(bar(B_XEMPTY + xs));  // the activation slot may be refilled once these are done
                }
                commit(bar(B_WEMPTY + ws));  // and the weight slot after its three planes
            }
            if (dead) break;
            commit(bar(B_ACCF + b));  // the tile's sums are complete
        }
        // Every MMA issued must finish before tensor memory is freed.
        commit(bar(B_DRAIN));
        mbar_wait(bar(B_DRAIN), 0);
    } else if (warp >= kEpiWarp0) {  // ---- epilogue ----
        const int q = warp & 3, h = (warp - kEpiWarp0) >> 2;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        int tl = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tl) {
            const MoeTile ti = a.tiles[t];
            const int b = tl % NACC;
            const int n = ti.wb * DM + 32 * q + lane;  // this thread's output column
            const int c0 = h * HALF, c1 = min(ti.rows, c0 + HALF);
            // Before the accumulator is ready: lane l fetches pairs c0 + 32 i + l of this warp's
            // columns -- its token's output row and its routing weight.
            int tok[NBAT];
            float w[NBAT];
#pragma unroll
            for (int i = 0; i < NBAT; ++i) {
                const int c = c0 + 32 * i + lane;
                tok[i] = c < c1 ? __ldg(a.perm + ti.row0 + c) : 0;
            }
#pragma unroll
            for (int i = 0; i < NBAT; ++i) {
                const int c = c0 + 32 * i + lane;
                w[i] = c < c1 ? __ldg(a.wts + tok[i]) : 0.0f;
                tok[i] /= a.topk;
            }
            if (!__all_sync(kFull, mbar_wait(bar(B_ACCF + b), (tl / NACC) & 1, lim))) {  // together
                dead = true;
                break;
            }
            fence_after();
#pragma unroll
            for (int k = 0; k < HALF; k += CW) {
                if (c0 + k >= c1) break;  // warp-uniform
                float v[CW];
                tmem_ld16(tmem + lane_base + b * ACC_COLS + c0 + k, v);
#pragma unroll
                for (int i = 0; i < CW; ++i) {
                    const int src = (k + i) & 31;  // the lane holding pair c0 + k + i
                    const int tt = __shfl_sync(kFull, tok[(k + i) / 32], src);
                    const float wi = __shfl_sync(kFull, w[(k + i) / 32], src);
                    if (c0 + k + i < c1 && n < a.N) atomicAdd(a.out + (long long)tt * a.N + n, wi * v[i]);
                }
            }
            fence_before();
            __syncwarp();
            if (lane == 0) arrive(bar(B_ACCE + b));
        }
    }
    if (dead) atomicOr(a.err, (unsigned)QL_DEVERR_TIMEOUT);

    fence_before();
    __syncthreads();
    if (warp == 2) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
    }
}

}  // namespace

cudaError_t launch_down_grouped(const __nv_bfloat16* act, const uint16_t* wd, int E, int N, int I, int rows_total,
                                const MoeTile* tiles, const int* n_tiles, int max_tiles, const int32_t* perm,
                                int topk, const float* wts, float* out, cudaStream_t s) {
    if (I % 64 || max_tiles < 1) return cudaErrorInvalidValue;
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    if ((size_t)SMEM_BYTES > di.smem_optin) return cudaErrorInvalidValue;
    DownArgs a{};
    if ((e = make_tmap_2d(wd, (long long)E * N, 2LL * I, 2LL * I, 128, DM, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmW)) !=
        cudaSuccess)
        return e;
    if ((e = make_tmap_2d(act, rows_total, 6LL * I, 6LL * I, 128, XBOX, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmX)) !=
        cudaSuccess)
        return e;
    if ((e = make_tmap_2d(act, rows_total, 6LL * I, 6LL * I, 128, XBIG, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmXb)) !=
        cudaSuccess)
        return e;
    a.tiles = tiles;
    a.n_tiles = n_tiles;
    a.perm = perm;
    a.wts = wts;
    a.out = out;
    a.err = di.err_word;
    a.N = N;
    a.GW = I / 64;
    a.topk = topk;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(k_down_grouped, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[dev] = true;
    }
    const int grid = max_tiles < di.sm_count ? max_tiles : di.sm_count;
    k_down_grouped<<<grid, kThreads, SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

}  // namespace ql
