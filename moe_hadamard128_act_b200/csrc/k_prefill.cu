// k_prefill.cu -- the prefill-shaped W8A8 GEMM (M >= 17 tokens) on the
// fifth-generation tensor cores: int8 activations (one fp32 scale per token
// per 128 values) times int8 weights (one bf16 scale per row per 128), each
// 128-wide group's integer dot product exact, both scales applied in fp32
// ("keptn/gemma4-12b-i8g", table "Format").
//
// Persistent CTAs, one per SM, walk 128 (tokens) x 128 (weight rows) output
// tiles, weight-tile-major so the token blocks that share a weight tile run at
// the same time and read it from L2.  Warp roles:
//  * warp 0 (one lane): TMA producer.  Per 128-K group it loads the
//    activation tile [128][128 B] and the weight tile [128][128 B] with
//    128-byte swizzle into a 6-slot ring (32 KB per slot).
//  * warp 1 (one lane): MMA issuer.  Four tcgen05.mma kind::i8 (K = 32 each)
//    per group into one of four 128-column int32 accumulators in tensor
//    memory, then tcgen05.commit frees the ring slot and signals the epilogue.
//  * warps 2..9: epilogue, two warpgroups of 64 columns each; thread i of a
//    warp owns tile row 32 * (warp % 4) + i (its tensor-memory lane).  Per
//    group it reads the accumulator (tcgen05.ld 32x32b), adds
//    s_x[m, g] * s_w[n, g] * acc into fp32 running sums held in registers, and
//    hands the accumulator back.
// The per-group promotion is the cost centre: both scales change every 128 K,
// so every output element is touched once per group.  To keep it to two fp32
// FMAs per element, the epilogue re-initialises each accumulator to the bit
// pattern of 1.5 * 2^23 instead of zero: the MMAs add the group's integer sum
// to it (|sum| <= 128 * 127^2 < 2^22), so the accumulator read as an fp32 is
// exactly 12582912 + sum; with the row's activation scale cut to 22
// significant bits, s_x * 12582912 is exact and one FMA yields s_x * sum
// rounded once, a second adds s_w * that to the running sum.
//
// All waits are bounded (200 ms); a role that gives up sets
// QL_DEVERR_TIMEOUT and the CTA winds down without leaving tensor memory
// allocated.
#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

constexpr int PM = 128;                   // tile rows (tokens)
constexpr int PN = 128;                   // tile columns (weight rows)
constexpr int PKB = 128;                  // K bytes per group
constexpr int PSTAGES = 6;
constexpr int A_BYTES = PM * PKB;         // 16 KB
constexpr int B_BYTES = PN * PKB;         // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kEpiWarps = 8;
constexpr int kPThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kMagic = 0x4B400000u;  // 12582912.0f
constexpr int NBUF = 4;                   // int32 accumulators in tensor memory, 128 columns each
constexpr uint32_t kTmemCols = 512;
constexpr int WGC = PN / 2;               // columns per epilogue warpgroup

// Shared memory: [ring][barriers: full, empty (per slot), acc_full, acc_empty (per accumulator)]
//                [tmem address, abort flag][weight scales: 2 warpgroups x 2 slots x 64 fp32][y staging]
constexpr int BAR_OFF = PSTAGES * STAGE_BYTES;
constexpr int MISC_OFF = (BAR_OFF + 8 * (2 * PSTAGES + 2 * NBUF + 1) + 15) / 16 * 16;  // + an MMA-drain barrier
constexpr int SW_OFF = MISC_OFF + 16;
// y staging: per warpgroup [128 rows][16 columns] fp32 with a row stride of 17
// (scalar stores by row-owning threads and row reads by lanes are conflict-free)
constexpr int YST_STRIDE = 17;
constexpr int YST_OFF = SW_OFF + 2 * 2 * WGC * 4;
constexpr int SMEM_BYTES = YST_OFF + 2 * 128 * YST_STRIDE * 4 + 1024;
static_assert(STAGE_BYTES % 1024 == 0, "ring slots must stay 1024-byte aligned for the 128-byte swizzle");
static_assert(SW_OFF % 16 == 0 && YST_OFF % 16 == 0, "scale and staging buffers are read with 16-byte loads");

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    // K-major, 128-byte swizzle: 8-row atoms 1024 bytes apart (SBO), version 1.
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// kind::i8, D s32, A s8, B s8, both K-major, N = 128, M = 128.
constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(PN >> 3) << 17) |
                              ((uint32_t)(PM >> 4) << 24);

__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

#define QL_TMEM_LD16(addr, v)                                                                                   \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}," \
                 " [%16];\n"                                                                                    \
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),         \
                   "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),     \
                   "=r"(v[14]), "=r"(v[15])                                                                    \
                 : "r"(addr))

__device__ __forceinline__ void tmem_fill_magic32(uint32_t addr) {
    const uint32_t m = kMagic;
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
        "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};\n" ::"r"(addr),
        "r"(m)
        : "memory");
}

struct PrefillArgs {
    CUtensorMap tmA;     // int8 activations [M][K], box [128 rows][128 B]
    CUtensorMap tmB;     // int8 weights [N][K], box [128 rows][128 B]
    const float* sx;     // [M][G] activation scales
    const uint16_t* sw;  // [N][G] bf16 weight scales
    float* y;            // [M][ldy]
    int32_t* acc;        // group sums [M][N][G] (check path only)
    unsigned* err;
    int M, N, G;
    long long ldy;
};

// 168 registers: registers are allocated per SM sub-partition, and the three
// warps of this 10-warp CTA that share one sub-partition must fit in its 16K.
template <bool ACC>
__global__ void __maxnreg__(168) k_prefill_w8a8(const __grid_constant__ PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const gb = smem_raw + (base - raw);
    const uint32_t bars = base + BAR_OFF;
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gb + MISC_OFF);
    volatile uint32_t* const abort_flag = tmem_slot + 1;
    float* const sw_s = reinterpret_cast<float*>(gb + SW_OFF);
    float* const yst_s = reinterpret_cast<float*>(gb + YST_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int MB = (a.M + PM - 1) / PM, NB = (a.N + PN - 1) / PN;
    const int tiles = MB * NB;
    const int my_tiles = blockIdx.x < tiles ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int G = a.G;
    const int total = my_tiles * G;  // (tile, group) steps of this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < PSTAGES; ++s) {
            mbar_init(bars + 8 * s, 1);              // full: producer's expect_tx
            mbar_init(bars + 8 * (PSTAGES + s), 1);  // empty: MMA commit
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(bars + 8 * (2 * PSTAGES + b), 1);                 // acc full: MMA commit
            mbar_init(bars + 8 * (2 * PSTAGES + NBUF + b), kEpiWarps);  // acc empty: one arrive per epilogue warp
        }
        mbar_init(bars + 8 * (2 * PSTAGES + 2 * NBUF), 1);  // MMA drain before tensor memory is freed
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {  // ---- TMA producer ----
            asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmA) : "memory");
            asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmB) : "memory");
            int tl = 0, g = 0, issued = 0;
            for (int k = 0; k < total; ++k) {
                const int s = k % PSTAGES;
                const unsigned ph = (unsigned)(k / PSTAGES) & 1u;
                if (*abort_flag || !mbar_wait(bars + 8 * (PSTAGES + s), ph ^ 1u)) {
                    *abort_flag = 1;
                    break;
                }
                ++issued;
                const int t = blockIdx.x + tl * gridDim.x;
                const int mb = t % MB, nb = t / MB;
                const uint32_t st = base + s * STAGE_BYTES;
                mbar_expect_tx(bars + 8 * s, STAGE_BYTES);
                tma_load_2d(st, &a.tmA, g * PKB, mb * PM, bars + 8 * s);
                tma_load_2d(st + A_BYTES, &a.tmB, g * PKB, nb * PN, bars + 8 * s);
                if (++g == G) {
                    g = 0;
                    ++tl;
                }
            }
            // Copies still in flight must land before the CTA's shared memory is released.
            for (int k = issued > PSTAGES ? issued - PSTAGES : 0; k < issued; ++k)
                if (!mbar_wait(bars + 8 * (k % PSTAGES), (unsigned)(k / PSTAGES) & 1u)) break;
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ---- MMA issuer ----
            for (int k = 0; k < total; ++k) {
                const int s = k % PSTAGES;
                const unsigned ph = (unsigned)(k / PSTAGES) & 1u;
                const int buf = k % NBUF;
                const unsigned aph = (unsigned)(k / NBUF) & 1u;
                if (*abort_flag || !mbar_wait(bars + 8 * s, ph) ||
                    !mbar_wait(bars + 8 * (2 * PSTAGES + NBUF + buf), aph)) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t st = base + s * STAGE_BYTES;
#pragma unroll
                for (int kk = 0; kk < PKB / 32; ++kk)
                    mma_i8(tmem + buf * PN, smem_desc_sw128(st + 32 * kk), smem_desc_sw128(st + A_BYTES + 32 * kk),
                           kIdescI8, 1u);
                mma_commit(bars + 8 * (PSTAGES + s));          // ring slot free once these MMAs are done
                mma_commit(bars + 8 * (2 * PSTAGES + buf));    // accumulator ready for the epilogue
            }
            // Every MMA issued must finish before tensor memory is freed.
            mma_commit(bars + 8 * (2 * PSTAGES + 2 * NBUF));
            mbar_wait(bars + 8 * (2 * PSTAGES + 2 * NBUF), 0);
        }
    } else {  // ---- epilogue ----
        const int ew = warp - 2;
        const int wg = ew >> 2;                // column half of the tile
        const int sub = warp & 3;              // tensor-memory lane quarter
        const int row = sub * 32 + lane;       // tile row of this thread
        const int ti = (ew & 3) * 32 + lane;   // index within the warpgroup (< WGC: the column whose scale it fetches)
        const uint32_t tlane = (uint32_t)(sub * 32) << 16;
        const uint32_t named = 1 + wg;
        auto wg_sync = [&]() { asm volatile("bar.sync %0, 128;\n" ::"r"(named) : "memory"); };

        // Every accumulator starts at the magic value.
#pragma unroll
        for (int b = 0; b < NBUF; ++b)
#pragma unroll
            for (int j = 0; j < WGC / 32; ++j) tmem_fill_magic32(tmem + tlane + b * PN + wg * WGC + 32 * j);
        asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int b = 0; b < NBUF; ++b) mbar_arrive(bars + 8 * (2 * PSTAGES + NBUF + b));

        // Scales of the steps (tile, group) for this thread, fetched three steps
        // ahead: its row's activation scale and its column's weight scale bits.
        int f_tl = 0, f_g = 0;  // position of the next step to fetch
        auto fetch_next = [&](float& sxv, uint32_t& swv) {
            sxv = 0.0f;
            swv = 0u;
            if (f_tl < my_tiles) {
                const int t = blockIdx.x + f_tl * gridDim.x;
                const int mb = t % MB;
                const int m = mb * PM + row, n = (t - mb) / MB * PN + wg * WGC + ti;
                if (m < a.M && a.sx) sxv = __ldg(a.sx + (long long)m * G + f_g);
                if (ti < WGC && n < a.N && a.sw) swv = __ldg(a.sw + (long long)n * G + f_g);
            }
            if (++f_g == G) {
                f_g = 0;
                ++f_tl;
            }
        };
        float sx_cur, sx_n1, sx_n2;
        uint32_t sw0, sw_n1, sw_n2;
        fetch_next(sx_cur, sw0);
        fetch_next(sx_n1, sw_n1);
        fetch_next(sx_n2, sw_n2);
        if (ti < WGC) sw_s[(wg * 2 + 0) * WGC + ti] = __uint_as_float(sw0 << 16);
        wg_sync();

        float yr[WGC];
#pragma unroll
        for (int i = 0; i < WGC; ++i) yr[i] = 0.0f;
        bool dead = false;
        int tl = 0, g = 0;
        for (int k = 0; k < total; ++k) {
            const int buf = k % NBUF;
            const unsigned aph = (unsigned)(k / NBUF) & 1u;
            if (!dead && (*abort_flag || !mbar_wait(bars + 8 * (2 * PSTAGES + buf), aph))) {
                dead = true;
                *abort_flag = 1;
            }
            const int t = blockIdx.x + tl * gridDim.x;
            const int m0 = (t % MB) * PM, n0 = (t / MB) * PN + wg * WGC;
            if (!dead) {
                tc_fence_after();
                const float* swp = sw_s + (wg * 2 + (k & 1)) * WGC;
                // s_x truncated to 22 significant bits makes s_x' * 12582912 exact, so
                // fma(s_x', acc_bits, -s_x' * 12582912) = round(s_x' * sum): one rounding, and
                // the promotion costs two FMAs per element (relative change of s_x <= 2^-22).
                const float sxr = __int_as_float(__float_as_int(sx_cur) & ~3);
                const float kbias = -sxr * 12582912.0f;
#pragma unroll
                for (int j = 0; j < WGC / 32; ++j) {
                    uint32_t v[32];
                    QL_TMEM_LD16(tmem + tlane + buf * PN + wg * WGC + 32 * j, v);
                    QL_TMEM_LD16(tmem + tlane + buf * PN + wg * WGC + 32 * j + 16, (v + 16));
                    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
                    if constexpr (ACC) {
                        const int m = m0 + row;
                        if (m < a.M)
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                const int n = n0 + 32 * j + i;
                                if (n < a.N) a.acc[((long long)m * a.N + n) * G + g] = (int)(v[i] - kMagic);
                            }
                    } else {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 c4 = *reinterpret_cast<const float4*>(swp + 32 * j + 4 * q);
                            const int e = 32 * j + 4 * q;
                            yr[e + 0] = fmaf(c4.x, fmaf(sxr, __uint_as_float(v[4 * q + 0]), kbias), yr[e + 0]);
                            yr[e + 1] = fmaf(c4.y, fmaf(sxr, __uint_as_float(v[4 * q + 1]), kbias), yr[e + 1]);
                            yr[e + 2] = fmaf(c4.z, fmaf(sxr, __uint_as_float(v[4 * q + 2]), kbias), yr[e + 2]);
                            yr[e + 3] = fmaf(c4.w, fmaf(sxr, __uint_as_float(v[4 * q + 3]), kbias), yr[e + 3]);
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < WGC / 32; ++j) tmem_fill_magic32(tmem + tlane + buf * PN + wg * WGC + 32 * j);
                asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + 8 * (2 * PSTAGES + NBUF + buf));
            }
            // Weight scales of the next step into the other slot; rotate the prefetch.
            if (ti < WGC) sw_s[(wg * 2 + ((k + 1) & 1)) * WGC + ti] = __uint_as_float(sw_n1 << 16);
            sx_cur = sx_n1;
            sx_n1 = sx_n2;
            sw_n1 = sw_n2;
            fetch_next(sx_n2, sw_n2);
            wg_sync();

            if (++g == G) {  // tile done: write the warpgroup's 128 x 64 block of y
                if (!ACC) {
                    float* const yst = yst_s + wg * 128 * YST_STRIDE;
                    const int wi = ew & 3;  // this warp writes tile rows 32 * wi .. 32 * wi + 31
#pragma unroll
                    for (int c = 0; c < WGC / 16; ++c) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) yst[row * YST_STRIDE + i] = yr[16 * c + i];
                        wg_sync();
                        const int col = lane & 15;
                        const int n = n0 + 16 * c + col;
#pragma unroll 4
                        for (int rr = 0; rr < 32; rr += 2) {
                            const int r = 32 * wi + rr + (lane >> 4);
                            const int m = m0 + r;
                            if (!dead && m < a.M && n < a.N) a.y[(long long)m * a.ldy + n] = yst[r * YST_STRIDE + col];
                        }
                        wg_sync();
                    }
                }
#pragma unroll
                for (int i = 0; i < WGC; ++i) yr[i] = 0.0f;
                g = 0;
                ++tl;
            }
        }
        if (dead && lane == 0) atomicOr(a.err, (unsigned)QL_DEVERR_TIMEOUT);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(a.err, (unsigned)QL_DEVERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_prefill_w8a8(const int8_t* qx, const float* sx, const int8_t* qw, const uint16_t* sw, int M,
                                int N, int K, float* y, long long ldy, int32_t* acc, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    if ((size_t)SMEM_BYTES > di.smem_optin) return cudaErrorInvalidValue;
    PrefillArgs a;
    if ((e = make_tmap_2d(qx, M, K, K, PKB, PM, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmA)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(qw, N, K, K, PKB, PN, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmB)) != cudaSuccess) return e;
    a.sx = sx;
    a.sw = sw;
    a.y = y;
    a.acc = acc;
    a.err = di.err_word;
    a.M = M;
    a.N = N;
    a.G = K / 128;
    a.ldy = ldy;
    const int tiles = ((M + PM - 1) / PM) * ((N + PN - 1) / PN);
    const int grid = tiles < di.sm_count ? tiles : di.sm_count;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        for (auto fn : {k_prefill_w8a8<false>, k_prefill_w8a8<true>}) {
            if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) != cudaSuccess)
                return e;
        }
        if (dev < 64) attr_set[dev] = true;
    }
    if (acc) k_prefill_w8a8<true><<<grid, kPThreads, SMEM_BYTES, s>>>(a);
    else k_prefill_w8a8<false><<<grid, kPThreads, SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

}  // namespace ql
