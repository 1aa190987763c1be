// k_prefill.cu -- the prefill-shaped W8A8 GEMM (M >= 17 tokens) on the
// fifth-generation tensor cores: int8 activations (one fp32 scale per token
// per 128 values) times int8 weights (one bf16 scale per row per 128), each
// 128-wide group's integer dot product exact, both scales applied in fp32
// ("keptn/gemma4-12b-i8g", table "Format").
//
// Persistent CTAs, one per SM, walk 128 (tokens) x PN (weight rows) output
// tiles, weight-tile-major so the token blocks that share a weight tile run at
// the same time and read it from L2.  A step is one (tile, 128-K group): four
// tcgen05.mma kind::i8 of M = 128, N = PN, K = 32 into one of 512 / PN int32
// accumulators in tensor memory, the first of the four overwriting it.  An
// M = 128 MMA takes about as long at N = 64 as at N = 256, so wide tiles keep
// the tensor core busy; PN = 192 balances that against the epilogue's
// registers (it divides the 21504 weight rows of the dense layer, too).
//
// Warpgroup 0 drives the pipeline and then holds only 24 registers per
// thread: lane 0 of warp 0 issues the TMA loads of the activation tile
// [128][128 B] and the weight tile [PN][128 B] (128-byte swizzle) into a
// 4-slot operand ring and bulk-copies each step's 128 activation scales and
// PN weight scales (fp32, transposed beforehand into contiguous runs) into an
// 8-slot scale ring; lane 0 of warp 1 issues the MMAs (for E4M3, lane 0 of warps
// 1 and 2 issue the even and the odd steps, one accumulator each, so that one
// thread's barrier waits and its single commit per step hide behind the other's
// MMAs).  Warps 4..19 (112
// registers each) are the epilogue: thread i of warp w owns tile row
// 32 * (w % 4) + i (its tensor-memory lane) and PN / 4 columns.  Per step it
// reads its accumulators (tcgen05.ld 32x32b, 16 columns at a time, the next
// read in flight while the last is used), folds s_x[m, g] * s_w[n, g] * sum
// into fp32 running sums held in registers, and hands the accumulator and the
// step's scales back.
//
// The per-group promotion is the epilogue's cost: both scales change every
// 128 K, so every output element takes two fp32 FMAs per group.  Two is the
// least: the integer sum plus 0x4B400000 (|sum| <= 128 * 127^2 < 2^22), read
// as fp32, is exactly 12582912 + sum; with the row's activation scale cut to
// 22 significant bits (relative change <= 2^-22), s_x * 12582912 is exact, so
// one FMA yields s_x * sum rounded once and a second adds s_w times that to
// the running sum.  The first runs as packed two-lane FMAs (FFMA2, heavy FMA
// pipe only), the second as scalar FMAs, so both FMA pipes are busy.
//
// The same kernel runs format 7 (E4M3 weights and E4M3 activations, an fp32
// scale per token per 128 and a bf16 scale per 128 x 128 weight block) with
// tcgen05.mma kind::f8f6f4 at the same rate: the tiles are bytes either way,
// the accumulators hold fp32 group sums, and since a weight scale covers a
// whole 128-row block the promotion is one FMA per element with s_x * s_w taken
// once per 16 columns.
//
// A finished tile leaves through shared memory: each epilogue warp stages its
// 32 rows x PN / 4 columns in two halves in a private 3 KB buffer and one lane
// writes each half with a TMA tensor store (rows and columns past the matrix are
// clipped by the store).  Stored straight from registers, every warp store
// instruction would touch 32 rows, 16 bytes each, and at this tile rate those
// scattered writes cost about a sixth of the kernel's time.  Rows of y that are
// not 16-byte multiples (N % 4 != 0) take plain stores.
//
// All waits are bounded (200 ms); on a timeout the CTA sets
// QL_DEVERR_TIMEOUT and winds down without leaving tensor memory allocated,
// MMAs running or copies in flight.
#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

constexpr int PM = kPrefillTileM;         // tile rows (tokens)
constexpr int PN = kPrefillTileN;         // tile columns (weight rows): one MMA covers all of them
constexpr int PKB = 128;                  // K bytes per group
constexpr int A_BYTES = PM * PKB;         // 16 KB
constexpr int B_BYTES = PN * PKB;         // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
#ifndef QL_PF_STAGES
#define QL_PF_STAGES (QL_PF_N > 192 ? 3 : 4)
#endif
constexpr int PSTAGES = QL_PF_STAGES;     // operand ring slots
constexpr uint32_t kTmemCols = 512;
constexpr int NBUF = kTmemCols / PN;      // int32 accumulators in tensor memory
constexpr int SCB = 8;                    // scale ring slots
constexpr int SR = PSTAGES;               // step-commit ring: at least as long as the operand and accumulator rings
constexpr int SXS = PM + 4;               // s_x span of a scale slot: grouped tiles start on any row, so
                                          // their copy starts at the 16-byte boundary below it
constexpr int SC_BYTES = (SXS + PN) * 4;  // s_x of the tile's rows, then s_w of its columns
constexpr int kEpiWarps = 16;             // warps 4..19; warps 0..3 (warpgroup 0) drive the pipeline
constexpr int kPThreads = 32 * (4 + kEpiWarps);
constexpr int WGC = PN / 4;               // columns per thread (per warp column quarter)
constexpr int CW = 16;                    // columns per tensor-memory read
constexpr int NCH = WGC / CW;             // reads per step
constexpr uint32_t kMagic = 0x4B400000u;  // 12582912.0f
static_assert(PN % 32 == 0 && PN >= 128 && PN <= 256 && NBUF >= 2, "one MMA per K chunk covers the tile; 2+ accumulators");
static_assert(WGC % CW == 0, "whole tensor-memory reads per thread");
static_assert(PN % CW == 0 && WGC % CW == 0 && 128 % CW == 0,
              "column chunks start on multiples of CW, so none crosses a 128-row weight block");
static_assert(PN % 64 == 0 || PN == 160, "tile widths whose column quarters are whole reads");
static_assert(SCB >= PSTAGES + NBUF, "the scale ring must not throttle the operand ring");
static_assert(SR >= PSTAGES && SR >= NBUF && NBUF % 2 == 0, "one commit per step serves both rings; each issuer its own accumulators");
static_assert((SCB & (SCB - 1)) == 0, "scale slots from step counters");

// Shared memory (from a 1024-aligned base):
//   [operand ring][scale ring][mbarriers][tmem address]
constexpr int SC_OFF = PSTAGES * STAGE_BYTES;
constexpr int BAR_OFF = SC_OFF + SCB * SC_BYTES;
constexpr int BAR_FULL = 0, BAR_STEP = PSTAGES, BAR_ACCE = BAR_STEP + SR, BAR_SCF = BAR_ACCE + NBUF,
              BAR_SCE = BAR_SCF + SCB, BAR_DRAIN = BAR_SCE + SCB, NBARS = BAR_DRAIN + 1;
constexpr int MISC_OFF = (BAR_OFF + 8 * NBARS + 15) / 16 * 16;  // tmem address
// Output staging: each epilogue warp writes its 32 rows x WGC columns of a
// finished tile in two halves of YH columns through a private buffer, and one
// lane stores each half with a TMA tensor store.
constexpr int YH = WGC / 2;
constexpr int Y_WARP_BYTES = 32 * YH * 4;
constexpr int Y_OFF = (MISC_OFF + 16 + 1023) / 1024 * 1024;
constexpr int SMEM_BYTES = Y_OFF + kEpiWarps * Y_WARP_BYTES + 1024;
static_assert((YH * 4) % 16 == 0 && YH % 4 == 0 && Y_WARP_BYTES % 128 == 0,
              "TMA store boxes: 16-byte rows, 128-byte aligned staging");
static_assert(STAGE_BYTES % 1024 == 0, "operand slots must stay 1024-byte aligned for the 128-byte swizzle");
static_assert(SC_OFF % 16 == 0 && SC_BYTES % 16 == 0, "scale slots take 16-byte bulk copies and loads");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
static_assert(Y_OFF >= MISC_OFF + 16, "staging after the tensor-memory address");

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    // K-major, 128-byte swizzle: 8-row atoms 1024 bytes apart (SBO), version 1.
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// MMA kinds of this kernel: int8 x int8 -> s32, and E4M3 x E4M3 -> f32.
enum { kKindI8 = 0, kKindE4M3 = 1 };
// kind::i8, D s32, A s8, B s8, both K-major, N = PN, M = 128.
constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(PN >> 3) << 17) |
                              ((uint32_t)(PM >> 4) << 24);
// kind::f8f6f4, D f32, A e4m3 (0), B e4m3 (0), both K-major, N = PN, M = 128.
constexpr uint32_t kIdescE4M3 = (1u << 4) | ((uint32_t)(PN >> 3) << 17) | ((uint32_t)(PM >> 4) << 24);

// D (+)= A * B^T with K = 32 bytes; acc_in = 0 overwrites D.
template <int KIND>
__device__ __forceinline__ void mma_k32(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t acc_in) {
    if (KIND == kKindI8)
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
            "l"(adesc), "l"(bdesc), "r"(kIdescI8), "r"(acc_in));
    else
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
            "l"(adesc), "l"(bdesc), "r"(kIdescE4M3), "r"(acc_in));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
// Bulk tensor store of a staged box (global <- shared), tracked by bulk groups.
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];\n" ::"l"(tmap), "r"(x),
                 "r"(y), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// This thread's committed stores have read their shared-memory source.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory"); }
// ... and have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }
// Makes this thread's shared-memory writes visible to the TMA (async proxy).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ __forceinline__ void sts128(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
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
// Waits for this thread's tensor-memory reads; naming the registers of the last
// read ties their uses to after the wait.
#define QL_TMEM_WAIT16(v)                                                                                     \
    asm volatile("tcgen05.wait::ld.sync.aligned;\n"                                                          \
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]),       \
                   "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]),   \
                   "+r"(v[14]), "+r"(v[15])                                                                  \
                 :                                                                                           \
                 : "memory")

// The registers of a read issued before the last wait: ties their uses to after it
// (volatile asm statements keep their order).
#define QL_TMEM_AFTER_WAIT16(v)                                                                          \
    asm volatile(""                                                                                     \
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]),  \
                   "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), \
                   "+r"(v[14]), "+r"(v[15]))

struct PrefillArgs {
    CUtensorMap tmA;    // int8 activations [M][K], box [128 rows][128 B] (grouped: [P permuted rows][K])
    CUtensorMap tmB;    // int8 weights [N][K], box [PN rows][128 B] (grouped: the stacked experts [E * N][K])
    CUtensorMap tmY;    // y as bytes [M][4 N], row pitch 4 ldy, box [32 rows][4 YH B] (when ytma)
    const float* sxT;   // [G][Mp] activation scales (ACC: unused)
    const float* swT;   // [G][Np] weight scales as fp32 (ACC: unused)
    float* y;           // [M][ldy]
    int32_t* acc;       // group sums [M][N][G] (check path only)
    unsigned* err;
    int M, N, G, Mp, Np;
    int ytma;           // y is written by TMA stores (16-byte aligned rows)
    long long ldy;
    // Grouped over experts (format 7 MoE): tiles (expert, first permuted row, rows, weight block
    // of PN rows) from the permute, its count on the device; sxT [G][Mp] holds the permuted rows'
    // scales, swT [E][G][Np] each expert's weight scales; row r of a tile goes to y[perm[r]][..N).
    const MoeTile* tiles;
    const int* n_tiles;
    int max_tiles;
    const int32_t* perm;
};

// Where tile t of the CTA's walk sits: activation rows m0 .. m0 + rows, weight
// rows wrow .. + PN of the (stacked) weight matrix, the tile's weight block wb
// and expert.  Dense tiles go weight-tile-major.
struct TilePos {
    int m0, rows, wrow, wb, expert;
};
template <bool GRP>
__device__ __forceinline__ TilePos tile_pos(const PrefillArgs& a, int t, int MB) {
    if (GRP) {
        const MoeTile ti = a.tiles[t];
        return TilePos{ti.row0, ti.rows, ti.expert * a.N + ti.wb * PN, ti.wb, ti.expert};
    }
    const int m0 = (t % MB) * PM;
    return TilePos{m0, min(PM, a.M - m0), (t / MB) * PN, t / MB, 0};
}

// Registers: 640 threads launch with 96 each (61440).  Warpgroup 0 drops to
// 24 (3072) and the four epilogue warpgroups rise to 112 (57344): 60416 in
// all; per SM sub-partition 24 * 32 + 4 * 112 * 32 = 15104 of 16384.
constexpr int kRegsDriver = 24, kRegsEpi = 112;
static_assert(128 * kRegsDriver + 32 * kEpiWarps * kRegsEpi <= kPThreads * 96, "register split");

template <bool ACC, int KIND, bool GRP = false>
__global__ void __launch_bounds__(kPThreads, 1) k_prefill_w8a8(const __grid_constant__ PrefillArgs a) {
    static_assert(!ACC || KIND == kKindI8, "the integer group sums exist for int8 only");
    static_assert(!GRP || (KIND == kKindE4M3 && !ACC), "the grouped mode runs the E4M3 experts");
    // Two MMA-issuing threads for E4M3, whose light epilogue leaves the issue as the
    // limit; one for int8, whose heavier epilogue needs the issue slots instead.
    constexpr int kIssuers = KIND == kKindE4M3 ? 2 : 1;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const gb = smem_raw + (base - raw);
    auto bar = [&](int i) { return base + BAR_OFF + 8u * (uint32_t)i; };
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gb + MISC_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int MB = (a.M + PM - 1) / PM, NB = (a.N + PN - 1) / PN;
    const int tiles = GRP ? min(*a.n_tiles, a.max_tiles) : MB * NB;
    const int my_tiles = (int)blockIdx.x < tiles ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int G = a.G;
    const int total = my_tiles * G;  // steps of this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < PSTAGES; ++s) mbar_init(bar(BAR_FULL + s), 1);  // expect_tx
        for (int s = 0; s < SR; ++s) mbar_init(bar(BAR_STEP + s), 1);       // the step's MMA commit
        for (int b = 0; b < NBUF; ++b) mbar_init(bar(BAR_ACCE + b), kEpiWarps);  // one arrive per epilogue warp
        for (int b = 0; b < SCB; ++b) {
            mbar_init(bar(BAR_SCF + b), 1);          // expect_tx
            mbar_init(bar(BAR_SCE + b), kEpiWarps);  // one arrive per epilogue warp
        }
        mbar_init(bar(BAR_DRAIN), kIssuers);  // one commit per issuing thread
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
    bool dead = false;
    // Pipeline waits are bounded by lim; the waits that let started copies and MMAs
    // finish before the CTA ends keep the default bound.
    const unsigned long long lim = wait_limit(a.err);

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsDriver));
        if (warp == 0 && lane == 0) {  // ---- producer ----
            asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmA) : "memory");
            asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmB) : "memory");
            int g = 0, t = blockIdx.x, k = 0;
            TilePos tp = total > 0 ? tile_pos<GRP>(a, t, MB) : TilePos{0, 0, 0, 0, 0};
            for (; k < total; ++k) {
                const int s = k % PSTAGES, c = k & (SCB - 1);
                // the slot's previous operands (step k - PSTAGES) are free once that step's MMAs are done
                if ((k >= PSTAGES && !mbar_wait(bar(BAR_STEP + (k - PSTAGES) % SR), ((k - PSTAGES) / SR) & 1, lim)) ||
                    (!ACC && !mbar_wait(bar(BAR_SCE + c), ((k / SCB) & 1) ^ 1, lim))) {
                    dead = true;
                    break;
                }
                const uint32_t st = base + s * STAGE_BYTES, fb = bar(BAR_FULL + s);
                mbar_expect_tx(fb, STAGE_BYTES);
                tma_load_2d(st, &a.tmA, g * PKB, tp.m0, fb);
                tma_load_2d(st + A_BYTES, &a.tmB, g * PKB, tp.wrow, fb);
                if (!ACC) {
                    const uint32_t ss = base + SC_OFF + c * SC_BYTES, sb = bar(BAR_SCF + c);
                    const int sx0 = GRP ? (tp.m0 & ~3) : tp.m0;  // 16-byte aligned start of the s_x copy
                    const int sxn = GRP ? SXS : PM;
                    const long long sw0 = GRP ? ((long long)tp.expert * G + g) * a.Np + (long long)tp.wb * PN
                                              : (long long)g * a.Np + tp.wrow;
                    mbar_expect_tx(sb, (unsigned)(sxn + PN) * 4);
                    bulk_load(ss, a.sxT + (long long)g * a.Mp + sx0, sxn * 4, sb);
                    bulk_load(ss + SXS * 4, a.swT + sw0, PN * 4, sb);
                }
                if (++g == G) {
                    g = 0;
                    t += gridDim.x;
                    if (k + 1 < total) tp = tile_pos<GRP>(a, t, MB);
                }
            }
            // Copies still in flight must land before the CTA's shared memory is released.
            for (int j = k > PSTAGES ? k - PSTAGES : 0; j < k; ++j)
                if (!mbar_wait(bar(BAR_FULL + j % PSTAGES), (j / PSTAGES) & 1)) break;
            if (!ACC)
                for (int j = k > SCB ? k - SCB : 0; j < k; ++j)
                    if (!mbar_wait(bar(BAR_SCF + (j & (SCB - 1))), (j / SCB) & 1)) break;
        } else if ((warp == 1 || (kIssuers == 2 && warp == 2)) && lane == 0) {  // ---- MMA issuer(s) ----
            // The descriptors of slot s are those of slot 0 plus s * STAGE_BYTES / 16 (the
            // start-address field cannot carry: shared addresses are below 2^18), each
            // K = 32 chunk 2 further.
            const uint64_t da0 = smem_desc_sw128(base), db0 = smem_desc_sw128(base + A_BYTES);
            for (int k = warp - 1; k < total; k += kIssuers) {  // two issuers: b = k % NBUF is this thread's
                const int s = k % PSTAGES, b = k % NBUF;
                if (!mbar_wait(bar(BAR_FULL + s), (k / PSTAGES) & 1, lim) ||
                    !mbar_wait(bar(BAR_ACCE + b), (k / NBUF) & 1, lim)) {
                    dead = true;
                    break;
                }
                tc_fence_after();
                const uint64_t so = (uint64_t)(s * (STAGE_BYTES >> 4));
                const uint32_t d = tmem + b * PN;
#pragma unroll
                for (int kk = 0; kk < PKB / 32; ++kk)
                    mma_k32<KIND>(d, da0 + so + 2 * kk, db0 + so + 2 * kk, kk ? 1u : 0u);
                // One commit per step: its accumulator is ready and its operand slot free.  A
                // waiter for step j cannot see slot j % SR complete again first: step j + SR
                // needs that waiter to have moved on (the producer's operands for it, or the
                // epilogue freeing the accumulator after step j + SR - NBUF).
                mma_commit(bar(BAR_STEP + k % SR));
            }
            // Every MMA issued (by both threads) must finish before tensor memory is freed.
            mma_commit(bar(BAR_DRAIN));
            mbar_wait(bar(BAR_DRAIN), 0);
        }
    } else {  // ---- epilogue ----
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsEpi));
        const int wq = (warp >> 2) - 1;      // column quarter of the tile
        const int sub = warp & 3;            // tensor-memory lane quarter
        const int row = sub * 32 + lane;     // tile row of this thread
        const uint32_t tlane = (uint32_t)(sub * 32) << 16;
        const int tcol = wq * WGC;
        const bool vec_ok = (a.ldy & 3) == 0;

        // Every accumulator starts free.
        if (lane == 0)
            for (int b = 0; b < NBUF; ++b) mbar_arrive(bar(BAR_ACCE + b));

        float yr[WGC];
#pragma unroll
        for (int i = 0; i < WGC; ++i) yr[i] = 0.0f;
        int t = blockIdx.x, g = 0;
        TilePos tp = total > 0 ? tile_pos<GRP>(a, t, MB) : TilePos{0, 0, 0, 0, 0};
        for (int k = 0; k < total; ++k) {
            const int b = k % NBUF, c = k & (SCB - 1);
            const bool ok = mbar_wait(bar(BAR_STEP + k % SR), (k / SR) & 1, lim) &&
                            (ACC || mbar_wait(bar(BAR_SCF + c), (k / SCB) & 1, lim));
            if (!__all_sync(kFull, ok)) {  // the warp gives up together
                dead = true;
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem + tlane + b * PN + tcol;
            const float* scp = reinterpret_cast<const float*>(gb + SC_OFF + c * SC_BYTES);
            float sxr = 0.0f, kb = 0.0f;
            if (!ACC && KIND == kKindE4M3) {
                sxr = scp[(GRP ? (tp.m0 & 3) : 0) + row];  // fp32 group sums: t = s_x * sum, no bias
            } else if (!ACC) {
                // s_x cut to 22 significant bits: s_x * 12582912 is exact, so the first FMA is
                // round(s_x * sum) (the accumulator bits read as fp32 are 12582912 + sum).
                sxr = __int_as_float(__float_as_int(scp[row]) & ~3);
                kb = -sxr * 12582912.0f;
            }
            if constexpr (!ACC && KIND == kKindE4M3 && WGC <= 48) {
                // All of this thread's columns are read at once and the accumulator goes
                // back to the MMAs before the math: a light promotion leaves the read
                // latency, not the arithmetic, on the accumulator's round trip.
                uint32_t v[WGC];
#pragma unroll
                for (int h = 0; h < NCH; ++h) QL_TMEM_LD16(taddr + h * CW, (v + h * CW));
                QL_TMEM_WAIT16(v);
#pragma unroll
                for (int h = 1; h < NCH; ++h) QL_TMEM_AFTER_WAIT16((v + h * CW));
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BAR_ACCE + b));
                // fp8 weights scale whole 128-row blocks, and a 16-column chunk starts on a
                // multiple of 16 weight rows, so it never crosses a block: one s_x * s_w per
                // chunk, then one FMA per element (half packed, half scalar: both FMA pipes).
#pragma unroll
                for (int h = 0; h < NCH; ++h) {
                    const float p = sxr * scp[SXS + tcol + h * CW];
                    const float2 p2 = make_float2(p, p);
#pragma unroll
                    for (int q = 0; q < CW / 4; ++q) {
                        const uint32_t* const cu = v + h * CW + 4 * q;
                        float* const yq = yr + h * CW + 4 * q;
                        const float2 u = __ffma2_rn(p2, make_float2(__uint_as_float(cu[0]), __uint_as_float(cu[1])),
                                                    make_float2(yq[0], yq[1]));
                        yq[0] = u.x;
                        yq[1] = u.y;
                        yq[2] = fmaf(p, __uint_as_float(cu[2]), yq[2]);
                        yq[3] = fmaf(p, __uint_as_float(cu[3]), yq[3]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BAR_SCE + c));
            } else {
            const uint32_t mg = kMagic;
            const float2 sx2 = make_float2(sxr, sxr), kb2 = make_float2(kb, kb);
            uint32_t v[2][CW];
            QL_TMEM_LD16(taddr, v[0]);
            QL_TMEM_WAIT16(v[0]);
#pragma unroll
            for (int h = 0; h < NCH; ++h) {
                uint32_t* const cur = v[h & 1];
                if (h + 1 < NCH) QL_TMEM_LD16(taddr + (h + 1) * CW, v[(h + 1) & 1]);  // in flight during this math
                if constexpr (ACC) {
                    const int m = (t % MB) * PM + row, n0 = (t / MB) * PN + tcol + h * CW;
                    if (m < a.M)
#pragma unroll
                        for (int i = 0; i < CW; ++i)
                            if (n0 + i < a.N) a.acc[((long long)m * a.N + n0 + i) * G + g] = (int)cur[i];
                } else if constexpr (KIND == kKindE4M3) {  // wide tiles: one s_x * s_w per chunk, as above
                    const float p = sxr * scp[SXS + tcol + h * CW];
                    const float2 p2 = make_float2(p, p);
#pragma unroll
                    for (int q = 0; q < CW / 4; ++q) {
                        float* const yq = yr + h * CW + 4 * q;
                        const float2 u = __ffma2_rn(p2, make_float2(__uint_as_float(cur[4 * q]),
                                                                    __uint_as_float(cur[4 * q + 1])),
                                                    make_float2(yq[0], yq[1]));
                        yq[0] = u.x;
                        yq[1] = u.y;
                        yq[2] = fmaf(p, __uint_as_float(cur[4 * q + 2]), yq[2]);
                        yq[3] = fmaf(p, __uint_as_float(cur[4 * q + 3]), yq[3]);
                    }
                } else {
                    // Weight scales read in place (volatile loads stay in their chunk instead of being
                    // hoisted, which would cost registers).
                    const uint32_t swa = smem_u32(scp + SXS + tcol + h * CW);
#pragma unroll
                    for (int q = 0; q < CW / 4; ++q) {
                        const uint4 cu = lds128(swa + 16 * q);
                        const float4 cs = make_float4(__uint_as_float(cu.x), __uint_as_float(cu.y),
                                                      __uint_as_float(cu.z), __uint_as_float(cu.w));
                        // sum + 0x4B400000, read as fp32, is exactly 12582912 + sum
                        const float2 t0 = __ffma2_rn(sx2, make_float2(__uint_as_float(cur[4 * q] + mg),
                                                                      __uint_as_float(cur[4 * q + 1] + mg)), kb2);
                        const float2 t1 = __ffma2_rn(sx2, make_float2(__uint_as_float(cur[4 * q + 2] + mg),
                                                                      __uint_as_float(cur[4 * q + 3] + mg)), kb2);
                        float* const yq = yr + h * CW + 4 * q;
                        yq[0] = fmaf(cs.x, t0.x, yq[0]);
                        yq[1] = fmaf(cs.y, t0.y, yq[1]);
                        yq[2] = fmaf(cs.z, t1.x, yq[2]);
                        yq[3] = fmaf(cs.w, t1.y, yq[3]);
                    }
                }
                if (h + 1 < NCH) QL_TMEM_WAIT16(v[(h + 1) & 1]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(BAR_ACCE + b));
                if (!ACC) mbar_arrive(bar(BAR_SCE + c));
            }
            }

            if (++g == G) {  // tile done: this thread's WGC columns of its row of y
                if constexpr (GRP) {  // row of the permuted order -> its (token, slot) row of y
                    const int n0 = tp.wb * PN + tcol;
                    if (row < tp.rows && n0 < a.N) {
                        const int pair = __ldg(a.perm + tp.m0 + row);
                        float* yrow = a.y + (long long)pair * a.ldy + n0;
                        if (vec_ok && n0 + WGC <= a.N) {
#pragma unroll
                            for (int q = 0; q < WGC / 4; ++q)
                                *reinterpret_cast<float4*>(yrow + 4 * q) =
                                    make_float4(yr[4 * q], yr[4 * q + 1], yr[4 * q + 2], yr[4 * q + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < WGC; ++i)
                                if (n0 + i < a.N) yrow[i] = yr[i];
                        }
                    }
#pragma unroll
                    for (int i = 0; i < WGC; ++i) yr[i] = 0.0f;
                } else if (!ACC && a.ytma) {
                    const int r0 = (t % MB) * PM + sub * 32, n0 = (t / MB) * PN + tcol;
                    const uint32_t yb = base + Y_OFF + (uint32_t)(warp - 4) * Y_WARP_BYTES;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        if (lane == 0) bulk_wait_read();  // the buffer's previous store has read it
                        __syncwarp();
#pragma unroll
                        for (int q = 0; q < YH / 4; ++q)
                            sts128(yb + (uint32_t)lane * (YH * 4) + 16 * q, yr[hh * YH + 4 * q], yr[hh * YH + 4 * q + 1],
                                   yr[hh * YH + 4 * q + 2], yr[hh * YH + 4 * q + 3]);
                        fence_async_smem();
                        __syncwarp();
                        // Rows past M and columns past N are clipped by the store; boxes wholly outside are skipped.
                        if (lane == 0 && r0 < a.M && n0 + hh * YH < a.N) {
                            tma_store_2d(&a.tmY, yb, (n0 + hh * YH) * 4, r0);
                            bulk_commit();
                        }
                    }
#pragma unroll
                    for (int i = 0; i < WGC; ++i) yr[i] = 0.0f;
                } else if (!ACC) {
                    const int m = (t % MB) * PM + row, n0 = (t / MB) * PN + tcol;
                    if (m < a.M) {
                        float* yrow = a.y + (long long)m * a.ldy + n0;
                        if (vec_ok && n0 + WGC <= a.N) {
#pragma unroll
                            for (int q = 0; q < WGC / 4; ++q)
                                *reinterpret_cast<float4*>(yrow + 4 * q) =
                                    make_float4(yr[4 * q], yr[4 * q + 1], yr[4 * q + 2], yr[4 * q + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < WGC; ++i)
                                if (n0 + i < a.N) yrow[i] = yr[i];
                        }
                    }
#pragma unroll
                    for (int i = 0; i < WGC; ++i) yr[i] = 0.0f;
                }
                g = 0;
                t += gridDim.x;
                if (k + 1 < total) tp = tile_pos<GRP>(a, t, MB);
            }
        }
    }
    if (dead) atomicOr(a.err, (unsigned)QL_DEVERR_TIMEOUT);
    // Outstanding output stores finish before the CTA (and its staging buffers) goes.
    if (!ACC && a.ytma && warp >= 4 && lane == 0) bulk_wait_all();

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
    }
}

// bf16 (or f16) weight scales [N][G] -> fp32 [G][Np], columns n >= N zero.  32 x 32
// tiles through shared memory, so reads and writes are both coalesced.
template <bool kF16>
__global__ void __launch_bounds__(256) k_prefill_prep(const uint16_t* sw, int N, int G, int Np, float* swT) {
    __shared__ float tile[32][33];
    const int g0 = blockIdx.x * 32, n0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty + 8 * i, n = n0 + r, g = g0 + tx;
        const uint16_t b = (n < N && g < G) ? sw[(long long)n * G + g] : 0;
        tile[r][tx] = kF16 ? __half2float(__ushort_as_half(b)) : __uint_as_float((uint32_t)b << 16);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int gg = ty + 8 * i, g = g0 + gg;
        if (g < G) swT[(long long)g * Np + n0 + tx] = tile[tx][gg];
    }
}

// int5 codes with zero points -> the int8 codes q - z in [-31, 31] that the W8A8
// GEMM multiplies, [N][K].  One thread per 32 codes: 20 bytes of the row's
// least-significant-bit-first stream (code k at bits 5k .. 5k+4) in five
// 32-bit words, out as two 16-byte stores.  A row is K * 5 / 8 bytes, a
// multiple of 80, so every 32-code run starts on a 4-byte boundary.
__global__ void __launch_bounds__(256) k_prefill_i5_codes(const uint8_t* codes, const uint8_t* zeros, int N, int K,
                                                          int8_t* out) {
    const long long u = (long long)blockIdx.x * 256 + threadIdx.x;
    const int per_row = K / 32;
    if (u >= (long long)N * per_row) return;
    const long long n = u / per_row;
    const int j = (int)(u - n * per_row);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(codes + n * ((long long)K * 5 / 8) + (long long)j * 20);
    uint32_t w[6];
#pragma unroll
    for (int i = 0; i < 5; ++i) w[i] = src[i];
    w[5] = 0;
    const int z = zeros[n * (K / 128) + (j * 32) / 128];
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = 0;
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const int bit = 5 * c, wi = bit >> 5, sh = bit & 31;
        const uint32_t v = (sh <= 27 ? (w[wi] >> sh) : ((w[wi] >> sh) | (w[wi + 1] << (32 - sh)))) & 31u;
        o[c >> 2] |= (uint32_t)(((int)v - z) & 0xFF) << (8 * (c & 3));
    }
    uint4* dst = reinterpret_cast<uint4*>(out + n * (long long)K + (long long)j * 32);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

// bf16 block scales [ceil(N/128)][G] -> fp32 [G][Np], each row's block scale
// repeated for the 128 rows of its block; columns n >= N zero.  Expert e
// (blockIdx.y) reads its scales at sw + e * ceil(N/128) * G and writes
// swT + e * G * Np.
__global__ void __launch_bounds__(256) k_prefill_prep_blk(const uint16_t* sw, int N, int G, int Np, float* swT) {
    const long long i = (long long)blockIdx.x * 256 + threadIdx.x;
    if (i >= (long long)G * Np) return;
    const int g = (int)(i / Np), n = (int)(i - (long long)g * Np);
    sw += (long long)blockIdx.y * ((N + 127) / 128) * G;
    swT += (long long)blockIdx.y * G * Np;
    swT[i] = n < N ? __uint_as_float((uint32_t)sw[(long long)(n >> 7) * G + g] << 16) : 0.0f;
}

}  // namespace

cudaError_t launch_prefill_prep_blk(const uint16_t* sw, int N, int K, void* scratch, cudaStream_t s, int E) {
    const int G = K / 128, Np = prefill_pad_n(N);
    const long long n = (long long)G * Np;
    k_prefill_prep_blk<<<dim3((unsigned)((n + 255) / 256), (unsigned)E), 256, 0, s>>>(sw, N, G, Np,
                                                                                      static_cast<float*>(scratch));
    return cudaGetLastError();
}

cudaError_t launch_prefill_prep(const uint16_t* sw, int N, int K, void* scratch, cudaStream_t s, bool f16) {
    const int G = K / 128, Np = prefill_pad_n(N);
    const dim3 grid((G + 31) / 32, Np / 32);
    if (f16) k_prefill_prep<true><<<grid, 256, 0, s>>>(sw, N, G, Np, static_cast<float*>(scratch));
    else k_prefill_prep<false><<<grid, 256, 0, s>>>(sw, N, G, Np, static_cast<float*>(scratch));
    return cudaGetLastError();
}

cudaError_t launch_prefill_i5_codes(const uint8_t* codes, const uint8_t* zeros, int N, int K, int8_t* out,
                                    cudaStream_t s) {
    const long long units = (long long)N * (K / 32);
    const long long blocks = (units + 255) / 256;
    k_prefill_i5_codes<<<(unsigned)blocks, 256, 0, s>>>(codes, zeros, N, K, out);
    return cudaGetLastError();
}

cudaError_t launch_prefill_w8a8(const int8_t* qx, const float* sxT, const int8_t* qw, int M, int N, int K, float* y,
                                long long ldy, int32_t* acc, const void* scratch, cudaStream_t s, bool e4m3) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    if ((size_t)SMEM_BYTES > di.smem_optin) return cudaErrorInvalidValue;
    if (!acc && (!sxT || !scratch || !y)) return cudaErrorInvalidValue;
    PrefillArgs a;
    if ((e = make_tmap_2d(qx, M, K, K, PKB, PM, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmA)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(qw, N, K, K, PKB, PN, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmB)) != cudaSuccess) return e;
    a.sxT = sxT;
    a.swT = static_cast<const float*>(scratch);
    a.y = y;
    a.acc = acc;
    a.err = di.err_word;
    a.M = M;
    a.N = N;
    a.G = K / 128;
    a.Mp = prefill_pad_m(M);
    a.Np = prefill_pad_n(N);
    a.ldy = ldy;
    a.ytma = 0;
    if (!acc && ldy % 4 == 0 && (reinterpret_cast<uintptr_t>(y) & 15) == 0) {
        if ((e = make_tmap_2d(y, M, 4LL * N, 4 * ldy, YH * 4, 32, CU_TENSOR_MAP_SWIZZLE_NONE, &a.tmY)) != cudaSuccess)
            return e;
        a.ytma = 1;
    }
    const int tiles = ((M + PM - 1) / PM) * ((N + PN - 1) / PN);
    const int grid = tiles < di.sm_count ? tiles : di.sm_count;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        for (auto fn : {k_prefill_w8a8<false, kKindI8>, k_prefill_w8a8<true, kKindI8>,
                        k_prefill_w8a8<false, kKindE4M3>}) {
            if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) != cudaSuccess)
                return e;
        }
        if (dev < 64) attr_set[dev] = true;
    }
    if (acc && e4m3) return cudaErrorInvalidValue;
    if (acc) k_prefill_w8a8<true, kKindI8><<<grid, kPThreads, SMEM_BYTES, s>>>(a);
    else if (e4m3) k_prefill_w8a8<false, kKindE4M3><<<grid, kPThreads, SMEM_BYTES, s>>>(a);
    else k_prefill_w8a8<false, kKindI8><<<grid, kPThreads, SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_prefill_e4m3_grouped(const uint8_t* qx, const float* sxT, int Mp, const uint8_t* codes,
                                        const float* swT, int E, int N, int K, int rows_total, const MoeTile* tiles,
                                        const int* n_tiles, int max_tiles, const int32_t* perm, float* y,
                                        cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    if ((size_t)SMEM_BYTES > di.smem_optin) return cudaErrorInvalidValue;
    if (Mp % 4 || (reinterpret_cast<uintptr_t>(sxT) & 15)) return cudaErrorInvalidValue;
    PrefillArgs a;
    if ((e = make_tmap_2d(qx, rows_total, K, K, PKB, PM, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmA)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(codes, (long long)E * N, K, K, PKB, PN, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmB)) != cudaSuccess)
        return e;
    a.sxT = sxT;
    a.swT = swT;
    a.y = y;
    a.acc = nullptr;
    a.err = di.err_word;
    a.M = rows_total;
    a.N = N;
    a.G = K / 128;
    a.Mp = Mp;
    a.Np = prefill_pad_n(N);
    a.ldy = N;
    a.ytma = 0;
    a.tiles = tiles;
    a.n_tiles = n_tiles;
    a.max_tiles = max_tiles;
    a.perm = perm;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        if ((e = cudaFuncSetAttribute(k_prefill_w8a8<false, kKindE4M3, true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) != cudaSuccess)
            return e;
        if (dev < 64) attr_set[dev] = true;
    }
    const int grid = max_tiles < di.sm_count ? max_tiles : di.sm_count;
    k_prefill_w8a8<false, kKindE4M3, true><<<grid, kPThreads, SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

}  // namespace ql
