// k_prefill_a16.cu -- the prefill-shaped GEMM (M >= 17 tokens) for the
// formats whose activations stay 16-bit: int8 codes with a bf16 or f16 scale
// per row per 128 of K ("gemma4-26b-a4b-dflash-i8" README, table "Weights")
// and FP8 E4M3 codes with a bf16 scale per 128 x 128 block
// ("gemma4-26b-a4b-dflash-fp8" README, table "Weights").
//
// The tensor cores run kind::f16 (f16 x f16, fp32 accumulation) with the
// roles turned around: the MMA's M = 128 rows are weight rows, its N = TN
// columns are tokens (192 by default).  Both operands are exact:
//  * the codes are converted to f16 exactly (every int8 and every e4m3 value
//    is an f16) by a converter warpgroup, which writes them straight into
//    tensor memory as the MMA's A operand -- no shared-memory round trip for
//    the widened weights;
//  * the activations are the f16 copy of x scaled per token by a power of two
//    (prepared by the activation prologue), loaded by TMA into shared memory
//    as the B operand.
// A grouped tile holds one expert's rows, about 128 of 192 when 2048 tokens are
// routed top-8 over 128 experts: its MMAs are as wide as its rows (rounded up
// to 16), a tile of at most 128 rows loads 128-row activation boxes, and the
// epilogue reads only the columns of its rows.
// One step is one 128-K group: eight MMAs with K = 16 into one of the fp32
// accumulators [128 weight rows x TN tokens] (two at TN = 192, three at
// TN = 128, as tensor memory allows next to two A tiles).  The epilogue thread that owns
// a weight row (its tensor-memory lane) folds the group's weight scale, a
// scalar for that thread, into fp32 running sums: one FMA per element per
// group.  At the end of a tile each sum is multiplied by its token's inverse
// factor and written to y (32 lanes of a warp write 32 consecutive y values).
//
// Warp roles: warpgroup 0 (24 registers per thread after setmaxnreg): lane 0
// of warp 0 issues the TMA loads of the code tiles [128 rows][128 B] into a 4-
// or 6-slot ring, lane 0 of warp 3 those of the activation tiles [TN rows][2 x
// 128 B] into a 3-slot ring (two threads, so that neither ring waits for the
// other and each loop fits the warpgroup's registers), lane 0 of warps 1 and 2
// issue the MMAs of the even and the odd steps.  The next one
// or two warpgroups (40 registers) convert: thread i of warp 4 + 4 h + q
// converts part h of weight row 32 q + i (the whole row with one warpgroup,
// halves with two).  The last four warpgroups (96 or 104 registers) are the
// epilogue: warp w owns rows 32 (w % 4) .. + 31 and TN / 4 of the tokens.
//
// The tensor pipe must never wait for its issuer: a tcgen05.mma is accepted
// only about one MMA ahead of the one executing, so every cycle an issuing
// thread spends on barriers and commits would leave the pipe idle.  Hence two
// issuing threads taking alternate steps (the steps are independent: each has
// its own accumulator, A tile and activation slot, so their MMAs may
// interleave), whose waits hide behind each other's MMAs, and a single commit
// per step: the consumers of a step (the epilogue reading its accumulator, the
// converters and the producer reusing its A tile and activation slot) all
// wait on that one commit, on a ring of 6 mbarriers (a multiple of the
// activation, A-tile and accumulator ring depths).
//
// The grouped mode (GRP: the MoE experts' tiles from the permute kernel) is
// not launched: it is withdrawn until the cause of an intermittent device
// fault seen with it, in repeated calls at 2048 tokens x top-8, is found.
//
// All waits are bounded (200 ms); on a timeout the CTA sets QL_DEVERR_TIMEOUT
// and winds down without leaving tensor memory allocated, MMAs running or
// copies in flight.
#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

constexpr int TM = 128;                   // weight rows per tile (MMA M)
constexpr int TN = kPrefillA16Tokens;     // tokens per tile (MMA N)
constexpr int GK = 128;                   // K per step (one group)
constexpr int CODE_BYTES = TM * GK;       // one code tile (1-byte codes), 16 KB
constexpr int XATOM = TN * 128;           // one activation box: [TN rows][64 f16 = 128 B]
constexpr int X_BYTES = 2 * XATOM;        // the step's activations, 48 KB
constexpr int CS = TN > 128 ? 4 : 6, XS = 3;  // ring slots (codes, activations)
constexpr int AS = 2;                     // converted A tiles in tensor memory
constexpr int NACC = (512 - AS * 64) / TN;  // fp32 accumulators [128 x TN] in tensor memory
constexpr int SR = 6;                     // step-commit ring: a multiple of XS, AS and NACC
constexpr int ACOLS = GK / 2;             // tensor-memory columns of one converted A tile (f16 pairs)
constexpr int A_COL0 = NACC * TN;         // A tiles follow the accumulators
constexpr uint32_t kTmemCols = 512;
constexpr int kConvWarps = TN > 128 ? 4 : 8;  // one or two per sub-partition (a row or half a row each)
constexpr int kRowParts = kConvWarps / 4;     // converter warps per weight row
constexpr int CPW = 8 / kRowParts;            // 16-byte code chunks per converter thread
constexpr int kEpiWarps = 16;
constexpr int kEpiWarp0 = 4 + kConvWarps;
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
constexpr int EPC = TN / 4;               // tokens per epilogue thread
constexpr int CW = 16;                    // columns per tensor-memory read
static_assert(A_COL0 + AS * ACOLS <= (int)kTmemCols, "tensor memory budget");
static_assert(SR % XS == 0 && SR % AS == 0 && SR % NACC == 0, "one commit ring serves every per-step resource");
static_assert(EPC % CW == 0 && EPC <= 64 && TN % 16 == 0 && TN <= 256, "token tile");
static_assert(XATOM % 1024 == 0, "activation boxes stay 1024-byte aligned for the 128-byte swizzle");

// Shared memory (from a 1024-aligned base): [code ring][activation ring][mbarriers][tmem address]
constexpr int X_OFF = CS * CODE_BYTES;
constexpr int BAR_OFF = X_OFF + XS * X_BYTES;
constexpr int B_CFULL = 0, B_CEMPTY = CS, B_XFULL = 2 * CS, B_AFULL = 2 * CS + XS, B_STEP = B_AFULL + AS,
              B_DEMPTY = B_STEP + SR, B_DRAIN = B_DEMPTY + NACC, NBARS = B_DRAIN + 1;
constexpr int MISC_OFF = (BAR_OFF + 8 * NBARS + 15) / 16 * 16;
constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");

// Registers: 896 threads (128-token tiles) launch with 72 each, 768 threads
// (wider tiles) with 80.  Warpgroup 0 drops to 24, the converters to 40, the
// epilogue (32 or 48 running sums per thread) rises to 96 or 104:
// 128 * 24 + 256 * 40 + 512 * 96 = 62464 <= 896 * 72, and
// 128 * 24 + 128 * 40 + 512 * 104 = 61440 <= 768 * 80.
constexpr int kRegsLaunch = (65536 / kThreads) & ~7, kRegsDriver = 24, kRegsConv = 40, kRegsEpi = TN > 128 ? 104 : 96;
static_assert(128 * kRegsDriver + 32 * kConvWarps * kRegsConv + 32 * kEpiWarps * kRegsEpi <= kThreads * kRegsLaunch,
              "register split");
static_assert(32 * (kRegsDriver + kRowParts * kRegsConv + 4 * kRegsEpi) <= 16384, "registers per sub-partition");

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    // K-major, 128-byte swizzle: 8-row atoms 1024 bytes apart (SBO), version 1.
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// kind::f16: D f32, A f16, B f16, both K-major, M = 128, N = n (a multiple of 16, at most TN).
__device__ __forceinline__ uint32_t idesc_f16(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
}

// D (+)= A * B^T with A in tensor memory; acc_in = 0 overwrites D.
__device__ __forceinline__ void mma_f16_ts(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t acc_in) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc_in));
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
// Waits for this thread's tensor-memory reads; naming the registers of the last
// read ties their uses to after the wait.
#define QL_TMEM_WAIT16(v)                                                                                     \
    asm volatile("tcgen05.wait::ld.sync.aligned;\n"                                                          \
                 : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]),       \
                   "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]),   \
                   "+r"(v[14]), "+r"(v[15])                                                                  \
                 :                                                                                           \
                 : "memory")
#define QL_TMEM_ST16(addr, w)                                                                                   \
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
                 "%15,%16};\n" ::"r"(addr),                                                                     \
                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),       \
                 "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])  \
                 : "memory")

struct A16Args {
    CUtensorMap tmW;       // codes [E * N][K] bytes (E = 1 when dense), box [128 rows][128 B]
    CUtensorMap tmX;       // f16 activations [M][K] as bytes, box [TN rows][128 B]
    CUtensorMap tmXb;      // the same, box [128 rows][128 B]
    const uint16_t* sw;    // scales per expert: [N][G] (int8 formats) or [ceil(N/128)][G] (fp8), bf16 or f16 bits
    const float* xf;       // inverse token factors: [M] (dense) or [T] (grouped, token of pair p = p / topk)
    float* y;              // dense: [M][ldy]; grouped: [T * topk][ldy = N]
    unsigned* err;
    int M, N, G;
    long long ldy;
    const MoeTile* tiles;  // grouped: the tile table and its length on the device
    const int* n_tiles;
    const int32_t* perm;   // grouped: permuted row -> pair index t * topk + j
    int topk;
    int E, max_tiles;      // grouped: experts, the tile table's capacity (bounds of its entries)
};

// The tile a CTA works on: expert, first activation row, rows, weight block.
template <bool GRP>
__device__ __forceinline__ MoeTile tile_at(const A16Args& a, int t, int TB) {
    if (GRP) return a.tiles[t];
    const int row0 = (t % TB) * kPrefillA16Tokens;
    return MoeTile{0, row0, min(kPrefillA16Tokens, a.M - row0), t / TB};
}

// 16 codes (bytes of u) -> 8 f16 pairs, element order kept (low half = lower k).
template <int FMT>
__device__ __forceinline__ void convert16(const uint4 u, uint32_t* w) {
    const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (FMT == QL_FP8_B128_BF16) {
            w[2 * i] = e4m3x2_to_f16x2(q[i] & 0xFFFFu);
            w[2 * i + 1] = e4m3x2_to_f16x2(q[i] >> 16);
        } else {
            i8x4_to_f16(q[i], w[2 * i], w[2 * i + 1]);
        }
    }
}

template <int FMT, bool GRP>
__global__ void __launch_bounds__(kThreads, 1) k_prefill_a16(const __grid_constant__ A16Args a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const gb = smem_raw + (base - raw);
    auto bar = [&](int i) { return base + BAR_OFF + 8u * (uint32_t)i; };
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(gb + MISC_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int WB = (a.N + TM - 1) / TM, TB = (a.M + TN - 1) / TN;
    // dense: weight-block-major, t -> (wb = t / TB, tb = t % TB); grouped: the permute's table
    int tiles = GRP ? *a.n_tiles : WB * TB;
    if (GRP) {
        // The tile table comes from the permute kernel on the device: a CTA runs only if the
        // count and every one of its tiles lie inside the buffers (else it flags and skips).
        bool bad = tiles < 0 || tiles > a.max_tiles;
        for (int t = blockIdx.x; !bad && t < tiles; t += gridDim.x) {
            const MoeTile ti = a.tiles[t];
            bad = ti.expert < 0 || ti.expert >= a.E || ti.rows < 1 || ti.rows > TN || ti.row0 < 0 ||
                  ti.row0 + ti.rows > a.M || ti.wb < 0 || ti.wb >= WB;
        }
        if (bad) {
            if (threadIdx.x == 0) atomicOr(a.err, (unsigned)QL_DEVERR_BOUNDS);
            tiles = 0;
        }
    }
    const int my_tiles = (int)blockIdx.x < tiles ? (tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int G = a.G;
    const int total = my_tiles * G;

    if (threadIdx.x == 0) {
        for (int s = 0; s < CS; ++s) {
            mbar_init(bar(B_CFULL + s), 1);           // expect_tx
            mbar_init(bar(B_CEMPTY + s), kConvWarps);  // one arrive per converter warp
        }
        for (int s = 0; s < XS; ++s) mbar_init(bar(B_XFULL + s), 1);           // expect_tx
        for (int s = 0; s < AS; ++s) mbar_init(bar(B_AFULL + s), kConvWarps);  // one arrive per converter warp
        for (int s = 0; s < SR; ++s) mbar_init(bar(B_STEP + s), 1);            // the step's MMA commit
        for (int s = 0; s < NACC; ++s) mbar_init(bar(B_DEMPTY + s), kEpiWarps);  // one arrive per epilogue warp
        mbar_init(bar(B_DRAIN), 2);  // one commit per issuing thread
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
        if (warp == 0 && lane == 0) {  // ---- producer of the code tiles ----
            asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmW) : "memory");
            int g = 0, t = blockIdx.x, k = 0;
            int n0 = 0;  // code row of the tile in the stacked experts
            for (; k < total; ++k) {
                if (g == 0) {
                    const MoeTile ti = tile_at<GRP>(a, t, TB);
                    n0 = ti.expert * a.N + ti.wb * TM;
                }
                const int c = k % CS;
                if (!mbar_wait(bar(B_CEMPTY + c), ((k / CS) & 1) ^ 1, lim)) {
                    dead = true;
                    break;
                }
                const uint32_t cb = bar(B_CFULL + c);
                mbar_expect_tx(cb, CODE_BYTES);
                tma_load_2d(base + c * CODE_BYTES, &a.tmW, g * GK, n0, cb);
                if (++g == G) {
                    g = 0;
                    t += gridDim.x;
                }
            }
            // Copies still in flight must land before the CTA's shared memory is released.
            for (int j = k > CS ? k - CS : 0; j < k; ++j)
                if (!mbar_wait(bar(B_CFULL + j % CS), (j / CS) & 1)) break;
        } else if (warp == 3 && lane == 0) {  // ---- producer of the activation tiles ----
            asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmX) : "memory");
            asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmXb) : "memory");
            int g = 0, t = blockIdx.x, k = 0;
            int m0 = 0, rows = 0;  // first activation row of the tile, its rows
            for (; k < total; ++k) {
                if (g == 0) {
                    const MoeTile ti = tile_at<GRP>(a, t, TB);
                    m0 = ti.row0;
                    rows = ti.rows;
                }
                const int x = k % XS;
                if (k >= XS && !mbar_wait(bar(B_STEP + (k - XS) % SR), ((k - XS) / SR) & 1, lim)) {
                    dead = true;  // the slot's previous activations are still in use
                    break;
                }
                const uint32_t xb = bar(B_XFULL + x), xd = base + X_OFF + x * X_BYTES;
                // A grouped tile of at most 128 rows loads 128-row boxes, a wider one the TN-row boxes.
                const bool narrow = GRP && rows <= 128;
                const CUtensorMap* const tm = narrow ? &a.tmXb : &a.tmX;
                mbar_expect_tx(xb, narrow ? 2 * 128 * 128 : X_BYTES);
                tma_load_2d(xd, tm, g * GK * 2, m0, xb);
                tma_load_2d(xd + XATOM, tm, g * GK * 2 + 128, m0, xb);
                if (++g == G) {
                    g = 0;
                    t += gridDim.x;
                }
            }
            for (int j = k > XS ? k - XS : 0; j < k; ++j)
                if (!mbar_wait(bar(B_XFULL + j % XS), (j / XS) & 1)) break;
        } else if ((warp == 1 || warp == 2) && lane == 0) {  // ---- MMA issuers: even / odd steps ----
            const uint64_t xd0 = smem_desc_sw128(base + X_OFF);
            // The step's tile (its position tcur among this CTA's tiles, and gk, the step within
            // it) advances by two steps per iteration without a division.
            int tcur = 0, gk = warp - 1;
            while (gk >= G) gk -= G, ++tcur;
            int tload = -1;               // tile position whose width idesc holds
            uint32_t idesc = idesc_f16(TN);  // the MMA's N: the tile's rows rounded up to 16 (grouped)
            for (int k = warp - 1; k < total; k += 2) {
                const int x = k % XS, ab = k % AS, db = k % NACC;
                if constexpr (GRP) {
                    if (tcur != tload) {
                        tload = tcur;
                        idesc = idesc_f16((tile_at<GRP>(a, (int)blockIdx.x + tcur * (int)gridDim.x, TB).rows + 15) & ~15);
                    }
                    gk += 2;
                    while (gk >= G) gk -= G, ++tcur;
                }
                if (!mbar_wait(bar(B_XFULL + x), (k / XS) & 1, lim) || !mbar_wait(bar(B_AFULL + ab), (k / AS) & 1, lim) ||
                    !mbar_wait(bar(B_DEMPTY + db), ((k / NACC) & 1) ^ 1, lim)) {
                    dead = true;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + db * TN, at = tmem + A_COL0 + ab * ACOLS;
                const uint64_t xo = (uint64_t)((x * X_BYTES) >> 4);
#pragma unroll
                for (int j = 0; j < GK / 16; ++j)
                    mma_f16_ts(d, at + 8 * j, xd0 + xo + (uint64_t)((j / 4) * (XATOM >> 4) + (j % 4) * 2), idesc,
                               j ? 1u : 0u);
                // One commit per step: its accumulator is ready for the epilogue, and its
                // A tile and activation slot may be refilled.  A waiter for step j checks
                // the parity of its completion on slot j % SR, and the slot cannot
                // complete again before that check: step j + SR needs the waiter to have
                // moved on first (the producer's activations for it, the converters' A
                // tile for it, or the epilogue freeing its accumulator after step
                // j + SR - NACC).
                mma_commit(bar(B_STEP + k % SR));
            }
            // Every MMA issued (by both threads) must finish before tensor memory is freed.
            mma_commit(bar(B_DRAIN));
            mbar_wait(bar(B_DRAIN), 0);
        }
    } else if (warp < kEpiWarp0) {  // ---- converters ----
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRegsConv));
        const int q = warp & 3, h = (warp - 4) >> 2, r = 32 * q + lane;  // weight row, part of its 128 codes
        const uint32_t tl = (uint32_t)(32 * q) << 16;
        for (int k = 0; k < total; ++k) {
            const int c = k % CS, ab = k % AS;
            const bool ok = mbar_wait(bar(B_CFULL + c), (k / CS) & 1, lim) &&
                            (k < AS || mbar_wait(bar(B_STEP + (k - AS) % SR), ((k - AS) / SR) & 1, lim));
            if (!__all_sync(kFull, ok)) {  // the warp gives up together
                dead = true;  // no codes, or the A tile's previous MMAs are still running
                break;
            }
            tc_fence_after();
            // Row r of the code tile: 16-byte chunk j sits at chunk j ^ (r & 7) (128-byte swizzle).
            const uint32_t rowp = base + c * CODE_BYTES + r * 128;
            const uint32_t at = tmem + tl + A_COL0 + ab * ACOLS + 8 * CPW * h;
#pragma unroll
            for (int j = 0; j < CPW / 2; ++j) {
                const int ch = CPW * h + 2 * j;  // 16-byte chunks ch, ch + 1: codes 16 ch .. 16 ch + 31
                uint32_t w[16];
                convert16<FMT>(lds128(rowp + ((ch ^ (r & 7)) << 4)), w);
                convert16<FMT>(lds128(rowp + (((ch + 1) ^ (r & 7)) << 4)), w + 8);
                QL_TMEM_ST16(at + 16 * j, w);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(B_AFULL + ab));
                mbar_arrive(bar(B_CEMPTY + c));
            }
        }
    } else {  // ---- epilogue ----
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kRegsEpi));
        const int q = warp & 3, cg = (warp - kEpiWarp0) >> 2;
        const uint32_t tl = (uint32_t)(32 * q) << 16;
        float yacc[EPC];
#pragma unroll
        for (int i = 0; i < EPC; ++i) yacc[i] = 0.0f;
        int t = blockIdx.x, g = 0;
        const int NBk = (a.N + TM - 1) / TM;
        // Everything a step or a tile end needs from global memory is requested well
        // before it is used, so no load latency sits between the tensor-memory reads:
        //  * the group scale (raw 16 bits) one step ahead, converted only at its use;
        //  * the next tile's descriptor one tile ahead;
        //  * the output rows and token factors of this thread's activation rows
        //    during the tile's first steps (lane l: rows l and 32 + l).
        int n = 0, row0 = 0, rows = 0, pr0 = 0, pr1 = 0;
        float f0 = 0.0f, f1 = 0.0f;
        const uint16_t* sp = nullptr;
        MoeTile nt = my_tiles > 0 ? tile_at<GRP>(a, t, TB) : MoeTile{0, 0, 0, 0};
        auto start_tile = [&](int tt) {
            const MoeTile ti = nt;
            if (tt + (int)gridDim.x < tiles) nt = tile_at<GRP>(a, tt + (int)gridDim.x, TB);
            n = ti.wb * TM + 32 * q + lane;
            row0 = ti.row0 + cg * EPC;
            rows = ti.rows - cg * EPC;
            if (FMT == QL_FP8_B128_BF16) sp = a.sw + ((long long)ti.expert * NBk + n / 128) * G;
            else sp = n < a.N ? a.sw + ((long long)ti.expert * a.N + n) * G : nullptr;  // rows past N: scale 0
            pr0 = pr1 = 0;
            if (GRP) {  // row r of the permuted activations is the pair perm[r] = t * topk + j
                if (lane < rows) pr0 = __ldg(a.perm + row0 + lane);
                if (32 + lane < min(rows, EPC)) pr1 = __ldg(a.perm + row0 + 32 + lane);
            } else {
                pr0 = row0 + lane;
                pr1 = row0 + 32 + lane;
            }
        };
        auto scale_raw = [&](int gg) -> uint32_t { return sp ? (uint32_t)__ldg(sp + gg) : 0u; };
        uint32_t sb_next = 0;
        if (my_tiles > 0) {
            start_tile(t);
            sb_next = scale_raw(0);
        }
        for (int k = 0; k < total; ++k) {
            const int db = k % NACC;
            const float s = FMT == QL_I8_G128_F16 ? f16_bits_to_float((uint16_t)sb_next)
                                                  : bf16_bits_to_float((uint16_t)sb_next);
            if (g + 1 < G) sb_next = scale_raw(g + 1);
            if (!__all_sync(kFull, mbar_wait(bar(B_STEP + k % SR), (k / SR) & 1, lim))) {  // together
                dead = true;
                break;
            }
            tc_fence_after();
            const uint32_t dt = tmem + tl + db * TN + cg * EPC;
#pragma unroll
            for (int h = 0; h < EPC / CW; ++h) {
                if (GRP && h * CW >= rows) break;  // columns past the tile's rows were not computed (warp-uniform)
                uint32_t v[CW];
                QL_TMEM_LD16(dt + h * CW, v);
                QL_TMEM_WAIT16(v);
#pragma unroll
                for (int i = 0; i < CW; ++i) yacc[h * CW + i] = fmaf(s, __uint_as_float(v[i]), yacc[h * CW + i]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(B_DEMPTY + db));

            if (g == min(1, G - 1)) {  // the token factors, once the output rows have arrived
                f0 = lane < rows ? __ldg(a.xf + (GRP ? pr0 / a.topk : pr0)) : 0.0f;
                f1 = 32 + lane < min(rows, EPC) ? __ldg(a.xf + (GRP ? pr1 / a.topk : pr1)) : 0.0f;
            }
            if (++g == G) {  // tile done: activation rows row0 .. row0 + EPC - 1 against weight row n
#pragma unroll
                for (int i = 0; i < EPC; ++i) {
                    const float f = __shfl_sync(kFull, i < 32 ? f0 : f1, i & 31);
                    const long long orow = __shfl_sync(kFull, i < 32 ? pr0 : pr1, i & 31);
                    if (i < rows && n < a.N) a.y[orow * a.ldy + n] = yacc[i] * f;
                }
#pragma unroll
                for (int i = 0; i < EPC; ++i) yacc[i] = 0.0f;
                g = 0;
                t += gridDim.x;
                if (k + 1 < total) {
                    start_tile(t);
                    sb_next = scale_raw(0);
                }
            }
        }
    }
    if (dead) atomicOr(a.err, (unsigned)QL_DEVERR_TIMEOUT);

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
    }
}

template <int FMT, bool GRP>
cudaError_t launch_fmt(const A16Args& a, int grid, cudaStream_t s) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(k_prefill_a16<FMT, GRP>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[dev] = true;
    }
    k_prefill_a16<FMT, GRP><<<grid, kThreads, SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

template <bool GRP>
cudaError_t launch_any(int fmt, const A16Args& a, int grid, cudaStream_t s) {
    switch (fmt) {
    case QL_I8_G128_BF16: return launch_fmt<QL_I8_G128_BF16, GRP>(a, grid, s);
    case QL_I8_G128_F16: return launch_fmt<QL_I8_G128_F16, GRP>(a, grid, s);
    default: return launch_fmt<QL_FP8_B128_BF16, GRP>(a, grid, s);
    }
}

}  // namespace

bool prefill_a16_supported(int fmt) {
    return fmt == QL_I8_G128_BF16 || fmt == QL_I8_G128_F16 || fmt == QL_FP8_B128_BF16;
}

cudaError_t launch_prefill_a16(int fmt, const __half* xs, const float* xf, const uint8_t* codes, const void* scales,
                               int M, int N, int K, float* y, long long ldy, cudaStream_t s) {
    if (!prefill_a16_supported(fmt)) return cudaErrorInvalidValue;
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    if ((size_t)SMEM_BYTES > di.smem_optin) return cudaErrorInvalidValue;
    A16Args a{};
    if ((e = make_tmap_2d(codes, N, K, K, GK, TM, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmW)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(xs, M, 2LL * K, 2LL * K, 128, TN, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmX)) != cudaSuccess ||
        (e = make_tmap_2d(xs, M, 2LL * K, 2LL * K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmXb)) != cudaSuccess)
        return e;
    a.sw = static_cast<const uint16_t*>(scales);
    a.xf = xf;
    a.y = y;
    a.err = di.err_word;
    a.M = M;
    a.N = N;
    a.G = K / GK;
    a.ldy = ldy;
    const int tiles = ((N + TM - 1) / TM) * ((M + TN - 1) / TN);
    const int grid = tiles < di.sm_count ? tiles : di.sm_count;
    return launch_any<false>(fmt, a, grid, s);
}


}  // namespace ql
