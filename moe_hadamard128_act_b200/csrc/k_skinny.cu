// k_skinny.cu -- the decode-shaped quantized GEMM y = x . dequant(W)^T for
// M <= 16 tokens (one target token plus up to 15 drafted ones: the verification
// shape of the DFlash drafter in "gemma4-26b-a4b-dflash-i8", "Speculator"), and
// its grouped form over MoE experts.  At these shapes the layer is bound by
// streaming the packed weights from HBM (the decode step times on the cards
// barely move from 1 to 8 sequences), so the kernel is built around that
// stream:
//
//  * Persistent grid, one 512-thread CTA per SM.  The work is cut into units
//    of 16 weight rows x 128 K (one scale group), numbered row-slab-major, and
//    every warp takes an equal contiguous range of units, so all SMs finish
//    together whatever N and K are.
//  * Each lane streams its part of a unit straight into registers with 16-byte
//    (int8, fp8), 8-byte (int4) or 4-byte (int5) non-caching loads, two units
//    ahead of the one it computes: 16 warps x 3 units x 2 KB keep ~96 KB per
//    SM in flight, enough to cover HBM latency.
//  * The activations of all tokens are staged once per CTA in shared memory,
//    padded and swizzled so that the fragment loads are bank-conflict free.
//  * Dequantisation is in registers: codes become exact small integers in
//    f16 with two byte-permutes and one packed add per 4 codes (int8), mask
//    and add (int4, int5 -- the int5 zero point is folded into the add), or a
//    hardware e4m3x2 -> f16x2 convert.  The tensor cores (mma.sync m16n8k16,
//    f16 in, fp32 accumulate; m16n8k32 s8 in, exact s32 accumulate for W8A8)
//    multiply them by the activations with the token dimension as the MMA's
//    N = 8 side, and every group's partial sum is scaled in fp32 before it is
//    added, so no weight is ever rounded after scaling.
//  * A lane's 32 contiguous bytes of a weight row are assigned to MMA
//    fragment slots through a fixed permutation of K inside the group; the
//    activations are laid out with the same permutation, which leaves every
//    dot product unchanged.
//  * Partial sums leave through fp32 atomic adds only when a warp's range
//    leaves a 16-row slab (about twice per warp), into a y the caller zeroed.
#include <algorithm>

#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

#ifndef QL_SKINNY_THREADS
#define QL_SKINNY_THREADS 512
#endif
#ifndef QL_SKINNY_STAGES
#define QL_SKINNY_STAGES 4
#endif
constexpr int kThreads = QL_SKINNY_THREADS;
constexpr int kWarps = kThreads / 32;

// Register image of one unit's weights, for one lane.
template <int FMT>
struct Regs;
template <>
struct Regs<QL_I8_G128_BF16> {
    uint4 w[2][2];  // [row g / g+8][16-byte half of the lane's 32 bytes]
    float s[2];
};
template <>
struct Regs<QL_I8_G128_F16> : Regs<QL_I8_G128_BF16> {};
template <>
struct Regs<QL_I8A8_G128_BF16> : Regs<QL_I8_G128_BF16> {};
template <>
struct Regs<QL_FP8_B128_BF16> : Regs<QL_I8_G128_BF16> {};
template <>
struct Regs<QL_FP8A8_B128_BF16> : Regs<QL_I8_G128_BF16> {};

// The experts' bf16 down projection (not a packed format of the ABI): units of
// 16 rows x 64 bf16 weights, the same 128-byte rows as the int8 formats.
constexpr int kFmtDown = 16;
template <>
struct Regs<kFmtDown> : Regs<QL_I8_G128_BF16> {};

// Formats whose activations are one-byte codes with an fp32 scale per token
// per 128 (int8 for W8A8, E4M3 for format 7), multiplied on the byte MMAs.
template <int FMT>
__host__ __device__ constexpr bool act8() { return FMT == QL_I8A8_G128_BF16 || FMT == QL_FP8A8_B128_BF16; }
// int8 codes with 16-bit activations: the codes enter the MMAs as subnormals (q + 128) * 2^-24,
// and the offset comes off with the token's group sum (as the int5 zero point does).
template <int FMT>
__host__ __device__ constexpr bool i8sub() { return FMT == QL_I8_G128_BF16 || FMT == QL_I8_G128_F16; }
constexpr float kI8Off = 7.62939453125e-06f;  // 128 * 2^-24
// Weight scales per 128 x 128 block rather than per row.
template <int FMT>
__host__ __device__ constexpr bool block_scaled() { return FMT == QL_FP8_B128_BF16 || FMT == QL_FP8A8_B128_BF16; }
template <>
struct Regs<QL_I4_G64_BF16> {
    uint2 w[2][2];  // [row][64-wide half group]: 16 codes each
    float s[2][2];
};
template <>
struct Regs<QL_I5Z_G128_F16> {
    uint32_t w[2][5];  // [row][160-bit stream of 32 codes]
    float s[2];
    float zz[2];  // zero point * 2^-24 (the codes' unit in the MMAs)
};

// Bytes of activations per token per 128-group in shared memory, and the
// padding that makes the row stride an odd (1) or 2-mod-8 multiple of 16 B.
template <int FMT>
__host__ __device__ constexpr int x_group_bytes() { return act8<FMT>() ? 128 : 256; }
template <int FMT>
__host__ __device__ constexpr int x_row_pad() { return (act8<FMT>() || FMT == QL_I4_G64_BF16) ? 16 : 32; }
template <int FMT>
__host__ __device__ constexpr bool x_swizzled() { return !(act8<FMT>() || FMT == QL_I4_G64_BF16); }

template <int FMT>
__device__ __forceinline__ int swz(int j) { return x_swizzled<FMT>() ? (j ^ ((j >> 3) & 1)) : j; }

template <int FMT>
__device__ __forceinline__ float load_scale(const void* scales, long long idx) {
    const uint16_t b = __ldg(static_cast<const uint16_t*>(scales) + idx);
    return (FMT == QL_I8_G128_F16 || FMT == QL_I5Z_G128_F16) ? f16_bits_to_float(b) : bf16_bits_to_float(b);
}

__device__ __forceinline__ uint32_t word_of(const uint4 (&w)[2], int s) {
    const uint4& q = w[s >> 2];
    switch (s & 3) {
    case 0: return q.x;
    case 1: return q.y;
    case 2: return q.z;
    default: return q.w;
    }
}

// With a single n-tile the MMAs of a group would form one dependent chain; they
// alternate between CH accumulators instead, summed here into chain 0.
template <int CH, int NT, typename T>
__device__ __forceinline__ void fold_chains(T (&acc)[CH][NT][4]) {
#pragma unroll
    for (int ch = 1; ch < CH; ++ch)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[0][nt][i] += acc[ch][nt][i];
}

// One int4 unit (16 rows x 128 K: two 64-groups, each with its own scale).  The
// activations of odd k, which meet the high nibbles, were staged divided by 16
// (XORD_I4), so the operands need no shift to line the high nibble up:
//  - one n-tile: the codes enter the MMAs as exact f16 subnormals with one mask
//    each (low nibble u * 2^-24, high nibble in place 16 u * 2^-24), and the
//    offset of q = u - 8 comes off with the token's sum over the 64-group, X
//    (same units): y += s * (acc - 8 * 2^-24 * X), the scale carrying the 2^24
//    back (side_to_regs).  X[2 i + h]: token 2 c + i, half h.
//  - two n-tiles: the offset comes off in f16 instead (1024 + u - 1032 = q and
//    1024 + 16 u - 1152 = 16 q, both exact); X is unused.
constexpr float kI4Off = 4.76837158203125e-07f;  // 8 * 2^-24
template <int NT, typename GetX>
__device__ __forceinline__ void unit_i4(const Regs<QL_I4_G64_BF16>& r, GetX getx, bool nt1_live, const float (&X)[4],
                                        float (&yacc)[NT][4]) {
    constexpr int CH = NT == 1 ? 2 : 1;  // independent accumulation chains per group (see fold_chains)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float acc[CH][NT][4];
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[ch][nt][0] = acc[ch][nt][1] = acc[ch][nt][2] = acc[ch][nt][3] = 0.0f;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            uint4 xv[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                if (nt == 0 || nt1_live) xv[nt] = getx(nt, 8 * h + p);
            const uint32_t v0 = p == 0 ? r.w[0][h].x : r.w[0][h].y;  // row g: 8 codes of the lane's run
            const uint32_t v1 = p == 0 ? r.w[1][h].x : r.w[1][h].y;  // row g + 8
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
                // bytes (sub, sub + 2): low nibbles -> k = 2 c, 2 c + 1; high nibbles -> 2 c + 8, 2 c + 9
                const uint32_t w0 = sub == 0 ? v0 : v0 >> 8, w1 = sub == 0 ? v1 : v1 >> 8;
                uint32_t a0, a1, a2, a3;
                if constexpr (NT == 1) {
                    a0 = w0 & 0x000F000Fu;
                    a2 = w0 & 0x00F000F0u;
                    a1 = w1 & 0x000F000Fu;
                    a3 = w1 & 0x00F000F0u;
                } else {
                    a0 = hadd2_u32(and_or(w0, 0x000F000Fu, 0x64006400u), 0xE408E408u);
                    a2 = hadd2_u32(and_or(w0, 0x00F000F0u, 0x64006400u), 0xE480E480u);
                    a1 = hadd2_u32(and_or(w1, 0x000F000Fu, 0x64006400u), 0xE408E408u);
                    a3 = hadd2_u32(and_or(w1, 0x00F000F0u, 0x64006400u), 0xE480E480u);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt == 1 && !nt1_live) continue;
                    const uint32_t b0 = sub == 0 ? xv[nt].x : xv[nt].z;
                    const uint32_t b1 = sub == 0 ? xv[nt].y : xv[nt].w;
                    mma_f16(acc[sub % CH][nt], a0, a1, a2, a3, b0, b1);
                }
            }
        }
        fold_chains<CH, NT>(acc);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float t = NT == 1 ? fmaf(-kI4Off, X[2 * (i & 1) + h], acc[0][nt][i]) : acc[0][nt][i];
                yacc[nt][i] = fmaf(r.s[i >> 1][h], t, yacc[nt][i]);
            }
    }
}

// The per-group MMAs of one unit for the byte weight-only formats (int8, E4M3).
// getx(nt, piece) returns the lane's 16-byte activation piece for n-tile nt.
// X: the group sums of the lane's column tokens (int8 codes only: their subnormal offset).
// yacc[nt][i] accumulates scale * partial; i = 0,1 row g, i = 2,3 row g + 8.
template <int FMT, int NT, typename GetX>
__device__ __forceinline__ void unit_a16(const Regs<FMT>& r, GetX getx, bool nt1_live, const float (&X)[NT][2],
                                         float (&yacc)[NT][4]) {
    constexpr int CH = NT == 1 ? 2 : 1;  // independent accumulation chains per group (see fold_chains)
    {
        float acc[CH][NT][4];
#pragma unroll
        for (int ch = 0; ch < CH; ++ch)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[ch][nt][0] = acc[ch][nt][1] = acc[ch][nt][2] = acc[ch][nt][3] = 0.0f;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            uint4 xv[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                if (nt == 0 || nt1_live) xv[nt] = getx(nt, p);
#pragma unroll
            for (int sub = 0; sub < 2; ++sub) {
                const int s = 2 * p + sub;
                uint32_t a0, a1, a2, a3;
                if constexpr (FMT == QL_FP8_B128_BF16) {
                    const uint32_t w0 = word_of(r.w[0], s), w1 = word_of(r.w[1], s);
                    a0 = e4m3x2_to_f16x2(w0);
                    a2 = e4m3x2_to_f16x2(w0 >> 16);
                    a1 = e4m3x2_to_f16x2(w1);
                    a3 = e4m3x2_to_f16x2(w1 >> 16);
                } else {
                    i8x4_to_f16sub(word_of(r.w[0], s), a0, a2);
                    i8x4_to_f16sub(word_of(r.w[1], s), a1, a3);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt == 1 && !nt1_live) continue;
                    const uint32_t b0 = sub == 0 ? xv[nt].x : xv[nt].z;
                    const uint32_t b1 = sub == 0 ? xv[nt].y : xv[nt].w;
                    mma_f16(acc[sub % CH][nt], a0, a1, a2, a3, b0, b1);
                }
            }
        }
        fold_chains<CH, NT>(acc);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float t = i8sub<FMT>() ? fmaf(-kI8Off, X[nt][i & 1], acc[0][nt][i]) : acc[0][nt][i];
                yacc[nt][i] = fmaf(r.s[i >> 1], t, yacc[nt][i]);
            }
    }
}

// int5 register pair Q of a row (kI5Pairs): the stream window at bit B masked to
// its two codes, each an exact f16 subnormal u * 2^(o - 24).
template <int Q>
__device__ __forceinline__ uint32_t i5_pair(const uint32_t (&w)[5]) {
    constexpr int B = kI5Pairs[Q].B, wi = B >> 5, sh = B & 31;
    constexpr uint32_t mask = (0x1Fu << i5_off_lo(Q)) | ((0x1Fu << i5_off_hi(Q)) << 16);
    uint32_t win;
    if constexpr (sh == 0) win = w[wi];
    else win = __funnelshift_r(w[wi], wi < 4 ? w[wi + 1] : 0u, sh);
    return win & mask;
}

// One int5 unit (16 rows x 128 K): 28 integer instructions per row make the
// 16 operand pairs, eight MMAs per n-tile sum u * x * 2^-24 over the group, and
// the zero point comes off with the token's group sum X (same units after
// zz = z * 2^-24) before the scale: y += s * (acc - zz * X).
template <int NT, typename GetX>
__device__ __forceinline__ void unit_i5(const Regs<QL_I5Z_G128_F16>& r, GetX getx, bool nt1_live,
                                        const float (&X)[NT][2], float (&yacc)[NT][4]) {
    uint32_t A[2][16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        A[h][0] = i5_pair<0>(r.w[h]);   A[h][1] = i5_pair<1>(r.w[h]);   A[h][2] = i5_pair<2>(r.w[h]);
        A[h][3] = i5_pair<3>(r.w[h]);   A[h][4] = i5_pair<4>(r.w[h]);   A[h][5] = i5_pair<5>(r.w[h]);
        A[h][6] = i5_pair<6>(r.w[h]);   A[h][7] = i5_pair<7>(r.w[h]);   A[h][8] = i5_pair<8>(r.w[h]);
        A[h][9] = i5_pair<9>(r.w[h]);   A[h][10] = i5_pair<10>(r.w[h]); A[h][11] = i5_pair<11>(r.w[h]);
        A[h][12] = i5_pair<12>(r.w[h]); A[h][13] = i5_pair<13>(r.w[h]); A[h][14] = i5_pair<14>(r.w[h]);
        A[h][15] = i5_pair<15>(r.w[h]);
    }
    constexpr int CH = NT == 1 ? 2 : 1;
    float acc[CH][NT][4];
#pragma unroll
    for (int ch = 0; ch < CH; ++ch)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[ch][nt][0] = acc[ch][nt][1] = acc[ch][nt][2] = acc[ch][nt][3] = 0.0f;
#pragma unroll
    for (int p = 0; p < 4; ++p) {  // the lane's 16-byte activation piece p feeds MMAs 2p and 2p + 1
        uint4 xv[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            if (nt == 0 || nt1_live) xv[nt] = getx(nt, p);
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
            const int m = 2 * p + sub;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (nt == 1 && !nt1_live) continue;
                mma_f16(acc[sub % CH][nt], A[0][2 * m], A[1][2 * m], A[0][2 * m + 1], A[1][2 * m + 1],
                        sub == 0 ? xv[nt].x : xv[nt].z, sub == 0 ? xv[nt].y : xv[nt].w);
            }
        }
    }
    fold_chains<CH, NT>(acc);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float t = fmaf(-r.zz[i >> 1], X[nt][i & 1], acc[0][nt][i]);
            yacc[nt][i] = fmaf(r.s[i >> 1], t, yacc[nt][i]);
        }
}

// E4M3 x E4M3 -> fp32 (format 7): the same fragments as the s8 MMA.
__device__ __forceinline__ void mma_e4m3(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// W8A8: exact int32 sums of one group (4 k-steps of m16n8k32).
template <int NT, typename GetX>
__device__ __forceinline__ void unit_w8a8(const Regs<QL_I8A8_G128_BF16>& r, GetX getx, int (&out)[NT][4]) {
    constexpr int CH = NT == 1 ? 2 : 1;
    int acc[CH][NT][4];
#pragma unroll
    for (int ch = 0; ch < CH; ++ch)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[ch][nt][0] = acc[ch][nt][1] = acc[ch][nt][2] = acc[ch][nt][3] = 0;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        uint4 xv[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) xv[nt] = getx(nt, p);
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
            const int s = 2 * p + sub;
            const uint32_t a0 = word_of(r.w[0], 2 * s), a2 = word_of(r.w[0], 2 * s + 1);
            const uint32_t a1 = word_of(r.w[1], 2 * s), a3 = word_of(r.w[1], 2 * s + 1);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint32_t b0 = sub == 0 ? xv[nt].x : xv[nt].z;
                const uint32_t b1 = sub == 0 ? xv[nt].y : xv[nt].w;
                mma_s8(acc[sub % CH][nt], a0, a1, a2, a3, b0, b1);
            }
        }
    }
    fold_chains<CH, NT>(acc);  // integer sums: exact in any order
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) out[nt][i] = acc[0][nt][i];
}

// Format 7: fp32 sums of one group's E4M3 products, the same walk as unit_w8a8.
template <int NT, typename GetX>
__device__ __forceinline__ void unit_e4m3(const Regs<QL_FP8A8_B128_BF16>& r, GetX getx, float (&out)[NT][4]) {
    constexpr int CH = NT == 1 ? 2 : 1;
    float acc[CH][NT][4];
#pragma unroll
    for (int ch = 0; ch < CH; ++ch)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[ch][nt][0] = acc[ch][nt][1] = acc[ch][nt][2] = acc[ch][nt][3] = 0.0f;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        uint4 xv[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) xv[nt] = getx(nt, p);
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
            const int s = 2 * p + sub;
            const uint32_t a0 = word_of(r.w[0], 2 * s), a2 = word_of(r.w[0], 2 * s + 1);
            const uint32_t a1 = word_of(r.w[1], 2 * s), a3 = word_of(r.w[1], 2 * s + 1);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint32_t b0 = sub == 0 ? xv[nt].x : xv[nt].z;
                const uint32_t b1 = sub == 0 ? xv[nt].y : xv[nt].w;
                mma_e4m3(acc[sub % CH][nt], a0, a1, a2, a3, b0, b1);
            }
        }
    }
    fold_chains<CH, NT>(acc);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) out[nt][i] = acc[0][nt][i];
}

__device__ __forceinline__ void mma_bf16(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The bf16 down projection of one unit (16 rows x 64 K): the weights are MMA
// operands as they are; the activation is three bf16 planes whose sum is the
// fp32 value, so the three products summed in fp32 carry its full precision.
// getx(nt, piece, plane) returns the lane's 16-byte piece (chunk c, or 4 + c)
// of a plane.  No scale: the sums go straight into yacc.
template <int NT, typename GetX>
__device__ __forceinline__ void unit_down(const Regs<kFmtDown>& r, GetX getx, bool nt1_live, float (&yacc)[NT][4]) {
#pragma unroll
    for (int piece = 0; piece < 2; ++piece) {
#pragma unroll
        for (int pl = 0; pl < 3; ++pl) {
            uint4 xv[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                if (nt == 0 || nt1_live) xv[nt] = getx(nt, piece, pl);
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
                const int s = 2 * piece + s2;
                const uint32_t a0 = word_of(r.w[0], 2 * s), a2 = word_of(r.w[0], 2 * s + 1);
                const uint32_t a1 = word_of(r.w[1], 2 * s), a3 = word_of(r.w[1], 2 * s + 1);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt == 1 && !nt1_live) continue;
                    mma_bf16(yacc[nt], a0, a1, a2, a3, s2 == 0 ? xv[nt].x : xv[nt].z, s2 == 0 ? xv[nt].y : xv[nt].w);
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Dense skinny GEMM, TMA-fed.
//
// Every warp owns a ring of shared-memory slots (stages_of below), each one or
// two units (16 rows of the packed weight x one 128-K group).  Lane 0 keeps the
// ring's slots in flight with cp.async.bulk.tensor (2-D tile [16 rows][unit
// bytes], zero-filled past row N) completing on a per-slot mbarrier; the whole
// warp waits on the slot, pulls its fragments out of shared memory, computes,
// and refills the slot with the units a ring ahead.  At int8, 16 warps x 2
// slots x 4 KB (or 4 x 2 KB) keep 128 KB of weight in flight per SM without
// holding it in registers.  Waits are bounded: a slot that never fills sets
// QL_DEVERR_TIMEOUT in the device error word and the CTA drains and returns.
//
// Units are numbered (K part, row slab, group within the part): a CTA's
// contiguous range touches at most two K parts, so it stages only those parts
// of the activations.
// ---------------------------------------------------------------------------
constexpr int kStages = QL_SKINNY_STAGES;

template <int FMT>
__host__ __device__ constexpr int unit_row_bytes() {
    return FMT == QL_I4_G64_BF16 ? 64 : (FMT == QL_I5Z_G128_F16 ? 80 : 128);
}
template <int FMT>
__host__ __device__ constexpr int stage_bytes() { return 16 * unit_row_bytes<FMT>(); }
template <int FMT>
__host__ __device__ constexpr int stage_align() {
    return FMT == QL_I4_G64_BF16 ? 512 : (FMT == QL_I5Z_G128_F16 ? 128 : 1024);
}
// Activation staging: bytes per token per group and the row padding that keeps
// the fragment loads conflict-free (see the piece index in tma_getx).
template <int FMT>
__host__ __device__ constexpr int tx_group_bytes() { return act8<FMT>() ? 128 : 256; }
template <int FMT>
__host__ __device__ constexpr int tx_row_pad() {
    return act8<FMT>() ? 64 : (FMT == QL_I5Z_G128_F16 ? 32 : 16);
}

// The nibble formats put UPS = 2 consecutive units of a row slab in one ring
// slot (one barrier): the per-slot waits, refills and bookkeeping then cover
// 2 KB (int4) or 2.5 KB (int5) of weights instead of half that.
// Ring depth, measured per format at 1 to 16 tokens: the int4 and int5 two-unit slots run
// best three deep, the byte formats' two-unit slots (4 KB) two deep, single-unit slots four
// deep but format 7's two.  Deeper rings were slower for every format: more copies in flight
// per SM do not raise the DRAM rate here, they only leave less shared memory to the staged
// activations.
template <int FMT, int UPS = 1>
__host__ __device__ constexpr int stages_of() {
    return UPS == 2 ? ((FMT == QL_I4_G64_BF16 || FMT == QL_I5Z_G128_F16) ? 3 : 2)
                    : (FMT == QL_FP8A8_B128_BF16 ? 2 : kStages);
}
template <int FMT, int UPS = 1>
__host__ __device__ constexpr size_t ring_bytes() {
    return (size_t)kWarps * stages_of<FMT, UPS>() * UPS * stage_bytes<FMT>();
}
// The grouped (MoE) kernel's ring depth.  It reads its activations through L1 (a
// chunk's tokens are scattered rows of the prepared x).  Measured per whole call at
// 1, 8 and 16 tokens, two slots beat three, four and six at every batch size.
constexpr int kMoeStages = 2;
template <int FMT>
__host__ __device__ constexpr size_t moe_ring_bytes() {
    return (size_t)kWarps * kMoeStages * stage_bytes<FMT>();
}

// Shared memory of the dense kernel staging `rows` token rows of XG groups.
// srows: rows of the int4 one-n-tile kernel's staged group sums, [srows][XG][2] fp32.
template <int FMT, int UPS>
__host__ __device__ constexpr size_t tma_smem(int rows, int XG, int srows = 0) {
    return 1024 /* alignment slack */ + ring_bytes<FMT, UPS>() + (size_t)kWarps * stages_of<FMT, UPS>() * 8 + 16 +
           (size_t)rows * ((size_t)XG * tx_group_bytes<FMT>() + tx_row_pad<FMT>()) + (size_t)srows * XG * 8;
}
// int4 with one n-tile offsets its subnormal codes with the tokens' 64-group sums (unit_i4).
template <int FMT, int NT>
__host__ __device__ constexpr bool i4_sums() { return FMT == QL_I4_G64_BF16 && NT == 1; }

// Position in the unit stream: K part, row slab, group within the part.
struct UnitPos {
    int part, slab, gi, gp;  // gp = groups in this part
    __device__ __forceinline__ void init(unsigned u, int slabs, int GP, int G) {
        const unsigned per_full = (unsigned)slabs * GP;
        part = (int)(u / per_full);
        const unsigned rem = u - (unsigned)part * per_full;
        gp = min(GP, G - part * GP);
        slab = (int)(rem / gp);
        gi = (int)(rem % gp);
    }
    __device__ __forceinline__ void next(int slabs, int GP, int G) {
        if (++gi == gp) {
            gi = 0;
            if (++slab == slabs) {
                slab = 0;
                ++part;
                gp = min(GP, G - part * GP);
            }
        }
    }
    __device__ __forceinline__ int grp(int GP) const { return part * GP + gi; }
};

// int4 with two units per ring slot loads the slot as one box of 16 rows x 128 bytes (both
// groups of each row contiguous, 128-byte swizzle) instead of two 64-byte-wide boxes: one copy
// per slot, and whole 128-byte row segments from DRAM.
template <int FMT, int UPS>
__host__ __device__ constexpr bool wide_i4() { return FMT == QL_I4_G64_BF16 && UPS == 2; }

// The lane's int4 fragments of unit ui (0, 1) of a wide slot: its bytes 64 ui .. 64 ui + 63 of
// each 128-byte row, 16-byte chunk j at j ^ (row & 7).  Each quarter-warp's eight 8-byte reads
// hit eight distinct chunks of one 128-byte swizzle row: conflict-free.
__device__ __forceinline__ void read_unit_i4_wide(Regs<QL_I4_G64_BF16>& r, uint32_t slot, int ui, int g, int c) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = g + 8 * h;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int j = 4 * ui + 2 * half + (c >> 1);
            const uint32_t a = slot + row * 128 + ((j ^ (row & 7)) << 4) + 8 * (c & 1);
            asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];\n" : "=r"(r.w[h][half].x), "=r"(r.w[h][half].y) : "r"(a));
        }
    }
}

// The lane's weight fragments of one unit, out of its ring slot.
template <int FMT>
__device__ __forceinline__ void read_unit_smem(Regs<FMT>& r, uint32_t st, int g, int c) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = g + 8 * h;
        if constexpr (FMT == QL_I4_G64_BF16) {
            // 64-byte rows, 64B swizzle: 16-byte chunk j lands at j ^ ((row >> 1) & 3).
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int j = 2 * half + (c >> 1);
                const uint32_t a = st + row * 64 + ((j ^ ((row >> 1) & 3)) << 4) + 8 * (c & 1);
                asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];\n" : "=r"(r.w[h][half].x), "=r"(r.w[h][half].y) : "r"(a));
            }
        } else if constexpr (FMT == QL_I5Z_G128_F16) {
            const uint32_t a = st + row * 80 + 20 * c;
#pragma unroll
            for (int i = 0; i < 5; ++i) asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(r.w[h][i]) : "r"(a + 4 * i));
        } else {
            // 128-byte rows, 128B swizzle: chunk j lands at j ^ (row & 7).  The lane
            // holds chunks c and 4 + c; odd rows read them in the other order so each
            // quarter-warp touches eight distinct 16-byte bank groups.
            const bool odd = (g & 1) != 0;
            const int j0 = odd ? 4 + c : c, j1 = odd ? c : 4 + c;
            const uint4 v0 = lds128(st + row * 128 + ((j0 ^ (row & 7)) << 4));
            const uint4 v1 = lds128(st + row * 128 + ((j1 ^ (row & 7)) << 4));
            r.w[h][0] = odd ? v1 : v0;
            r.w[h][1] = odd ? v0 : v1;
        }
    }
}

#ifdef QL_SKINNY_PROFILE
__device__ unsigned long long g_skinny_prof[148 * 16];
#define QL_PROF(slot)                                                                        \
    if (threadIdx.x == 0 && blockIdx.x < 148)                                                  \
        g_skinny_prof[blockIdx.x * 16 + (slot)] = (slot) == 0 ? global_ns() : clock64() - prof_c0;
#else
#define QL_PROF(slot)
#endif

// Per-unit side data, fetched a ring ahead of use together with the
// weight tile: raw scale bits (converted only when the unit is computed, so
// the loads never stall the issuing loop), int5 zero points, and for W8A8 the
// activation scales of the lane's output tokens (W8A8 and format 7).
template <int FMT, int NT>
struct Side {
    uint32_t sw[2][1];  // weight scale bits [row g / g+8] (int4: both 64-groups' bf16 scales in one word)
    uint32_t z[2];      // int5 zero points
    float sx[NT][2];    // byte activations: scales of tokens 8nt + 2c + {0, 1}; int5, int8 A16: their group sums
};

template <int FMT, int NT>
__device__ __forceinline__ void load_side_x(Side<FMT, NT>& d, const float* sx, int M, int Gtot, int gabs, int c) {
    if constexpr (act8<FMT>() || FMT == QL_I5Z_G128_F16 || i8sub<FMT>()) {  // int5, int8 A16: the group sums
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int t = 8 * nt + 2 * c + i;
                d.sx[nt][i] = (t < M && sx) ? __ldg(sx + (long long)t * Gtot + gabs) : 0.0f;
            }
    }
}

template <int FMT>
__device__ __forceinline__ float scale_value(uint32_t bits) {
    return (FMT == QL_I8_G128_F16 || FMT == QL_I5Z_G128_F16) ? __half2float(__ushort_as_half((unsigned short)bits))
                                                             : __uint_as_float(bits << 16);
}

template <int FMT, int NT>
__device__ __forceinline__ void side_to_regs(Regs<FMT>& r, const Side<FMT, NT>& d) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if constexpr (FMT == QL_I4_G64_BF16) {
            // one n-tile: the unit's sums carry 2^-24 (the subnormal codes), the scale 2^24
            constexpr float k = NT == 1 ? 16777216.0f : 1.0f;
            r.s[h][0] = __uint_as_float(d.sw[h][0] << 16) * k;
            r.s[h][1] = __uint_as_float(d.sw[h][0] & 0xFFFF0000u) * k;
        } else {
            r.s[h] = scale_value<FMT>(d.sw[h][0]);
        }
        if constexpr (FMT == QL_I5Z_G128_F16) r.zz[h] = (float)d.z[h] * 5.9604644775390625e-8f;  // z * 2^-24
    }
}

//
// Slot positions count in slots of UPS units (UPS consecutive groups of one
// slab): G, GP and the unit positions below are in those, the activations'
// staging and the scale indices in groups.  Only the token rows that exist
// are staged; fragments of the others are zeros taken without a load.
template <int FMT, int NT, bool ACC, int UPS>
__global__ void __launch_bounds__(kThreads, 1) k_skinny_tma(const __grid_constant__ SkinnyArgs a) {
    extern __shared__ uint8_t smem_raw[];
#ifdef QL_SKINNY_PROFILE
    const long long prof_c0 = clock64();
    if (threadIdx.x == 0 && blockIdx.x < 148) g_skinny_prof[blockIdx.x * 16 + 15] = 0;
#endif
    QL_PROF(0)
    constexpr int XGB = tx_group_bytes<FMT>();
    constexpr int ST = stages_of<FMT, UPS>();
    constexpr int SB1 = stage_bytes<FMT>();  // one unit
    constexpr int SB = UPS * SB1;             // one ring slot
    constexpr int URB = unit_row_bytes<FMT>();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int G = a.G / UPS, GP = a.GP / UPS, slabs = (a.N + 15) / 16;
    if (lane == 0) asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmap) : "memory");
    const unsigned long long lim = wait_limit(a.err);  // requested first: its latency hides behind the setup

    // Shared memory: [rings][mbarriers][activation barrier][activations], 1024-aligned base.
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const gbase = smem_raw + (base - raw);
    constexpr uint32_t RB = (uint32_t)ring_bytes<FMT, UPS>();
    const uint32_t ring = base + (uint32_t)(warp * ST * SB);
    const uint32_t bars = base + RB + (uint32_t)(warp * ST * 8);
    const uint32_t xbar = base + RB + kWarps * ST * 8;
    const uint32_t xs_off = RB + kWarps * ST * 8 + 16;
    const int R = a.XG * XGB + tx_row_pad<FMT>();
    const uint32_t xs_base = base + xs_off;
    (void)gbase;

    // Work: the CTA's contiguous unit range, split contiguously over its warps
    // (32-bit: the host keeps units * gridDim below 2^31).
    const unsigned units = (unsigned)slabs * G;
    const unsigned cu0 = units * blockIdx.x / gridDim.x, cu1 = units * (blockIdx.x + 1) / gridDim.x;
    const unsigned u0 = cu0 + (cu1 - cu0) * warp / kWarps, u1 = cu0 + (cu1 - cu0) * (warp + 1) / kWarps;

    UnitPos cp;  // slot of units being computed
    if (u0 < u1) cp.init(u0, slabs, GP, G);
    UnitPos ip = cp;  // next slot to issue
    Side<FMT, NT> sd[ST][UPS];
    unsigned issued = u0;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < ST; ++s) mbar_init(bars + 8 * s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncwarp();
    QL_PROF(7)
    // Issues slot s's TMA boxes (UPS consecutive groups of one slab) and fetches their side data.
    // This lane's two scale rows (and int5 zero rows) of the issue side's slab, recomputed only when
    // the slab changes; a row past N reads as scale 0.
    int i_slab = -1;
    const uint16_t* i_srow[2] = {nullptr, nullptr};
    const uint8_t* i_zrow[2] = {nullptr, nullptr};
    auto issue = [&](int s) {
        if (lane == 0) {
            mbar_expect_tx(bars + 8 * s, SB);
            if constexpr (wide_i4<FMT, UPS>()) {
                tma_load_2d(ring + s * SB, &a.tmap, UPS * ip.grp(GP) * URB, ip.slab * 16, bars + 8 * s);
            } else {
#pragma unroll
                for (int i = 0; i < UPS; ++i)
                    tma_load_2d(ring + s * SB + i * SB1, &a.tmap, (UPS * ip.grp(GP) + i) * URB, ip.slab * 16,
                                bars + 8 * s);
            }
        }
        if (ip.slab != i_slab) {
            i_slab = ip.slab;
            const uint16_t* const sc = static_cast<const uint16_t*>(a.scales);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int n = ip.slab * 16 + g + 8 * h;
                const bool ok = n < a.N && sc;
                const long long row = block_scaled<FMT>() ? (long long)(n >> 7) * a.Gtot
                                      : FMT == QL_I4_G64_BF16 ? (long long)n * (2 * a.Gtot)
                                                               : (long long)n * a.Gtot;
                i_srow[h] = ok ? sc + row : nullptr;
                if constexpr (FMT == QL_I5Z_G128_F16) i_zrow[h] = ok ? a.zeros + (long long)n * a.Gtot : nullptr;
            }
        }
#pragma unroll
        for (int i = 0; i < UPS; ++i) {
            const int gabs = a.g0 + UPS * ip.grp(GP) + i;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if constexpr (FMT == QL_I4_G64_BF16)  // the unit's two bf16 scales, adjacent: one 32-bit load
                    sd[s][i].sw[h][0] = i_srow[h] ? __ldg(reinterpret_cast<const uint32_t*>(i_srow[h] + 2 * gabs)) : 0u;
                else
                    sd[s][i].sw[h][0] = i_srow[h] ? (uint32_t)__ldg(i_srow[h] + gabs) : 0u;
                if constexpr (FMT == QL_I5Z_G128_F16) sd[s][i].z[h] = i_zrow[h] ? __ldg(i_zrow[h] + gabs) : 0u;
            }
        }
    };
    // Start the weight stream first: it never depends on the kernel before.
#pragma unroll
    for (int s = 0; s < ST; ++s) {
        if (issued < u1) {
            issue(s);
            ip.next(slabs, GP, G);
            ++issued;
        }
    }
    QL_PROF(8)

    // The activations (and the zeroed y) come from the kernel launched just
    // before this one: wait for it (a no-op without a programmatic dependency).
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    QL_PROF(2)

    // Stage the activations of the K parts this CTA touches, one bulk copy per
    // token row, while the weight stream runs (groups gs0 .. gs0 + ngs).
    int gs0 = 0, ngs = 0;
    if (cu1 > cu0) {
        UnitPos p0, p1;
        p0.init(cu0, slabs, GP, G);
        p1.init(cu1 - 1, slabs, GP, G);
        gs0 = p0.part * GP * UPS;
        ngs = min(G, (p1.part + 1) * GP) * UPS - gs0;
    }
    const int rows_x = ngs > 0 ? min(a.M, NT * 8) : 0;
    // Lanes whose token row does not exist read a row of zeros staged after the real ones, so
    // the fragment loads need no test.
    uint32_t xrow_off[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) xrow_off[nt] = (uint32_t)((8 * nt + g < rows_x ? 8 * nt + g : rows_x) * R);
    // int4, one n-tile: the group-sum rows of this lane's accumulator columns (tokens 2 c + i)
    uint32_t srow_off[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) srow_off[i] = (uint32_t)(8 * (2 * c + i < rows_x ? 2 * c + i : 0) * a.XG);
    if (rows_x < NT * 8) {
        const int pieces = ngs * XGB / 16;
        for (int i = threadIdx.x; i < pieces; i += kThreads)
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(xs_base + (uint32_t)(rows_x * R + 16 * i)),
                         "r"(0u)
                         : "memory");
    }
    if (threadIdx.x == 0) {
        mbar_init(xbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        if (rows_x > 0) {
            const unsigned row_bytes = (unsigned)(ngs * XGB);
            mbar_expect_tx(xbar, row_bytes * rows_x);
            const uint8_t* xsrc = static_cast<const uint8_t*>(a.xs);
            const long long ldx_b = a.ldx * (act8<FMT>() ? 1 : 2);
            for (int t = 0; t < rows_x; ++t)
                bulk_load(xs_base + (uint32_t)(t * R), xsrc + t * ldx_b + (long long)gs0 * XGB, row_bytes, xbar);
        }
    }
    // int4, one n-tile: the staged tokens' sums over each 64-group, [token][group][half], after
    // the activation rows (a lane whose token is absent reads token 0's: its column is never stored).
    const uint32_t xsum_s = xs_base + (uint32_t)((a.M < NT * 8 ? a.M + 1 : NT * 8) * R);
    if constexpr (i4_sums<FMT, NT>()) {
        const int per_row = 2 * ngs;
        for (int i = threadIdx.x; i < rows_x * per_row; i += kThreads) {
            const int t = i / per_row, j = i - t * per_row;
            const float v = __ldg(a.xsum + (long long)t * 2 * a.Gtot + 2 * (a.g0 + gs0) + j);
            asm volatile("st.shared.f32 [%0], %1;\n" ::"r"(xsum_s + (uint32_t)(8 * (t * a.XG) + 4 * j)), "f"(v)
                         : "memory");
        }
    }
    // Per-token side data of the units already in flight: the activation scales (byte
    // activations) or the group sums (int5), written by the kernel before this one.
    const float* const xside = (FMT == QL_I5Z_G128_F16 || i8sub<FMT>()) ? a.xsum : a.xf;
    if constexpr (act8<FMT>() || FMT == QL_I5Z_G128_F16 || i8sub<FMT>()) {
        UnitPos q = cp;
#pragma unroll
        for (int s = 0; s < ST; ++s) {
            if (u0 + s < issued)
#pragma unroll
                for (int i = 0; i < UPS; ++i)
                    load_side_x<FMT, NT>(sd[s][i], xside, a.M, a.Gtot, a.g0 + UPS * q.grp(GP) + i, c);
            q.next(slabs, GP, G);
        }
    }
    QL_PROF(4)
    __syncthreads();
    QL_PROF(5)
    if (u0 >= u1) return;
    bool timed_out = rows_x > 0 && !__all_sync(kFull, mbar_wait(xbar, 0, lim));
    QL_PROF(1)

    const bool nt1_live = NT > 1 && a.M > 8;
    float yacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) yacc[nt][0] = yacc[nt][1] = yacc[nt][2] = yacc[nt][3] = 0.0f;
    int cur_key = cp.part * slabs + cp.slab;

    auto flush = [&](int key) {
        const int slab = key % slabs;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = 8 * nt + 2 * c + (i & 1);
                const int n = slab * 16 + g + 8 * (i >> 1);
                if (t < a.M && n < a.N) {
                    const float f = act8<FMT>() ? 1.0f : __ldg(a.xf + t);
                    atomicAdd(a.y + (long long)t * a.ldy + n, yacc[nt][i] * f);
                }
                yacc[nt][i] = 0.0f;
            }
    };

    unsigned phase = 0;
    unsigned u = u0;
    while (u < u1 && !timed_out) {
#pragma unroll
        for (int s = 0; s < ST; ++s) {
            if (u >= u1) break;
            const int key = cp.part * slabs + cp.slab;
            if (!ACC && key != cur_key) {
                flush(cur_key);
                cur_key = key;
            }
            if (!__all_sync(kFull, mbar_wait(bars + 8 * s, phase, lim))) {  // the warp gives up together
                timed_out = true;
                break;
            }
#pragma unroll
            for (int ui = 0; ui < UPS; ++ui) {
                Regs<FMT> r;
                side_to_regs<FMT, NT>(r, sd[s][ui]);
                if constexpr (wide_i4<FMT, UPS>())
                    read_unit_i4_wide(r, ring + s * SB, ui, g, c);
                else
                    read_unit_smem<FMT>(r, ring + s * SB + ui * SB1, g, c);
                const int grp = UPS * cp.grp(GP) + ui;
                const int lg = grp - gs0;  // group index in the staged activations
                auto getx = [&](int nt, int p) -> uint4 {
                    int j;
                    if constexpr (act8<FMT>())
                        j = lg * 8 + 4 * p + c;
                    else if constexpr (FMT == QL_I4_G64_BF16)
                        j = lg * 16 + (p & 8) + 2 * c + (p & 1);
                    else if constexpr (FMT == QL_I5Z_G128_F16) {
                        j = lg * 16 + 4 * c + p;
                        j ^= (j >> 3) & 1;
                    } else
                        j = lg * 16 + (p >> 1) * 8 + 2 * c + (p & 1);
                    return lds128(xs_base + xrow_off[nt] + (uint32_t)(16 * j));
                };
                if constexpr (FMT == QL_I8A8_G128_BF16) {
                    int acc[NT][4];
                    unit_w8a8<NT>(r, getx, acc);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int t = 8 * nt + 2 * c + (i & 1);
                            const int n = cp.slab * 16 + g + 8 * (i >> 1);
                            if (ACC) {
                                if (t < a.M && n < a.N)
                                    a.acc[((long long)t * a.N + n) * a.Gtot + a.g0 + grp] = acc[nt][i];
                            } else {
                                // |acc| <= 128 * 127^2 < 2^22: the magic-number conversion is exact.
                                const float fa = __int_as_float(0x4B400000 + acc[nt][i]) - 12582912.0f;
                                yacc[nt][i] = fmaf(r.s[i >> 1] * sd[s][ui].sx[nt][i & 1], fa, yacc[nt][i]);
                            }
                        }
                } else if constexpr (FMT == QL_FP8A8_B128_BF16) {
                    float acc[NT][4];
                    unit_e4m3<NT>(r, getx, acc);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            yacc[nt][i] = fmaf(r.s[i >> 1] * sd[s][ui].sx[nt][i & 1], acc[nt][i], yacc[nt][i]);
                } else if constexpr (FMT == QL_I5Z_G128_F16) {
                    unit_i5<NT>(r, getx, nt1_live, sd[s][ui].sx, yacc);
                } else if constexpr (FMT == QL_I4_G64_BF16) {
                    float X[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    if constexpr (i4_sums<FMT, NT>()) {
#pragma unroll
                        for (int i = 0; i < 2; ++i)
                            asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];\n"
                                         : "=f"(X[2 * i]), "=f"(X[2 * i + 1])
                                         : "r"(xsum_s + srow_off[i] + (uint32_t)(8 * lg)));
                    }
                    unit_i4<NT>(r, getx, nt1_live, X, yacc);
                } else {
                    unit_a16<FMT, NT>(r, getx, nt1_live, sd[s][ui].sx, yacc);
                }
            }
            __syncwarp();
            if (issued < u1) {  // refill this slot with the units ST slots ahead
                issue(s);
#pragma unroll
                for (int i = 0; i < UPS; ++i)
                    load_side_x<FMT, NT>(sd[s][i], xside, a.M, a.Gtot, a.g0 + UPS * ip.grp(GP) + i, c);
                ip.next(slabs, GP, G);
                ++issued;
            }
            cp.next(slabs, GP, G);
            ++u;
        }
        phase ^= 1u;
    }
    if (timed_out) {
        if (lane == 0) atomicOr(a.err, (unsigned)QL_DEVERR_TIMEOUT);
        if (rows_x > 0) mbar_wait(xbar, 0);
        // Let the copies still in flight land before the CTA's memory is released.
        for (unsigned v = u; v < issued; ++v) {
            const int s = (int)((v - u0) % ST);
            const unsigned ph = ((v - u0) / ST) & 1u;
            if (!mbar_wait(bars + 8 * s, ph)) break;
        }
        return;
    }
    if (!ACC) flush(cur_key);
#ifdef QL_SKINNY_PROFILE
    if (lane == 0 && blockIdx.x < 148) atomicMax(&g_skinny_prof[blockIdx.x * 16 + 15], (unsigned long long)(clock64() - prof_c0));
    if (threadIdx.x == 0 && blockIdx.x < 148) g_skinny_prof[blockIdx.x * 16 + 6] = clock64() - prof_c0;
#endif
}

// Grouped (MoE) skinny GEMM: units are (row chunk of one expert, slab, group),
// in that order.  Every warp streams its contiguous unit range through its own
// ring of TMA copies, as the dense kernel does, from one tensor map over the
// stacked experts' codes [E * N][K] (a unit is the box at row expert * N +
// 16 * slab, byte 128 * group).  The activations of a chunk's (at most 16)
// tokens are read from the prepared [T, K] buffer, which stays in L2, and the
// results are added into y[(t, j), :] (zeroed by the prologue).
//
// Small batches (T * topk <= kMoeFusedMaxPairs) skip the permute kernel: every
// CTA ranks the routing ids itself in shared memory -- the position of pair i
// is the number of valid ids below its expert plus the number of equal ids
// before it, which is the stable (expert, t, j) order -- and cuts each expert's
// segment into chunks of 16.  It then starts its weight stream at once and
// waits for the activation prologue (programmatic dependent launch) only before
// it reads the activations or adds into y.
//
// With FMT == kFmtDown the same walk runs the experts' bf16 down projection:
// K is the intermediate size (units of 64 bf16), xs the activation of every
// pair as three bf16 planes [pairs][3][K], and each chunk row, a pair (t, j),
// is added into y[t][:] (zeroed by the prologue) scaled by its routing weight.
template <int FMT, int NT>
__global__ void __launch_bounds__(kThreads, 1) k_moe_tma(const __grid_constant__ MoeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    constexpr bool DOWN = FMT == kFmtDown;
    constexpr int SB = stage_bytes<FMT>();
    const unsigned long long lim = wait_limit(a.err);  // requested first: its latency hides behind the setup
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int G = DOWN ? a.K / 64 : a.K / 128;
    const int slabs = (a.N + 15) / 16;
    const long long per_chunk = (long long)slabs * G;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const bool fused = a.ids != nullptr;
    constexpr int CR = 8 * NT;  // rows per chunk of the fused mode: one or two n-tiles
    // Routing state of the fused mode, after the rings and barriers.
    int* const s_ids = reinterpret_cast<int*>(smem_raw + (base - raw) + moe_ring_bytes<FMT>() + kWarps * kMoeStages * 8);
    int* const s_perm = s_ids + kMoeFusedMaxPairs;   // permuted position -> pair index t * topk + j
    int* const s_bef = s_perm + kMoeFusedMaxPairs;   // per position: pairs of the same expert before it
    int* const s_cnt = s_bef + kMoeFusedMaxPairs;    // per position: pairs of its expert
    int* const s_exp = s_cnt + kMoeFusedMaxPairs;    // per position: its expert
    MoeChunk* const s_ch = reinterpret_cast<MoeChunk*>(s_exp + kMoeFusedMaxPairs);
    int* const s_nch = reinterpret_cast<int*>(s_ch + kMoeFusedMaxPairs);
    long long nch;
    if (fused) {
        // The ids are complete: the activation prologue this grid depends on is an
        // ordinary launch, so it started only after all earlier work on the stream
        // (the router included), and this grid starts no earlier than it.
        const int P = a.T * a.topk;
        for (int i = threadIdx.x; i < P; i += kThreads) s_ids[i] = a.ids[i];
        __syncthreads();
        for (int i = threadIdx.x; i < P; i += kThreads) {
            const int e = s_ids[i];
            int less = 0, before = 0, same = 0;
            for (int j = 0; j < P; ++j) {
                const int f = s_ids[j];
                less += f >= 0 && f < e;
                same += f == e;
                before += f == e && j < i;
            }
            if (e < 0 || e >= a.E) {  // routed to no expert: flagged, its output row stays zero
                if (blockIdx.x == 0) atomicOr(a.err, (unsigned)QL_DEVERR_EXPERT_ID);
                continue;
            }
            const int pos = less + before;
            s_perm[pos] = i;
            s_bef[pos] = before;
            s_cnt[pos] = same;
            s_exp[pos] = e;
        }
        __syncthreads();
        int nv = 0;  // valid pairs: positions 0 .. nv - 1
        for (int j = 0; j < P; ++j) nv += s_ids[j] >= 0 && s_ids[j] < a.E;
        for (int p = threadIdx.x; p < nv; p += kThreads) {
            if (s_bef[p] % CR) continue;  // a chunk starts at every CR-th row of an expert's segment
            int idx = 0;
            for (int q = 0; q < p; ++q) idx += s_bef[q] % CR == 0;
            s_ch[idx] = MoeChunk{s_exp[p], p, min(CR, s_cnt[p] - s_bef[p])};
        }
        if (threadIdx.x == 0) {
            int n = 0;
            for (int q = 0; q < nv; ++q) n += s_bef[q] % CR == 0;
            *s_nch = n;
        }
        __syncthreads();
        nch = *s_nch;
    } else {
        asm volatile("griddepcontrol.wait;\n" ::: "memory");  // the chunk table comes from the permute kernel
        nch = min((long long)*a.n_chunks, a.max_chunks);
    }
    const MoeChunk* const chunks = fused ? s_ch : a.chunks;
    const int* const perm = fused ? s_perm : a.perm;
    const long long units = nch * per_chunk;
    const long long wid = (long long)blockIdx.x * kWarps + warp, nw = (long long)gridDim.x * kWarps;
    const long long u0 = units * wid / nw, u1 = units * (wid + 1) / nw;
    if (lane == 0) asm volatile("prefetch.tensormap [%0];\n" ::"l"(&a.tmap) : "memory");

    const uint32_t ring = base + (uint32_t)(warp * kMoeStages * SB);
    const uint32_t bars = base + (uint32_t)moe_ring_bytes<FMT>() + (uint32_t)(warp * kMoeStages * 8);
    if (u0 >= u1) return;
    const long long expert_scales = block_scaled<FMT>() ? (long long)((a.N + 127) / 128) * G : (long long)a.N * G;
    const uint16_t* const sc0 = static_cast<const uint16_t*>(a.scales);

    // Unit position, stepped without divisions: chunk, slab, group.
    struct Pos {
        int ch, slab, grp;
        __device__ void next(int slabs, int G) {
            if (++grp == G) {
                grp = 0;
                if (++slab == slabs) {
                    slab = 0;
                    ++ch;
                }
            }
        }
    };
    Pos cp;
    cp.ch = (int)(u0 / per_chunk);
    cp.slab = (int)((u0 % per_chunk) / G);
    cp.grp = (int)(u0 % G);
    Pos ip = cp;
    Side<FMT, NT> sd[kMoeStages];
    long long issued = u0;
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < kMoeStages; ++st) mbar_init(bars + 8 * st, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncwarp();
    // The issue side's (chunk, slab): its weight row in the stacked experts and this lane's two
    // scale rows, recomputed only when the slab changes (every G units).
    int i_ch = -1, i_slab = -1, i_wrow = 0;
    const uint16_t* i_srow[2] = {nullptr, nullptr};
    auto issue = [&](int st) {
        if (ip.ch != i_ch || ip.slab != i_slab) {
            i_ch = ip.ch;
            i_slab = ip.slab;
            const MoeChunk ch = chunks[ip.ch];
            i_wrow = ch.expert * a.N + ip.slab * 16;
            if constexpr (!DOWN) {
                const uint16_t* const se = sc0 + (long long)ch.expert * expert_scales;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int n = ip.slab * 16 + g + 8 * h;
                    i_srow[h] = n < a.N ? se + (long long)(block_scaled<FMT>() ? (n >> 7) : n) * G : nullptr;
                }
            }
        }
        if (lane == 0) {
            mbar_expect_tx(bars + 8 * st, SB);
            tma_load_2d(ring + st * SB, &a.tmap, ip.grp * 128, i_wrow, bars + 8 * st);
        }
        if constexpr (!DOWN) {
#pragma unroll
            for (int h = 0; h < 2; ++h) sd[st].sw[h][0] = i_srow[h] ? (uint32_t)__ldg(i_srow[h] + ip.grp) : 0u;
        }
        ip.next(slabs, G);
        ++issued;
    };
#pragma unroll
    for (int st = 0; st < kMoeStages; ++st)
        if (issued < u1) issue(st);

    float yacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) yacc[nt][0] = yacc[nt][1] = yacc[nt][2] = yacc[nt][3] = 0.0f;
    // The weight stream is running; the activations and the zeroed y come from the prologue.
    if (fused) asm volatile("griddepcontrol.wait;\n" ::: "memory");
    MoeChunk chc = chunks[cp.ch];  // the chunk being computed
    // This lane's activation row per n-tile (the MMA's B column it loads), as a byte pointer.  A
    // lane past the chunk's rows loads the chunk's first row instead: its MMA column is computed
    // and never stored, so no test sits in the fragment loads.
    const uint8_t* xrow[NT];
    const float* xsr[NT][2];  // int8 codes: the group-sum rows of this lane's accumulator columns (null: none)
    int ctok[NT][2];                 // format 7: the tokens of this lane's accumulator columns
    auto load_tokens = [&]() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int slot = 8 * nt + g;  // (the down projection's activations are per pair)
            const int tk = perm[chc.start + (slot < chc.count ? slot : 0)] / (DOWN ? 1 : a.topk);
            // row bytes: E4M3 codes K, f16 K * 2, the down projection's three bf16 planes K * 6
            xrow[nt] = static_cast<const uint8_t*>(a.xs) + (long long)tk * a.K * (DOWN ? 6 : act8<FMT>() ? 1 : 2);
            if constexpr (act8<FMT>()) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int cs = 8 * nt + 2 * c + i;
                    ctok[nt][i] = cs < chc.count ? perm[chc.start + cs] / a.topk : -1;
                }
            }
            if constexpr (i8sub<FMT>()) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int cs = 8 * nt + 2 * c + i;
                    xsr[nt][i] = cs < chc.count ? a.xsum + (long long)(perm[chc.start + cs] / a.topk) * G : nullptr;
                }
            }
        }
    };
    load_tokens();
    int cur_ch = cp.ch, cur_slab = cp.slab;

    auto flush = [&]() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int slot = 8 * nt + 2 * c + (i & 1);
                const int n = cur_slab * 16 + g + 8 * (i >> 1);
                if (slot < chc.count && n < a.N) {
                    const int pair = perm[chc.start + slot];
                    if constexpr (DOWN) {  // the routing-weighted sum over the token's slots
                        atomicAdd(a.y + (long long)(pair / a.topk) * a.N + n, yacc[nt][i] * __ldg(a.wts + pair));
                    } else {
                        const float f = act8<FMT>() ? 1.0f : __ldg(a.xf + pair / a.topk);
                        atomicAdd(a.y + (long long)pair * a.N + n, yacc[nt][i] * f);
                    }
                }
                yacc[nt][i] = 0.0f;
            }
    };

    bool timed_out = false;
    unsigned phase = 0;
    long long u = u0;
    while (u < u1 && !timed_out) {
#pragma unroll
        for (int st = 0; st < kMoeStages; ++st) {
            if (u >= u1) break;
            if (cp.ch != cur_ch || cp.slab != cur_slab) {
                flush();
                if (cp.ch != cur_ch) {
                    chc = chunks[cp.ch];
                    load_tokens();
                }
                cur_ch = cp.ch;
                cur_slab = cp.slab;
            }
            if (!__all_sync(kFull, mbar_wait(bars + 8 * st, phase, lim))) {  // the warp gives up together
                timed_out = true;
                break;
            }
            Regs<FMT> r;
            if constexpr (!DOWN) side_to_regs<FMT, NT>(r, sd[st]);
            read_unit_smem<FMT>(r, ring + st * SB, g, c);
            const int grp = cp.grp;
            // The fragments read_unit_smem hands out pair with these 16-byte x pieces of the group
            // (the same order as the dense kernel's staged activations).
            auto getx = [&](int nt, int p) -> uint4 {
                if constexpr (act8<FMT>()) {  // E4M3 codes: the dense kernel's piece order, 16 B each
                    const int j = 4 * p + c;
                    return __ldg(reinterpret_cast<const uint4*>(xrow[nt] + grp * 128 + 16 * j));
                } else {
                    const int j = (p >> 1) * 8 + 2 * c + (p & 1);
                    return __ldg(reinterpret_cast<const uint4*>(xrow[nt] + grp * 256 + 16 * j));
                }
            };
            if constexpr (DOWN) {
                auto getx3 = [&](int nt, int piece, int pl) -> uint4 {
                    return __ldg(reinterpret_cast<const uint4*>(xrow[nt] + ((long long)pl * a.K + grp * 64) * 2 +
                                                                16 * (piece ? 4 + c : c)));
                };
                unit_down<NT>(r, getx3, chc.count > 8, yacc);
            } else if constexpr (act8<FMT>()) {
                // fp32 sums of the group's E4M3 products, then both scales: the block's weight
                // scale and the scale of the column's token for this group.
                float acc[NT][4];
                unit_e4m3<NT>(r, getx, acc);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const float sx = ctok[nt][i] >= 0 ? __ldg(a.xf + (long long)ctok[nt][i] * G + grp) : 0.0f;
                        yacc[nt][i] = fmaf(r.s[0] * sx, acc[nt][i], yacc[nt][i]);
                        yacc[nt][2 + i] = fmaf(r.s[1] * sx, acc[nt][2 + i], yacc[nt][2 + i]);
                    }
            } else {
                float X[NT][2];  // int8 codes: the column tokens' sums of this group's activations
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 2; ++i) X[nt][i] = i8sub<FMT>() && xsr[nt][i] ? __ldg(xsr[nt][i] + grp) : 0.0f;
                unit_a16<FMT, NT>(r, getx, chc.count > 8, X, yacc);
            }
            __syncwarp();
            if (issued < u1) issue(st);  // refill this slot with the unit kMoeStages ahead
            cp.next(slabs, G);
            ++u;
        }
        phase ^= 1u;
    }
    if (timed_out) {
        if (lane == 0) atomicOr(a.err, (unsigned)QL_DEVERR_TIMEOUT);
        // Let the copies still in flight land before the CTA's memory is released.
        for (long long v = u; v < issued; ++v) {
            const int st = (int)((v - u0) % kMoeStages);
            const unsigned ph = (unsigned)(((v - u0) / kMoeStages) & 1);
            if (!mbar_wait(bars + 8 * st, ph)) break;
        }
        return;
    }
    flush();
}

// ---- host side of the dense kernel -------------------------------------------------

template <int FMT>
int swizzle_mode() {
    return FMT == QL_I4_G64_BF16 ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : (FMT == QL_I5Z_G128_F16 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B);
}

// Groups of activations one CTA can stage for `rows` tokens (and `srows` rows of group sums)
// next to its rings.
template <int FMT, int UPS = 1>
int max_staged_groups(int rows, size_t smem_optin, int srows = 0) {
    for (int xg = 256; xg >= 1; --xg)
        if (tma_smem<FMT, UPS>(rows, xg, srows) <= smem_optin) return xg;
    return 0;
}

// Largest K-part size GP whose parts, as the CTAs' contiguous unit ranges cut
// them, never need more than XG staged groups in one CTA.
int plan_parts(int G, int slabs, int ctas, int XG) {
    for (int GP = G; GP >= 1; --GP) {
        const long long units = (long long)slabs * G, per = (long long)slabs * GP;
        int worst = 0;
        for (int b = 0; b < ctas; ++b) {
            const long long cu0 = units * b / ctas, cu1 = units * (b + 1) / ctas;
            if (cu1 <= cu0) continue;
            const long long p0 = cu0 / per, p1 = (cu1 - 1) / per;
            const int ngs = (int)(std::min<long long>(G, (p1 + 1) * GP) - p0 * GP);
            worst = std::max(worst, ngs);
        }
        if (worst <= XG) return GP;
    }
    return 0;
}

template <int FMT, int NT, bool ACC, int UPS = 1>
cudaError_t run_skinny(const SkinnyArgs& in, cudaStream_t s, const DeviceInfo& di) {
    SkinnyArgs a = in;
    if (a.G % UPS) return cudaErrorInvalidValue;
    // token rows staged, plus one row of zeros for the lanes of absent tokens
    const int rows = a.M < NT * 8 ? a.M + 1 : NT * 8;
    const int srows = i4_sums<FMT, NT>() ? std::min(a.M, NT * 8) : 0;
    const int XG = max_staged_groups<FMT, UPS>(rows, di.smem_optin, srows);
    if (XG < UPS) return cudaErrorInvalidValue;
    a.XG = XG;
    // K parts in whole slots, so a slot never straddles two parts
    a.GP = UPS * plan_parts(a.G / UPS, (a.N + 15) / 16, di.sm_count, XG / UPS);
    if (a.GP < 1) return cudaErrorInvalidValue;
    if ((long long)((a.N + 15) / 16) * a.G * (di.sm_count + 1) >= (1LL << 31)) return cudaErrorInvalidValue;
    a.err = di.err_word;
    constexpr bool wide = wide_i4<FMT, UPS>();
    cudaError_t e = make_tmap_2d(a.W, a.N, (long long)a.G * unit_row_bytes<FMT>(), a.ldw,
                                 wide ? 2 * unit_row_bytes<FMT>() : unit_row_bytes<FMT>(), 16,
                                 wide ? (int)CU_TENSOR_MAP_SWIZZLE_128B : swizzle_mode<FMT>(), &a.tmap);
    if (e != cudaSuccess) return e;
    const size_t smem = tma_smem<FMT, UPS>(rows, XG, srows);
    static bool attr_set[64] = {};  // per device ordinal
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(k_skinny_tma<FMT, NT, ACC, UPS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)di.smem_optin);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k_skinny_tma<FMT, NT, ACC, UPS>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[dev] = true;
    }
    // Programmatic dependent launch: the kernel may start while the kernel before
    // it (the activation prologue) finishes; it waits for it before touching x.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(di.sm_count);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = a.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_skinny_tma<FMT, NT, ACC, UPS>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int FMT>
cudaError_t run_skinny_fmt(const SkinnyArgs& a, cudaStream_t s, const DeviceInfo& di) {
    // Two units per ring slot up to 8 tokens, for every format (int8 and fp8: 4 KB slots two
    // deep, the same 128 KB ring per SM as one-unit slots four deep, with half the waits,
    // refills and bookkeeping).  With 16 tokens the nibble formats' doubled ring leaves room
    // for fewer staged activation groups, K splits into more parts, and that costs more than
    // the slots save.
    if (a.G % 2 == 0 && a.M <= 8) return run_skinny<FMT, 1, false, 2>(a, s, di);
    // Two n-tiles: two-unit slots measured faster for the fp8 codes only (FP8 3%, format 7 7% at
    // 16 tokens); the int8 formats ran slower with them (W8A8 spills at that register count).
    if constexpr (FMT == QL_FP8_B128_BF16 || FMT == QL_FP8A8_B128_BF16)
        if (a.G % 2 == 0 && a.M > 8) return run_skinny<FMT, 2, false, 2>(a, s, di);
    if (a.M > 8) return run_skinny<FMT, 2, false>(a, s, di);
    return run_skinny<FMT, 1, false>(a, s, di);
}

}  // namespace

int skinny_max_k(int fmt) {
    DeviceInfo di;
    if (device_info(&di) != cudaSuccess) return 0;
    int xg = 0;
    switch (fmt) {
    case QL_I8A8_G128_BF16:
    case QL_FP8A8_B128_BF16: xg = max_staged_groups<QL_I8A8_G128_BF16>(16, di.smem_optin); break;
    case QL_I4_G64_BF16: xg = max_staged_groups<QL_I4_G64_BF16, 2>(16, di.smem_optin); break;
    case QL_I5Z_G128_F16: xg = max_staged_groups<QL_I5Z_G128_F16, 2>(16, di.smem_optin); break;
    default: xg = max_staged_groups<QL_I8_G128_BF16>(16, di.smem_optin); break;
    }
    return xg * 128;  // with G <= XG a single part always fits
}

#ifdef QL_SKINNY_PROFILE
__global__ void k_empty_bigsmem() { extern __shared__ uint8_t sm[]; if (threadIdx.x == 9999) sm[0] = 1; }
extern "C" int ql_prof_empty_launch(void* stream) {
    DeviceInfo di;
    device_info(&di);
    cudaFuncSetAttribute(k_empty_bigsmem, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)di.smem_optin);
    k_empty_bigsmem<<<di.sm_count, kThreads, di.smem_optin - 1024, (cudaStream_t)stream>>>();
    return cudaGetLastError() == cudaSuccess ? 0 : 5;
}
extern "C" int ql_skinny_prof_read(unsigned long long* out, int n) {
    return cudaMemcpyFromSymbol(out, g_skinny_prof, sizeof(unsigned long long) * n) == cudaSuccess ? 0 : 5;
}
#endif

cudaError_t launch_skinny(int fmt, const SkinnyArgs& a, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    if (a.acc) {
        if (fmt != QL_I8A8_G128_BF16) return cudaErrorInvalidValue;
        if (a.M > 8) return run_skinny<QL_I8A8_G128_BF16, 2, true, 1>(a, s, di);
        return run_skinny<QL_I8A8_G128_BF16, 1, true, 1>(a, s, di);
    }
    switch (fmt) {
    case QL_I8_G128_BF16: return run_skinny_fmt<QL_I8_G128_BF16>(a, s, di);
    case QL_I8_G128_F16: return run_skinny_fmt<QL_I8_G128_F16>(a, s, di);
    case QL_I8A8_G128_BF16: return run_skinny_fmt<QL_I8A8_G128_BF16>(a, s, di);
    case QL_I4_G64_BF16: return run_skinny_fmt<QL_I4_G64_BF16>(a, s, di);
    case QL_I5Z_G128_F16: return run_skinny_fmt<QL_I5Z_G128_F16>(a, s, di);
    case QL_FP8_B128_BF16: return run_skinny_fmt<QL_FP8_B128_BF16>(a, s, di);
    case QL_FP8A8_B128_BF16: return run_skinny_fmt<QL_FP8A8_B128_BF16>(a, s, di);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_moe_down(const MoeArgs& in, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    MoeArgs a = in;
    a.err = di.err_word;
    // the stacked bf16 weights as bytes: [E * N rows][2 K bytes], units of 16 rows x 128 B
    if ((e = make_tmap_2d(a.codes, (long long)a.E * a.N, 2LL * a.K, 2LL * a.K, 128, 16, CU_TENSOR_MAP_SWIZZLE_128B,
                          &a.tmap)) != cudaSuccess)
        return e;
    const size_t smem = 1024 + moe_ring_bytes<kFmtDown>() + (size_t)kWarps * kMoeStages * 8 +
                        (5 * sizeof(int) + sizeof(MoeChunk)) * kMoeFusedMaxPairs + 16;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        for (auto kern : {k_moe_tma<kFmtDown, 1>, k_moe_tma<kFmtDown, 2>})
            if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
                return e;
        if (dev < 64) attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(di.sm_count);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = a.ids ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // the fused mode cuts its own chunks at 8 rows (one n-tile); the permute's chunks hold up to 16
    e = a.ids ? cudaLaunchKernelEx(&cfg, k_moe_tma<kFmtDown, 1>, a) : cudaLaunchKernelEx(&cfg, k_moe_tma<kFmtDown, 2>, a);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_moe_skinny(const MoeArgs& in, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    MoeArgs a = in;
    a.err = di.err_word;
    if ((e = make_tmap_2d(a.codes, (long long)a.E * a.N, a.K, a.K, 128, 16, CU_TENSOR_MAP_SWIZZLE_128B, &a.tmap)) !=
        cudaSuccess)
        return e;
    // rings, their mbarriers, and the routing state of the fused small-batch mode
    const size_t smem = 1024 + moe_ring_bytes<QL_I8_G128_BF16>() + (size_t)kWarps * kMoeStages * 8 +
                        (5 * sizeof(int) + sizeof(MoeChunk)) * kMoeFusedMaxPairs + 16;
    static bool attr_set[64] = {};  // per device ordinal, for all four instantiations at once
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        for (auto kern : {k_moe_tma<QL_I8_G128_BF16, 2>, k_moe_tma<QL_I8_G128_F16, 2>, k_moe_tma<QL_FP8_B128_BF16, 2>,
                          k_moe_tma<QL_FP8A8_B128_BF16, 2>, k_moe_tma<QL_I8_G128_BF16, 1>, k_moe_tma<QL_I8_G128_F16, 1>,
                          k_moe_tma<QL_FP8_B128_BF16, 1>, k_moe_tma<QL_FP8A8_B128_BF16, 1>}) {
            if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
                return e;
        }
        if (dev < 64) attr_set[dev] = true;
    }
    auto run = [&](auto kern) -> cudaError_t {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(di.sm_count);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        // With the permute kernel before it everything depends on its table; in the
        // fused mode only the activations and y do, so the weight stream may start early.
        attr[0].val.programmaticStreamSerializationAllowed = a.ids ? 1 : 0;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t r = cudaLaunchKernelEx(&cfg, kern, a);
        return r != cudaSuccess ? r : cudaGetLastError();
    };
    // The fused mode cuts its own chunks at 8 rows: one n-tile per MMA (NT = 1); the permute
    // kernel's chunks hold up to 16 rows (NT = 2).
    const bool one = a.ids != nullptr;
    switch (a.fmt) {
    case QL_I8_G128_BF16: return one ? run(k_moe_tma<QL_I8_G128_BF16, 1>) : run(k_moe_tma<QL_I8_G128_BF16, 2>);
    case QL_I8_G128_F16: return one ? run(k_moe_tma<QL_I8_G128_F16, 1>) : run(k_moe_tma<QL_I8_G128_F16, 2>);
    case QL_FP8_B128_BF16: return one ? run(k_moe_tma<QL_FP8_B128_BF16, 1>) : run(k_moe_tma<QL_FP8_B128_BF16, 2>);
    case QL_FP8A8_B128_BF16:
        return one ? run(k_moe_tma<QL_FP8A8_B128_BF16, 1>) : run(k_moe_tma<QL_FP8A8_B128_BF16, 2>);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ql
