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
#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

constexpr int kThreads = 512;
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
struct Regs<QL_I4_G64_BF16> {
    uint2 w[2][2];  // [row][64-wide half group]: 16 codes each
    float s[2][2];
};
template <>
struct Regs<QL_I5Z_G128_F16> {
    uint32_t w[2][5];  // [row][160-bit stream of 32 codes]
    float s[2];
    uint32_t nz[2];  // f16x2 of -(1024 + zero point)
};

// Bytes of activations per token per 128-group in shared memory, and the
// padding that makes the row stride an odd (1) or 2-mod-8 multiple of 16 B.
template <int FMT>
__host__ __device__ constexpr int x_group_bytes() { return FMT == QL_I8A8_G128_BF16 ? 128 : 256; }
template <int FMT>
__host__ __device__ constexpr int x_row_pad() { return (FMT == QL_I8A8_G128_BF16 || FMT == QL_I4_G64_BF16) ? 16 : 32; }
template <int FMT>
__host__ __device__ constexpr bool x_swizzled() { return !(FMT == QL_I8A8_G128_BF16 || FMT == QL_I4_G64_BF16); }

template <int FMT>
__device__ __forceinline__ int swz(int j) { return x_swizzled<FMT>() ? (j ^ ((j >> 3) & 1)) : j; }

template <int FMT>
__device__ __forceinline__ float load_scale(const void* scales, long long idx) {
    const uint16_t b = __ldg(static_cast<const uint16_t*>(scales) + idx);
    return (FMT == QL_I8_G128_F16 || FMT == QL_I5Z_G128_F16) ? f16_bits_to_float(b) : bf16_bits_to_float(b);
}

// Load one unit (rows n0 = slab*16 + g and n0 + 8, group grp) for lane (g, c).
// `wbase` points at the codes of row 0 of the matrix (group offset applied),
// `sbase`/`zbase` index the scales and zeros with row stride Gtot.
template <int FMT>
__device__ __forceinline__ void load_unit(Regs<FMT>& r, const uint8_t* wbase, long long ldw, const void* scales,
                                          const uint8_t* zeros, int N, int Gtot, int gabs, int slab, int grp, int g,
                                          int c) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int n = slab * 16 + g + 8 * h;
        const bool ok = n < N;
        const uint8_t* row = wbase + (long long)n * ldw;
        if constexpr (FMT == QL_I4_G64_BF16) {
            if (ok) {
                const uint8_t* p = row + grp * 64 + 8 * c;
                r.w[h][0] = ldg_stream64(p);
                r.w[h][1] = ldg_stream64(p + 32);
                r.s[h][0] = load_scale<FMT>(scales, (long long)n * (2 * Gtot) + 2 * gabs);
                r.s[h][1] = load_scale<FMT>(scales, (long long)n * (2 * Gtot) + 2 * gabs + 1);
            } else {
                r.w[h][0] = r.w[h][1] = make_uint2(0x88888888u, 0x88888888u);
                r.s[h][0] = r.s[h][1] = 0.0f;
            }
        } else if constexpr (FMT == QL_I5Z_G128_F16) {
            if (ok) {
                const uint8_t* p = row + grp * 80 + 20 * c;
#pragma unroll
                for (int i = 0; i < 5; ++i) r.w[h][i] = ldg_stream32(p + 4 * i);
                r.s[h] = load_scale<FMT>(scales, (long long)n * Gtot + gabs);
                const float z = (float)__ldg(zeros + (long long)n * Gtot + gabs);
                const __half nz = __float2half_rn(-(1024.0f + z));
                r.nz[h] = (uint32_t)__half_as_ushort(nz) * 0x10001u;
            } else {
#pragma unroll
                for (int i = 0; i < 5; ++i) r.w[h][i] = 0;
                r.s[h] = 0.0f;
                r.nz[h] = 0xE400E400u;  // -1024
            }
        } else {
            if (ok) {
                const uint8_t* p = row + grp * 128 + 32 * c;
                r.w[h][0] = ldg_stream128(p);
                r.w[h][1] = ldg_stream128(p + 16);
                if constexpr (FMT == QL_FP8_B128_BF16)
                    r.s[h] = load_scale<FMT>(scales, (long long)(n >> 7) * Gtot + gabs);
                else  // the integer-only W8A8 check path has no scales
                    r.s[h] = scales ? load_scale<FMT>(scales, (long long)n * Gtot + gabs) : 0.0f;
            } else {
                r.w[h][0] = r.w[h][1] = make_uint4(0, 0, 0, 0);
                r.s[h] = 0.0f;
            }
        }
    }
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

// The per-group MMAs of one unit for the weight-only formats.
// getx(nt, piece) returns the lane's 16-byte activation piece for n-tile nt.
// yacc[nt][i] accumulates scale * partial; i = 0,1 row g, i = 2,3 row g + 8.
template <int FMT, int NT, typename GetX>
__device__ __forceinline__ void unit_a16(const Regs<FMT>& r, GetX getx, bool nt1_live, float (&yacc)[NT][4]) {
    if constexpr (FMT == QL_I4_G64_BF16) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                uint4 xv[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    if (nt == 0 || nt1_live) xv[nt] = getx(nt, 8 * h + p);
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    const int j = 2 * sub;
                    const uint32_t w0 = p == 0 ? r.w[0][h].x : r.w[0][h].y;
                    const uint32_t w1 = p == 0 ? r.w[1][h].x : r.w[1][h].y;
                    const uint32_t a0 = hadd2_u32(((w0 >> (4 * j)) & 0x000F000Fu) | 0x64006400u, 0xE408E408u);
                    const uint32_t a2 = hadd2_u32(((w0 >> (4 * j + 4)) & 0x000F000Fu) | 0x64006400u, 0xE408E408u);
                    const uint32_t a1 = hadd2_u32(((w1 >> (4 * j)) & 0x000F000Fu) | 0x64006400u, 0xE408E408u);
                    const uint32_t a3 = hadd2_u32(((w1 >> (4 * j + 4)) & 0x000F000Fu) | 0x64006400u, 0xE408E408u);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (nt == 1 && !nt1_live) continue;
                        const uint32_t b0 = sub == 0 ? xv[nt].x : xv[nt].z;
                        const uint32_t b1 = sub == 0 ? xv[nt].y : xv[nt].w;
                        mma_f16(acc[nt], a0, a1, a2, a3, b0, b1);
                    }
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                yacc[nt][0] = fmaf(r.s[0][h], acc[nt][0], yacc[nt][0]);
                yacc[nt][1] = fmaf(r.s[0][h], acc[nt][1], yacc[nt][1]);
                yacc[nt][2] = fmaf(r.s[1][h], acc[nt][2], yacc[nt][2]);
                yacc[nt][3] = fmaf(r.s[1][h], acc[nt][3], yacc[nt][3]);
            }
        }
    } else {
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
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
                if constexpr (FMT == QL_I5Z_G128_F16) {
                    const int bit = 20 * s, wi = bit >> 5, sh = bit & 31;
                    const uint32_t t0 = __funnelshift_r(r.w[0][wi], wi < 4 ? r.w[0][wi + 1] : 0u, sh);
                    const uint32_t t1 = __funnelshift_r(r.w[1][wi], wi < 4 ? r.w[1][wi + 1] : 0u, sh);
                    a0 = hadd2_u32((t0 & 0x1Fu) | ((t0 << 1) & 0x1F0000u) | 0x64006400u, r.nz[0]);
                    a2 = hadd2_u32(((t0 >> 5) & 0x1Fu) | ((t0 << 6) & 0x1F0000u) | 0x64006400u, r.nz[0]);
                    a1 = hadd2_u32((t1 & 0x1Fu) | ((t1 << 1) & 0x1F0000u) | 0x64006400u, r.nz[1]);
                    a3 = hadd2_u32(((t1 >> 5) & 0x1Fu) | ((t1 << 6) & 0x1F0000u) | 0x64006400u, r.nz[1]);
                } else if constexpr (FMT == QL_FP8_B128_BF16) {
                    const uint32_t w0 = word_of(r.w[0], s), w1 = word_of(r.w[1], s);
                    a0 = e4m3x2_to_f16x2(w0);
                    a2 = e4m3x2_to_f16x2(w0 >> 16);
                    a1 = e4m3x2_to_f16x2(w1);
                    a3 = e4m3x2_to_f16x2(w1 >> 16);
                } else {
                    i8x4_to_f16(word_of(r.w[0], s), a0, a2);
                    i8x4_to_f16(word_of(r.w[1], s), a1, a3);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt == 1 && !nt1_live) continue;
                    const uint32_t b0 = sub == 0 ? xv[nt].x : xv[nt].z;
                    const uint32_t b1 = sub == 0 ? xv[nt].y : xv[nt].w;
                    mma_f16(acc[nt], a0, a1, a2, a3, b0, b1);
                }
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            yacc[nt][0] = fmaf(r.s[0], acc[nt][0], yacc[nt][0]);
            yacc[nt][1] = fmaf(r.s[0], acc[nt][1], yacc[nt][1]);
            yacc[nt][2] = fmaf(r.s[1], acc[nt][2], yacc[nt][2]);
            yacc[nt][3] = fmaf(r.s[1], acc[nt][3], yacc[nt][3]);
        }
    }
}

// W8A8: exact int32 sums of one group (4 k-steps of m16n8k32).
template <int NT, typename GetX>
__device__ __forceinline__ void unit_w8a8(const Regs<QL_I8A8_G128_BF16>& r, GetX getx, int (&acc)[NT][4]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0;
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
                mma_s8(acc[nt], a0, a1, a2, a3, b0, b1);
            }
        }
    }
}

template <int FMT>
constexpr size_t skinny_smem(int NT, int G) {
    return (size_t)NT * 8 * ((size_t)G * x_group_bytes<FMT>() + x_row_pad<FMT>()) +
           (FMT == QL_I8A8_G128_BF16 ? (size_t)16 * G * 4 : 16 * 4);
}

// Dense skinny GEMM over one (token chunk, K chunk).
template <int FMT, int NT, bool ACC>
__global__ void __launch_bounds__(kThreads, 1) k_skinny(SkinnyArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr int XGB = x_group_bytes<FMT>();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int G = a.G;
    const long long R = (long long)G * XGB + x_row_pad<FMT>();
    float* fac = reinterpret_cast<float*>(smem + NT * 8 * R);

    const int slabs = (a.N + 15) / 16;
    const long long units = (long long)slabs * G;
    const long long wid = (long long)blockIdx.x * kWarps + warp, nw = (long long)gridDim.x * kWarps;
    const long long u0 = units * wid / nw, u1 = units * (wid + 1) / nw;

    Regs<FMT> r0, r1, r2;
    auto load = [&](Regs<FMT>& r, long long u) {
        const int slab = (int)(u / G), grp = (int)(u % G);
        load_unit<FMT>(r, a.W, a.ldw, a.scales, a.zeros, a.N, a.Gtot, a.g0 + grp, slab, grp, g, c);
    };
    // Start the weight stream before staging the activations.
    if (u0 < u1) load(r0, u0);
    if (u0 + 1 < u1) load(r1, u0 + 1);

    // Stage activations: token rows [0, NT*8), zero beyond M.
    {
        const int pieces_per_row = G * XGB / 16;
        const int total = NT * 8 * pieces_per_row;
        const uint8_t* xsrc = static_cast<const uint8_t*>(a.xs);
        const long long ldx_b = a.ldx * (FMT == QL_I8A8_G128_BF16 ? 1 : 2);
        for (int i = threadIdx.x; i < total; i += kThreads) {
            const int t = i / pieces_per_row, j = i % pieces_per_row;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (t < a.M) v = *reinterpret_cast<const uint4*>(xsrc + t * ldx_b + 16LL * j);
            *reinterpret_cast<uint4*>(smem + t * R + 16LL * swz<FMT>(j)) = v;
        }
        if constexpr (FMT == QL_I8A8_G128_BF16) {
            for (int i = threadIdx.x; i < 16 * G; i += kThreads) {
                const int t = i / G, gg = i % G;
                fac[i] = (t < a.M && a.xf) ? a.xf[(long long)t * a.Gtot + a.g0 + gg] : 0.0f;
            }
        } else {
            if (threadIdx.x < 16) fac[threadIdx.x] = threadIdx.x < a.M ? a.xf[threadIdx.x] : 0.0f;
        }
    }
    __syncthreads();
    if (u0 >= u1) return;

    const uint32_t xs_base = smem_u32(smem);
    const bool nt1_live = NT > 1 && a.M > 8;
    float yacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) yacc[nt][0] = yacc[nt][1] = yacc[nt][2] = yacc[nt][3] = 0.0f;
    int cur_slab = (int)(u0 / G);

    auto flush = [&](int slab) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = 8 * nt + 2 * c + (i & 1);
                const int n = slab * 16 + g + 8 * (i >> 1);
                if (t < a.M && n < a.N) {
                    const float f = (FMT == QL_I8A8_G128_BF16) ? 1.0f : fac[t];
                    atomicAdd(a.y + (long long)t * a.ldy + n, yacc[nt][i] * f);
                }
                yacc[nt][i] = 0.0f;
            }
    };

    auto process = [&](const Regs<FMT>& r, long long u) {
        const int slab = (int)(u / G), grp = (int)(u % G);
        if (!ACC && slab != cur_slab) {
            flush(cur_slab);
            cur_slab = slab;
        }
        auto getx = [&](int nt, int p) -> uint4 {
            // p: piece of the lane's chunk; for int4 bit 3 of p selects the 64-wide half
            int j;
            if constexpr (FMT == QL_I8A8_G128_BF16)
                j = grp * 8 + 2 * c + p;
            else if constexpr (FMT == QL_I4_G64_BF16)
                j = grp * 16 + (p & 8) + 2 * c + (p & 1);
            else
                j = grp * 16 + 4 * c + p;
            return lds128(xs_base + (uint32_t)((8 * nt + g) * R + 16 * swz<FMT>(j)));
        };
        if constexpr (FMT == QL_I8A8_G128_BF16) {
            int acc[NT][4];
            unit_w8a8<NT>(r, getx, acc);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = 8 * nt + 2 * c + (i & 1);
                    const int n = slab * 16 + g + 8 * (i >> 1);
                    if (ACC) {
                        if (t < a.M && n < a.N) a.acc[((long long)t * a.N + n) * a.Gtot + a.g0 + grp] = acc[nt][i];
                    } else {
                        const float sc = r.s[i >> 1] * fac[t * G + grp];
                        yacc[nt][i] = fmaf(sc, __int2float_rn(acc[nt][i]), yacc[nt][i]);
                    }
                }
        } else {
            unit_a16<FMT, NT>(r, getx, nt1_live, yacc);
        }
    };

    long long u = u0;
    while (u < u1) {
        if (u + 2 < u1) load(r2, u + 2);
        process(r0, u);
        if (++u >= u1) break;
        if (u + 2 < u1) load(r0, u + 2);
        process(r1, u);
        if (++u >= u1) break;
        if (u + 2 < u1) load(r1, u + 2);
        process(r2, u);
        ++u;
    }
    if (!ACC) flush(cur_slab);
}

// Grouped (MoE) skinny GEMM: units are (row chunk of one expert, slab, group);
// the activations of a chunk's tokens are gathered from the prepared [T, K]
// buffer (L2-resident) and results are scattered to y[(t, j), :] rows.
template <int FMT, int NT>
__global__ void __launch_bounds__(kThreads, 1) k_moe_skinny(MoeArgs a) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int G = a.K / 128;
    const int slabs = (a.N + 15) / 16;
    const long long per_chunk = (long long)slabs * G;
    const long long nch = min((long long)*a.n_chunks, a.max_chunks);
    const long long units = nch * per_chunk;
    const long long wid = (long long)blockIdx.x * kWarps + warp, nw = (long long)gridDim.x * kWarps;
    const long long u0 = units * wid / nw, u1 = units * (wid + 1) / nw;
    if (u0 >= u1) return;
    const long long ldw = a.K;  // int8 / fp8 rows
    const long long expert_codes = (long long)a.N * a.K;
    const long long expert_scales = FMT == QL_FP8_B128_BF16 ? (long long)((a.N + 127) / 128) * G : (long long)a.N * G;

    Regs<FMT> r0, r1, r2;
    auto load = [&](Regs<FMT>& r, long long u) {
        const MoeChunk ch = a.chunks[u / per_chunk];
        const long long rem = u % per_chunk;
        const int slab = (int)(rem / G), grp = (int)(rem % G);
        const uint8_t* wb = a.codes + (long long)ch.expert * expert_codes;
        const void* sb = static_cast<const uint16_t*>(a.scales) + (long long)ch.expert * expert_scales;
        load_unit<FMT>(r, wb, ldw, sb, nullptr, a.N, G, grp, slab, grp, g, c);
    };
    if (u0 < u1) load(r0, u0);
    if (u0 + 1 < u1) load(r1, u0 + 1);

    float yacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) yacc[nt][0] = yacc[nt][1] = yacc[nt][2] = yacc[nt][3] = 0.0f;
    long long cur_key = u0 / G;  // (chunk, slab)

    auto flush = [&](long long key) {
        const MoeChunk ch = a.chunks[key / slabs];
        const int slab = (int)(key % slabs);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int slot = 8 * nt + 2 * c + (i & 1);
                const int n = slab * 16 + g + 8 * (i >> 1);
                if (slot < ch.count && n < a.N) {
                    const int pair = a.perm[ch.start + slot];
                    const float f = a.xf[pair / a.topk];
                    atomicAdd(a.y + (long long)pair * a.N + n, yacc[nt][i] * f);
                }
                yacc[nt][i] = 0.0f;
            }
    };

    auto process = [&](const Regs<FMT>& r, long long u) {
        const long long key = u / G;
        const int grp = (int)(u % G);
        if (key != cur_key) {
            flush(cur_key);
            cur_key = key;
        }
        const MoeChunk ch = a.chunks[key / slabs];
        int tok[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int slot = 8 * nt + g;
            tok[nt] = slot < ch.count ? a.perm[ch.start + slot] / a.topk : -1;
        }
        auto getx = [&](int nt, int p) -> uint4 {
            if (tok[nt] < 0) return make_uint4(0, 0, 0, 0);
            return __ldg(reinterpret_cast<const uint4*>(a.xs + (long long)tok[nt] * a.K + grp * 128 + 32 * c + 8 * p));
        };
        unit_a16<FMT, NT>(r, getx, ch.count > 8, yacc);
    };

    long long u = u0;
    while (u < u1) {
        if (u + 2 < u1) load(r2, u + 2);
        process(r0, u);
        if (++u >= u1) break;
        if (u + 2 < u1) load(r0, u + 2);
        process(r1, u);
        if (++u >= u1) break;
        if (u + 2 < u1) load(r1, u + 2);
        process(r2, u);
        ++u;
    }
    flush(cur_key);
}

template <int FMT, int NT, bool ACC>
cudaError_t run_skinny(const SkinnyArgs& a, cudaStream_t s, const DeviceInfo& di) {
    const size_t smem = skinny_smem<FMT>(NT, a.G);
    if (smem > di.smem_optin) return cudaErrorInvalidValue;
    static bool attr_set[64] = {};  // per device ordinal
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 64 || !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_skinny<FMT, NT, ACC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)di.smem_optin);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_set[dev] = true;
    }
    k_skinny<FMT, NT, ACC><<<di.sm_count, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t run_skinny_fmt(const SkinnyArgs& a, cudaStream_t s, const DeviceInfo& di) {
    if (a.M > 8) return run_skinny<FMT, 2, false>(a, s, di);
    return run_skinny<FMT, 1, false>(a, s, di);
}

}  // namespace

int skinny_max_k(int fmt) {
    DeviceInfo di;
    if (device_info(&di) != cudaSuccess) return 0;
    for (int G = 256; G >= 1; --G) {
        size_t need = fmt == QL_I8A8_G128_BF16 ? skinny_smem<QL_I8A8_G128_BF16>(2, G)
                                                : skinny_smem<QL_I8_G128_BF16>(2, G);
        if (need <= di.smem_optin) return G * 128;
    }
    return 0;
}

cudaError_t launch_skinny(int fmt, const SkinnyArgs& a, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    if (a.acc) {
        if (fmt != QL_I8A8_G128_BF16) return cudaErrorInvalidValue;
        if (a.M > 8) return run_skinny<QL_I8A8_G128_BF16, 2, true>(a, s, di);
        return run_skinny<QL_I8A8_G128_BF16, 1, true>(a, s, di);
    }
    switch (fmt) {
    case QL_I8_G128_BF16: return run_skinny_fmt<QL_I8_G128_BF16>(a, s, di);
    case QL_I8_G128_F16: return run_skinny_fmt<QL_I8_G128_F16>(a, s, di);
    case QL_I8A8_G128_BF16: return run_skinny_fmt<QL_I8A8_G128_BF16>(a, s, di);
    case QL_I4_G64_BF16: return run_skinny_fmt<QL_I4_G64_BF16>(a, s, di);
    case QL_I5Z_G128_F16: return run_skinny_fmt<QL_I5Z_G128_F16>(a, s, di);
    case QL_FP8_B128_BF16: return run_skinny_fmt<QL_FP8_B128_BF16>(a, s, di);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_moe_skinny(const MoeArgs& a, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    switch (a.fmt) {
    case QL_I8_G128_BF16: k_moe_skinny<QL_I8_G128_BF16, 2><<<di.sm_count, kThreads, 0, s>>>(a); break;
    case QL_I8_G128_F16: k_moe_skinny<QL_I8_G128_F16, 2><<<di.sm_count, kThreads, 0, s>>>(a); break;
    case QL_FP8_B128_BF16: k_moe_skinny<QL_FP8_B128_BF16, 2><<<di.sm_count, kThreads, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace ql
