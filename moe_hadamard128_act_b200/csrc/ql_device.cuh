// ql_device.cuh -- device helpers shared by the kernels of libqlinear.so:
// the warp-wide 128-point Walsh-Hadamard transform, the small-integer and
// e4m3 to f16 conversions, and the mma.sync wrappers used by the skinny GEMM.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ql {

constexpr unsigned kFull = 0xffffffffu;

// fp32 nearest to 1/sqrt(128): the orthonormal scale of the 128-point transform.
__device__ __forceinline__ float fwht_scale() { return __int_as_float(0x3DB504F3); }

// In-warp Walsh-Hadamard transform of 128 values in Sylvester order.  Lane l
// holds elements 4l .. 4l+3 in v[0..3].  Butterflies (a, b) -> (a + b, a - b)
// run with strides 1, 2 (inside the lane), then 4, 8, 16, 32, 64 (across
// lanes l ^ 1 .. l ^ 16), each rounded to nearest in fp32, then every value
// is multiplied by fwht_scale().  The order and the roundings are fixed so
// that the result is reproducible bit for bit.
__device__ __forceinline__ void fwht128_warp(float v[4], int lane) {
    float a, b;
    a = v[0]; b = v[1]; v[0] = __fadd_rn(a, b); v[1] = __fsub_rn(a, b);
    a = v[2]; b = v[3]; v[2] = __fadd_rn(a, b); v[3] = __fsub_rn(a, b);
    a = v[0]; b = v[2]; v[0] = __fadd_rn(a, b); v[2] = __fsub_rn(a, b);
    a = v[1]; b = v[3]; v[1] = __fadd_rn(a, b); v[3] = __fsub_rn(a, b);
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        // lower lane: v + o; upper lane: o - v.  Both are o + sgn * v with sgn = +-1, one
        // FMA whose product is exact, so the single rounding is that of the add or subtract.
        const float sgn = (lane & m) ? -1.0f : 1.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float o = __shfl_xor_sync(kFull, v[i], m);
            v[i] = __fmaf_rn(sgn, v[i], o);
        }
    }
    const float c = fwht_scale();
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __fmul_rn(v[i], c);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
    return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Four consecutive bf16 values (8-byte aligned) as fp32.
__device__ __forceinline__ void load4_bf16(const __nv_bfloat16* p, float v[4]) {
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(raw.x << 16);
    v[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    v[2] = __uint_as_float(raw.y << 16);
    v[3] = __uint_as_float(raw.y & 0xFFFF0000u);
}

// The int8 quantiser of one 128-group held 4 values per lane by a warp:
// s = fp32(amax / 127), q = clamp(rne(fp32(v * fp32(127 / amax))), -127, 127);
// amax = 0 gives s = 0 and q = 0.  Returns the lane's 4 codes packed low byte
// first; *s is the group's scale in every lane.
__device__ __forceinline__ uint32_t quant_i8_group_warp(const float v[4], float* s_out) {
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    amax = warp_max(amax);
    uint32_t packed = 0;
    float s = 0.0f;
    if (amax > 0.0f) {
        s = __fdiv_rn(amax, 127.0f);
        const float inv = __fdiv_rn(127.0f, amax);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int c = __float2int_rn(__fmul_rn(v[i], inv));
            c = max(-127, min(127, c));
            packed |= (uint32_t)(c & 0xFF) << (8 * i);
        }
    }
    *s_out = s;
    return packed;
}
// Two fp32 values to E4M3 by the hardware conversion (round to nearest even,
// saturating to +-448): the low byte holds `lo`, the high byte `hi`.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float hi, float lo) {
    uint16_t r;
    asm("{\n .reg .b16 t;\n cvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n mov.b16 %0, t;\n}\n" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
// The E4M3 quantiser of one 128-group held 4 values per lane by a warp: the
// int8 rule with 448, the largest finite E4M3 value, in place of 127:
// s = fp32(amax / 448), q = e4m3(fp32(v * fp32(448 / amax))); amax = 0 gives
// s = 0 and q = 0.  Returns the lane's 4 codes packed low byte first.
__device__ __forceinline__ uint32_t quant_e4m3_group_warp(const float v[4], float* s_out) {
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    amax = warp_max(amax);
    uint32_t packed = 0;
    float s = 0.0f;
    if (amax > 0.0f) {
        s = __fdiv_rn(amax, 448.0f);
        const float inv = __fdiv_rn(448.0f, amax);
        const uint32_t lo = cvt_e4m3x2(__fmul_rn(v[1], inv), __fmul_rn(v[0], inv));
        const uint32_t hi = cvt_e4m3x2(__fmul_rn(v[3], inv), __fmul_rn(v[2], inv));
        packed = lo | (hi << 16);
    }
    *s_out = s;
    return packed;
}
__device__ __forceinline__ float f16_bits_to_float(uint16_t b) { return __half2float(__ushort_as_half(b)); }

// int5 codes straight into f16 MMA operands.  A lane holds 32 codes of a row
// as a 160-bit stream (code k at bits 5k .. 5k+4).  A 32-bit window of the
// stream starting at bit B, masked to one code inside the low half's mantissa
// (bits 0..9) and one inside the high half's, is an f16x2 pair of exact
// subnormals u * 2^(o - 24), o the code's offset inside its half.  The table
// lists the 16 pairs (window start, low code, high code): 4 windows are whole
// words, 12 take one funnel shift, so 32 codes cost 28 integer instructions.
// The activation of each code's MMA slot is staged pre-divided by 2^o, so every
// product is u * x * 2^-24; the zero point is taken off once per group with the
// token's sum of that group's activations.  Register r holds the codes of MMA
// slots (2c, 2c+1) of MMA r / 2 when r is even, (2c+8, 2c+9) when odd.
struct I5Pair {
    int B, klo, khi;
};
constexpr I5Pair kI5Pairs[16] = {{0, 0, 4},    {4, 1, 5},    {10, 2, 6},   {14, 3, 7},   {37, 8, 11},  {43, 9, 12},
                                 {49, 10, 14}, {64, 13, 17}, {72, 15, 18}, {76, 16, 19}, {96, 20, 23}, {100, 21, 24},
                                 {109, 22, 25}, {128, 26, 29}, {130, 27, 30}, {137, 28, 31}};
__host__ __device__ constexpr int i5_off_lo(int r) { return 5 * kI5Pairs[r].klo - kI5Pairs[r].B; }
__host__ __device__ constexpr int i5_off_hi(int r) { return 5 * kI5Pairs[r].khi - kI5Pairs[r].B - 16; }
// Slot s (0..31) of a lane's 32 activation values: MMA s / 4, register 2 (s / 4) + ((s / 2) & 1),
// its low half when s is even.  Returns the code index (0..31) it multiplies and its offset o.
__host__ __device__ constexpr int i5_slot_code(int s) {
    return (s & 1) ? kI5Pairs[2 * (s >> 2) + ((s >> 1) & 1)].khi : kI5Pairs[2 * (s >> 2) + ((s >> 1) & 1)].klo;
}
__host__ __device__ constexpr int i5_slot_off(int s) {
    return (s & 1) ? i5_off_hi(2 * (s >> 2) + ((s >> 1) & 1)) : i5_off_lo(2 * (s >> 2) + ((s >> 1) & 1));
}

// (a & b) | c in one LOP3 (truth table 0xEA).
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b) {
    __half2 r = __hadd2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
    __half2 r = __hfma2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b), *reinterpret_cast<__half2*>(&c));
    return *reinterpret_cast<uint32_t*>(&r);
}

// Four int8 codes (bytes 0..3 of w) -> f16x2 pairs lo = (c0, c1), hi = (c2, c3).
// Biasing to unsigned u = c + 128 and placing u in the low mantissa byte of
// 1024.0 gives 1024 + u exactly; adding -1152 leaves c, exact in f16.
__device__ __forceinline__ void i8x4_to_f16(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    lo = hadd2_u32(__byte_perm(u, 0x64646464u, 0x4140), 0xE480E480u);
    hi = hadd2_u32(__byte_perm(u, 0x64646464u, 0x4342), 0xE480E480u);
}

// Four int8 codes (bytes 0..3 of w) -> f16x2 pairs lo = (c0, c1), hi = (c2, c3)
// as subnormals: u = c + 128 placed in the low byte of a zero f16 is exactly
// u * 2^-24.  A dot product over a group then carries 2^-24 * (sum c x + 128 sum x);
// the caller takes the offset off with the activations' group sum.
__device__ __forceinline__ void i8x4_to_f16sub(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    lo = __byte_perm(u, 0u, 0x4140);
    hi = __byte_perm(u, 0u, 0x4342);
}

// Two e4m3 bytes (low, high) -> f16x2, exact (every e4m3 value is an f16).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_bytes) {
    __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two_bytes & 0xFFFFu), __NV_E4M3);
    return (uint32_t)r.x | ((uint32_t)r.y << 16);
}

// D(16x8, f32) += A(16x16, f16, row) * B(16x8, f16, col).
__device__ __forceinline__ void mma_f16(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D(16x8, s32) += A(16x32, s8, row) * B(32x8, s8, col); exact integer sums.
__device__ __forceinline__ void mma_s8(int d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Streaming loads of weight codes: read once, keep them out of L1.
__device__ __forceinline__ uint4 ldg_stream128(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ uint2 ldg_stream64(const void* p) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];\n" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ldg_stream32(const void* p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];\n" : "=r"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
    return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarriers, TMA and bulk copies (shared memory addresses are 32-bit) ----
__device__ __forceinline__ void mbar_init(uint32_t bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, unsigned phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(phase)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;\n" : "=l"(t));
    return t;
}
// Wait for phase `phase` of the mbarrier; false after ~lim ns without it.  The
// kernels bound their pipeline waits by wait_limit() and the waits that let
// work already started finish (copies in flight, MMAs before tensor memory is
// freed) by the default kWaitNs.
constexpr unsigned long long kWaitNs = 200ull * 1000 * 1000;
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, unsigned phase) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(phase)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, unsigned phase, unsigned long long lim = kWaitNs) {
    // A bound of at most 1 ns: one probe that does not block (try_wait may suspend for
    // a while, long enough for a copy to land), so the wait gives up unless done already.
    if (lim <= 1) return mbar_test_wait(bar, phase);
    if (mbar_try_wait(bar, phase)) return true;
    const unsigned long long t0 = global_ns();
    for (unsigned it = 0;; ++it) {
        if (mbar_try_wait(bar, phase)) return true;
        if (((it & 255u) == 255u || lim < kWaitNs) && global_ns() - t0 > lim) return false;
    }
}
// The pipeline wait limit: the override that ql_set_wait_limit stores next to
// the device error word (err[2..3]), or kWaitNs when it is 0.
__device__ __forceinline__ unsigned long long wait_limit(const unsigned* err) {
    const unsigned long long v = *reinterpret_cast<const volatile unsigned long long*>(err + 2);
    return v ? v : kWaitNs;
}
// One contiguous global -> shared copy, completing on an mbarrier (16-byte
// aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, unsigned bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
            dst),
        "l"(tmap), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

}  // namespace ql
