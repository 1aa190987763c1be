// k_act.cu -- activation-side kernels: the 128-wide Walsh-Hadamard rotation
// ("transform=fwht128" of the int8 experts in "gemma4-26b-a4b-dflash-i8"), the
// fused rotation + int8 quantiser with one scale per token per 128 values
// ("keptn/gemma4-12b-i8g", table "Format"), and the preparation of bf16
// activations for the weight-only skinny GEMM.
//
// Both transform kernels put one warp on one (token, 128-group): each lane
// loads 4 consecutive bf16 (8 bytes, so a warp reads one 256-byte group fully
// coalesced), the butterflies run in registers and through warp shuffles, and
// the max for the quantiser is a shuffle reduction.  They are bound by HBM
// (2 bytes in and 2 or 1 + 4/128 bytes out per element).
#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

constexpr int kWarpsPerBlock = 8;

__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_rotate_bf16(const __nv_bfloat16* x, int M, int K,
                                                                     __nv_bfloat16* y) {
    const int lane = threadIdx.x & 31;
    const long long G = K / 128;
    const long long nw = (long long)gridDim.x * kWarpsPerBlock;
    for (long long u = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); u < (long long)M * G; u += nw) {
        const long long off = (u / G) * K + (u % G) * 128 + 4 * lane;
        float v[4];
        load4_bf16(x + off, v);
        fwht128_warp(v, lane);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(v[2], v[3]);
        uint2 out;
        out.x = *reinterpret_cast<const uint32_t*>(&lo);
        out.y = *reinterpret_cast<const uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(y + off) = out;
    }
}

// Grid-stride zero of y[0 .. n) (16-byte stores; y is 16-byte aligned).
__device__ __forceinline__ void zero_fill(float* y, long long n) {
    if (!y) return;
    const long long stride = (long long)gridDim.x * blockDim.x;
    float4* y4 = reinterpret_cast<float4*>(y);
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n / 4; i += stride)
        y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (long long i = (n & ~3LL) + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) y[i] = 0.f;
}

// s = fp32(amax / 127), q = clamp(rne(fp32(v * fp32(127 / amax))), -127, 127);
// with E4M3 set, the E4M3 rule (448 for 127, codes by the hardware conversion).
// With inv != null (the grouped expert GEMM) token t's codes and scales go to
// rows inv[t * topk + j] of q and sxT (j < topk, negative entries skipped)
// instead of row t: the permuted order.
template <bool E4M3>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) k_act_quant(const __nv_bfloat16* x, int M, int K, int rotate,
                                                                   int8_t* q, float* sx, float* sxT, int Mp,
                                                                   float* yz, long long nz, const int32_t* inv,
                                                                   int topk) {
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");  // let the GEMM start its weight stream
    zero_fill(yz, nz);  // the GEMM that follows accumulates into y
    const int lane = threadIdx.x & 31;
    const int G = K / 128;
    // This warp's (token, group) units u = t * G + g, grid-strided by nw; the position is
    // stepped by (nw / G, nw % G) with a carry instead of divided out every time.
    const int nw = gridDim.x * kWarpsPerBlock, dt = nw / G, dg = nw % G;
    const int u0 = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    int t = u0 / G, g = u0 % G;
    for (; t < M; t += dt, g += dg) {
        if (g >= G) {
            g -= G;
            ++t;
            if (t >= M) break;
        }
        const long long u = (long long)t * G + g;
        const long long off = (long long)t * K + g * 128 + 4 * lane;
        float v[4];
        load4_bf16(x + off, v);
        if (rotate) fwht128_warp(v, lane);
        float s;
        const uint32_t packed = E4M3 ? quant_e4m3_group_warp(v, &s) : quant_i8_group_warp(v, &s);
        if (inv) {
            for (int j = 0; j < topk; ++j) {
                const int r = __ldg(inv + t * topk + j);
                if (r < 0) continue;
                *reinterpret_cast<uint32_t*>(q + (long long)r * K + g * 128 + 4 * lane) = packed;
                if (lane == 0) sxT[(long long)g * Mp + r] = s;
            }
            continue;
        }
        *reinterpret_cast<uint32_t*>(q + off) = packed;
        if (lane == 0) {
            if (sx) sx[u] = s;                                 // [M][G] row-major: u = m * G + g
            if (sxT) sxT[(long long)g * Mp + t] = s;           // [G][Mp], the prefill GEMM's layout
        }
    }
}

// One CTA per token.  The (optionally rotated and bf16-rounded) row is kept in
// shared memory as fp32; its max |x| picks a power of two f with
// max|x| * f in [2^14, 2^15), and xs = f16(x * f) is written in the element
// order of the format (within each 8-block [0,4,1,5,2,6,3,7] for int4,
// natural otherwise), and xf = 1 / f.  For int5 each 32-element run of a
// 128-group holds, in MMA slot order, the activations of the run's codes as
// the decode GEMM extracts them (kI5Pairs), each divided by 2^o for its code's
// offset o; the 16-byte pieces of each group are also swapped pairwise in
// their upper half (the shared-memory layout the GEMM reads without bank
// conflicts); xsum[t][g] = the group's sum of f16(x * f) (for the zero point),
// and xf = 2^24 / f (the codes enter the MMAs as u * 2^-24).  The natural
// order with xsum requested is the int8 decode's: the same group sums and
// 2^24 / f (its codes enter the MMAs as the subnormals (q + 128) * 2^-24).
// For int4 the activations of odd k (those that meet a byte's high nibble,
// which the decode GEMM uses in place as 16 u * 2^-24) are stored divided by
// 16, xsum holds the sums per 64-group, [M][K/64], and xf stays 1 / f (the
// int4 GEMM puts the 2^24 into its scales where it needs it).
// f16 holds every bf16 value of the scaled row exactly down to 2^-14 (its
// normal range); below that the rounding error is under 2^-39 of the row's
// max, far beneath the fp32 accumulation error of the GEMM.
// With inv != null the row is written to rows inv[t * topk + j] (j < topk,
// negative entries skipped, entries at or past xs_rows flagged as
// QL_DEVERR_BOUNDS and skipped) instead of row t: the permuted order of the
// grouped expert GEMM.
// Slots SL .. 31 of one int5 lane run starting at element b: the f16 activation
// of the slot's code (i5_slot_code), divided by 2^o (i5_slot_off), to its
// place with the pairwise piece swap.
template <int SL>
__device__ __forceinline__ void i5_stage_run(const float* r, float f, __half* out, int b) {
    if constexpr (SL < 32) {
        constexpr int code = i5_slot_code(SL), off = i5_slot_off(SL);
        const __half h = __float2half_rn(__fmul_rn(r[code], f));
        const int k = b + SL;
        out[k ^ (((k >> 6) & 1) << 3)] = __float2half_rn(__fmul_rn(__half2float(h), 1.0f / (float)(1 << off)));
        i5_stage_run<SL + 1>(r, f, out, b);
    }
}

__global__ void __launch_bounds__(256) k_prep_a16(const __nv_bfloat16* x, int M, int K, int rotate, int order,
                                                  __half* xs, float* xf, float* yz, long long nz, const int32_t* inv,
                                                  int topk, float* xsum, int xs_rows, unsigned* err) {
    extern __shared__ float row[];  // [K] fp32, then (natural order) [K] f16
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");  // let the GEMM start its weight stream
    zero_fill(yz, nz);  // the GEMM that follows accumulates into y (CTAs past M only help with this)
    const int t = blockIdx.x;
    if (t >= M) return;
    __shared__ float red[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const __nv_bfloat16* xr = x + (long long)t * K;
    float amax = 0.0f;
    for (int g = warp; g < K / 128; g += 8) {
        float v[4];
        load4_bf16(xr + g * 128 + 4 * lane, v);
        if (rotate) {
            fwht128_warp(v, lane);
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            row[g * 128 + 4 * lane + i] = v[i];
            amax = fmaxf(amax, fabsf(v[i]));
        }
    }
    amax = warp_max(amax);
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = red[0];
        for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
        int e = 0;
        if (m > 0.0f && m <= 3.4e38f) frexpf(m, &e);
        e = max(-100, min(128, e));
        red[0] = ldexpf(1.0f, 15 - e);
        xf[t] = ldexpf(1.0f, e - 15 + (xsum && order != XORD_I4 ? 24 : 0));
    }
    __syncthreads();
    const float f = red[0];
    if (xsum) {  // the groups' sums of the f16 activations (for the codes' offset); int4: per 64
        const bool g64 = order == XORD_I4;
        for (int g = warp; g < K / 128; g += 8) {
            float sum = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) sum += __half2float(__float2half_rn(__fmul_rn(row[g * 128 + 4 * lane + i], f)));
            for (int m = g64 ? 8 : 16; m > 0; m >>= 1) sum += __shfl_xor_sync(kFull, sum, m);
            if (!g64 && lane == 0) xsum[(long long)t * (K / 128) + g] = sum;
            if (g64 && (lane & 15) == 0) xsum[(long long)t * (K / 64) + 2 * g + (lane >> 4)] = sum;
        }
    }
    if (order == XORD_NATURAL) {  // converted once into shared memory, then 16-byte copies per output row
        uint4* const hrow = reinterpret_cast<uint4*>(row + K);  // [K / 8] x 8 f16
        const int K8 = K / 8;
        for (int c = threadIdx.x; c < K8; c += 256) {
            const float* r = row + 8 * c;
            uint32_t h[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __half2 p = __halves2half2(__float2half_rn(__fmul_rn(r[2 * i], f)),
                                                 __float2half_rn(__fmul_rn(r[2 * i + 1], f)));
                h[i] = *reinterpret_cast<const uint32_t*>(&p);
            }
            hrow[c] = make_uint4(h[0], h[1], h[2], h[3]);
        }
        __syncthreads();
        const int nrep = inv ? topk : 1;
        for (int idx = threadIdx.x; idx < nrep * K8; idx += 256) {
            const int j = idx / K8, c = idx - j * K8;
            const long long orow = inv ? (long long)__ldg(inv + (long long)t * topk + j) : (long long)t;
            if (orow >= xs_rows) {  // a permuted row outside xs (the permutation is device data): flag, skip
                if (c == 0) atomicOr(err, (unsigned)QL_DEVERR_BOUNDS);
            } else if (orow >= 0) {
                reinterpret_cast<uint4*>(xs + orow * K)[c] = hrow[c];
            }
        }
        return;
    }
    __half* out = xs + (long long)t * K;
    if (order == XORD_I5) {
        for (int run = threadIdx.x; run < K / 32; run += 256)  // one lane's 32 codes of a group
            i5_stage_run<0>(row + run * 32, f, out, run * 32);
        return;
    }
    for (int k = threadIdx.x; k < K; k += 256) {
        int src = k;
        if (order == XORD_I4) {
            const int p = k & 7;
            src = (k & ~7) + ((p & 1) ? 4 + (p >> 1) : (p >> 1));
        }
        __half h = __float2half_rn(__fmul_rn(row[src], f));
        // int4: an odd k meets a high nibble, which enters the MMA as 16 u * 2^-24
        if (order == XORD_I4 && (src & 1)) h = __float2half_rn(__fmul_rn(__half2float(h), 0.0625f));
        out[k] = h;
    }
}

// The activation between the experts' gate_up and down projections: for each
// (token, slot) pair p routed to an expert, a_i = gelu(h[p][i]) * h[p][I + i]
// in fp32, where h is the pair's gate_up output (gate half first) and gelu is
// the tanh form v * sigmoid(2 sqrt(2/pi) (v + 0.044715 v^3)), written with the
// logistic function so that nothing cancels for negative v.  a is stored as
// three bf16 planes a0 = bf16(a), a1 = bf16(a - a0), a2 = bf16(a - a0 - a1)
// (each difference exact in fp32), whose sum is a to within 2^-24 |a|, so the
// bf16 tensor-core products of the down projection keep fp32 precision.  One
// thread per 8 values (two 32-byte loads, three 16-byte stores).  Also zeroes
// out[0 .. nz), which the down projection accumulates into.
__device__ __forceinline__ float gelu_tanh_f32(float v) {
    const float u = 0.7978845608028654f * (v + 0.044715f * v * v * v);  // sqrt(2 / pi) (v + 0.044715 v^3)
    return v / (1.0f + expf(-2.0f * u));
}

__global__ void __launch_bounds__(256) k_moe_act(const float* h, const int32_t* ids, int P, int E, int I,
                                                 __nv_bfloat16* act, float* out, long long nz, const int32_t* inv) {
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");  // let the down GEMM start its weight stream
    zero_fill(out, nz);
    const int I8 = I / 8;
    const long long n = (long long)P * I8;
    for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < n; u += (long long)gridDim.x * blockDim.x) {
        const long long p = u / I8;
        const int i0 = (int)(u - p * I8) * 8;
        const int e = __ldg(ids + p);
        if (e < 0 || e >= E) continue;
        const float* hp = h + p * 2 * I;
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(hp + i0));
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(hp + i0 + 4));
        const float4 u0 = __ldg(reinterpret_cast<const float4*>(hp + I + i0));
        const float4 u1 = __ldg(reinterpret_cast<const float4*>(hp + I + i0 + 4));
        const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        uint32_t pl[3][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float r[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) r[k] = __fmul_rn(gelu_tanh_f32(gv[2 * q + k]), uv[2 * q + k]);
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(r[0], r[1]);
                pl[l][q] = *reinterpret_cast<const uint32_t*>(&b);
                r[0] = __fsub_rn(r[0], __low2float(b));
                r[1] = __fsub_rn(r[1], __high2float(b));
            }
        }
        const long long row = inv ? (long long)__ldg(inv + p) : p;
#pragma unroll
        for (int l = 0; l < 3; ++l)
            *reinterpret_cast<uint4*>(act + (row * 3 + l) * I + i0) = make_uint4(pl[l][0], pl[l][1], pl[l][2], pl[l][3]);
    }
}

// The GEMM that follows these kernels runs with (nearly) all of the SM's
// shared memory; asking for the same L1/shared split here avoids an SM
// reconfiguration between the two launches.
// Once per kernel and device (kernels of one signature share F, so the flag is
// kept per kernel address).
template <typename F>
cudaError_t prefer_max_shared(F* kernel) {
    struct Done {
        const void* k;
        int dev;
    };
    static Done done[64];
    static int n = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    for (int i = 0; i < n; ++i)
        if (done[i].k == (const void*)kernel && done[i].dev == dev) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess && n < 64) done[n++] = Done{(const void*)kernel, dev};
    return e;
}

int grid_for(long long warps, int sm_count) {
    long long blocks = (warps + kWarpsPerBlock - 1) / kWarpsPerBlock;
    long long cap = (long long)sm_count * 16;
    return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace

cudaError_t launch_rotate_bf16(const void* x, int M, int K, void* y, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    k_rotate_bf16<<<grid_for((long long)M * (K / 128), di.sm_count), kWarpsPerBlock * 32, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), M, K, static_cast<__nv_bfloat16*>(y));
    return cudaGetLastError();
}

cudaError_t launch_act_quant(const void* x, int M, int K, int rotate, int8_t* q, float* sx, float* sxT, int Mp,
                             float* yz, long long nz, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    if ((e = prefer_max_shared(k_act_quant<false>)) != cudaSuccess) return e;
    k_act_quant<false><<<grid_for((long long)M * (K / 128), di.sm_count), kWarpsPerBlock * 32, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), M, K, rotate, q, sx, sxT, Mp, yz, nz, nullptr, 0);
    return cudaGetLastError();
}

cudaError_t launch_act_quant_e4m3(const void* x, int M, int K, int rotate, uint8_t* q, float* sx, float* sxT, int Mp,
                                  float* yz, long long nz, cudaStream_t s, const int32_t* inv, int topk) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    if ((e = prefer_max_shared(k_act_quant<true>)) != cudaSuccess) return e;
    k_act_quant<true><<<grid_for((long long)M * (K / 128), di.sm_count), kWarpsPerBlock * 32, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), M, K, rotate, reinterpret_cast<int8_t*>(q), sx, sxT, Mp, yz, nz, inv,
        topk);
    return cudaGetLastError();
}

cudaError_t launch_prep_a16(const void* x, int M, int K, int rotate, int order, __half* xs, float* xf, float* yz,
                            long long nz, cudaStream_t s, float* xsum) {
    if ((order == XORD_I5 || order == XORD_I4) && !xsum) return cudaErrorInvalidValue;
    const size_t smem = (size_t)K * (sizeof(float) + sizeof(__half));  // the fp32 row and its f16 copy
    cudaError_t e = prefer_max_shared(k_prep_a16);
    if (e != cudaSuccess) return e;
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(k_prep_a16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    DeviceInfo di;
    if ((e = device_info(&di)) != cudaSuccess) return e;
    // Small M: extra CTAs (no row work) share the zeroing of y, about 8 KB each.
    const long long zb = yz ? (nz * 4 + 8191) / 8192 : 0;
    const long long zc = zb < 2LL * di.sm_count ? zb : 2LL * di.sm_count;
    const int grid = (int)(M > zc ? M : zc);
    k_prep_a16<<<grid, 256, smem, s>>>(static_cast<const __nv_bfloat16*>(x), M, K, rotate, order, xs, xf, yz, nz,
                                       nullptr, 1, xsum, M, di.err_word);
    return cudaGetLastError();
}


}  // namespace ql

namespace ql {
cudaError_t launch_moe_act(const float* h, const int32_t* ids, int P, int E, int I, __nv_bfloat16* act, float* out,
                           long long nz, cudaStream_t s, const int32_t* inv) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    if ((e = prefer_max_shared(k_moe_act)) != cudaSuccess) return e;
    const long long work = (long long)P * (I / 8);
    const long long zb = (nz + 1023) / 1024;
    long long blocks = ((work > zb * 256 ? work : zb * 256) + 255) / 256;
    if (blocks > 8LL * di.sm_count) blocks = 8LL * di.sm_count;
    if (blocks < 1) blocks = 1;
    k_moe_act<<<(unsigned)blocks, 256, 0, s>>>(h, ids, P, E, I, act, out, nz, inv);
    return cudaGetLastError();
}
}  // namespace ql
