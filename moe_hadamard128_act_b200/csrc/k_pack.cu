// k_pack.cu -- weight packing ("rtn codes=... group=... scale=... [transform=
// fwht128] clamp=sym" in the recipes of the "gemma4-26b-a4b-dflash-i8" and
// "-fp8" READMEs; the int4 g64 layout of "Gemma4-26B-CIRU-AMD-STRIX-vLLM"; the
// int5 + zero point layout of "keptn/gemma4-31b-w5").
//
// Round-to-nearest quantisers: one warp per (row, 128 columns), 4 fp32 per
// lane (16-byte loads), optional in-register Walsh-Hadamard transform, the
// group max by shuffles; the int8 scale search scores its 21 candidate scales
// on 21 lanes of the same warp.  FP8 takes one CTA per 128x128 block, whose rotated
// values are staged in shared memory for the block max.  Packers of given
// codes run one thread per 8 codes.
#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

__device__ __forceinline__ void load4_f32(const float* p, float v[4]) {
    const float4 r = *reinterpret_cast<const float4*>(p);
    v[0] = r.x; v[1] = r.y; v[2] = r.z; v[3] = r.w;
}

// int8, group 128: s = scale_fmt(fp32(amax / 127)); q = clamp(rne(fp32(w / s)), -127, 127).
template <bool kF16Scale>
__global__ void __launch_bounds__(256) k_rtn_i8(const float* W, int N, int K, int hadamard, int8_t* q,
                                                uint16_t* s) {
    const int lane = threadIdx.x & 31;
    const long long G = K / 128;
    const long long nw = (long long)gridDim.x * 8;
    for (long long u = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); u < (long long)N * G; u += nw) {
        const long long off = (u / G) * K + (u % G) * 128 + 4 * lane;
        float v[4];
        load4_f32(W + off, v);
        if (hadamard) fwht128_warp(v, lane);
        float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
        amax = warp_max(amax);
        const float raw = __fdiv_rn(amax, 127.0f);
        uint16_t sb;
        float sf;
        if (kF16Scale) {
            const __half h = __float2half_rn(raw);
            sb = __half_as_ushort(h);
            sf = __half2float(h);
        } else {
            const __nv_bfloat16 b = __float2bfloat16_rn(raw);
            sb = __bfloat16_as_ushort(b);
            sf = __bfloat162float(b);
        }
        uint32_t packed = 0;
        if (sf != 0.0f) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int c = __float2int_rn(__fdiv_rn(v[i], sf));
                c = max(-127, min(127, c));
                packed |= (uint32_t)(c & 0xFF) << (8 * i);
            }
        }
        *reinterpret_cast<uint32_t*>(q + off) = packed;
        if (lane == 0) s[u] = sb;
    }
}

// int8, group 128, with the scale search of the int8 experts' recipe (rule=search, "round to
// nearest with a scale search"): candidate i = 0..20 quantises the group by round to nearest
// with s_i = scale_fmt(fp32(fp32(amax / 127) * fp32((100 - i) / 100))) and scores it by its
// squared error, summed over k = 0..127 in order in fp64 with every product, difference and sum
// rounded on its own; the least error wins, the smaller i on a tie.  One warp per group: lane i
// scores candidate i over the group staged in shared memory (its sum is sequential, so the
// result does not depend on how the work is split), then every lane writes its four codes.
template <bool kF16Scale>
__global__ void __launch_bounds__(256) k_search_i8(const float* W, int N, int K, int hadamard, int8_t* q,
                                                   uint16_t* s) {
    __shared__ float grp[8][128];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const long long G = K / 128;
    const long long nw = (long long)gridDim.x * 8;
    for (long long u = (long long)blockIdx.x * 8 + wib; u < (long long)N * G; u += nw) {
        const long long off = (u / G) * K + (u % G) * 128 + 4 * lane;
        float v[4];
        load4_f32(W + off, v);
        if (hadamard) fwht128_warp(v, lane);
        float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
        amax = warp_max(amax);
        *reinterpret_cast<float4*>(&grp[wib][4 * lane]) = make_float4(v[0], v[1], v[2], v[3]);
        __syncwarp();
        const float r = __fdiv_rn(amax, 127.0f);
        double err = INFINITY;
        float sf_i = 0.0f;
        uint32_t sb_i = 0;
        if (lane <= 20) {
            const float raw = __fmul_rn(r, __fdiv_rn((float)(100 - lane), 100.0f));
            if (kF16Scale) {
                const __half h = __float2half_rn(raw);
                sb_i = __half_as_ushort(h);
                sf_i = __half2float(h);
            } else {
                const __nv_bfloat16 b = __float2bfloat16_rn(raw);
                sb_i = __bfloat16_as_ushort(b);
                sf_i = __bfloat162float(b);
            }
            const double sd = (double)sf_i;
            double e = 0.0;
            for (int k = 0; k < 128; ++k) {
                const float w = grp[wib][k];
                const int c = sf_i != 0.0f ? max(-127, min(127, __float2int_rn(__fdiv_rn(w, sf_i)))) : 0;
                const double d = __dsub_rn((double)w, __dmul_rn(sd, (double)c));
                e = __dadd_rn(e, __dmul_rn(d, d));
            }
            // A NaN score (a scale that overflowed f16) never wins, except at candidate 0,
            // which a sequential scan starts from and only a smaller score replaces.
            err = isnan(e) ? (lane == 0 ? -INFINITY : INFINITY) : e;
        }
        int best = lane;
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
            const double oe = __shfl_xor_sync(kFull, err, m);
            const int ob = __shfl_xor_sync(kFull, best, m);
            if (oe < err || (oe == err && ob < best)) {
                err = oe;
                best = ob;
            }
        }
        const float sf = __shfl_sync(kFull, sf_i, best);
        const uint32_t sb = __shfl_sync(kFull, sb_i, best);
        uint32_t packed = 0;
        if (sf != 0.0f) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int c = __float2int_rn(__fdiv_rn(v[i], sf));
                c = max(-127, min(127, c));
                packed |= (uint32_t)(c & 0xFF) << (8 * i);
            }
        }
        *reinterpret_cast<uint32_t*>(q + off) = packed;
        if (lane == 0) s[u] = (uint16_t)sb;
        __syncwarp();  // the group's shared-memory copy is read before the next one lands
    }
}

// int4, group 64: s = bf16(fp32(amax / 7)); q = clamp(rne(fp32(w / s)), -8, 7);
// stored offset-binary, two codes per byte, low nibble first.
__global__ void __launch_bounds__(256) k_rtn_i4(const float* W, int N, int K, int hadamard, uint8_t* q,
                                                uint16_t* s) {
    const int lane = threadIdx.x & 31;
    const long long C = K / 128;
    const long long nw = (long long)gridDim.x * 8;
    for (long long u = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); u < (long long)N * C; u += nw) {
        const long long n = u / C, c = u % C;
        const long long off = n * K + c * 128 + 4 * lane;
        float v[4];
        load4_f32(W + off, v);
        if (hadamard) fwht128_warp(v, lane);
        float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
        for (int m = 8; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, m));  // per 16 lanes
        const __nv_bfloat16 b = __float2bfloat16_rn(__fdiv_rn(amax, 7.0f));
        const float sf = __bfloat162float(b);
        uint32_t nib = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int cq = 0;
            if (sf != 0.0f) cq = max(-8, min(7, __float2int_rn(__fdiv_rn(v[i], sf))));
            nib |= (uint32_t)(cq + 8) << (4 * i);
        }
        *reinterpret_cast<uint16_t*>(q + n * (K / 2) + c * 64 + 2 * lane) = (uint16_t)nib;
        if ((lane & 15) == 0) s[n * (K / 64) + c * 2 + (lane >> 4)] = __bfloat16_as_ushort(b);
    }
}

// FP8 E4M3 per 128x128 block: s = bf16(fp32(amax / 448)); q = e4m3_rne_satfinite(fp32(w / s)).
__global__ void __launch_bounds__(256) k_rtn_fp8(const float* W, int N, int K, int hadamard, uint8_t* q,
                                                 uint16_t* s) {
    extern __shared__ float tile[];  // [128][128]
    __shared__ float red[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nb = blockIdx.x, g = blockIdx.y, G = K / 128;
    float amax = 0.0f;
    for (int r = warp; r < 128; r += 8) {
        const long long n = (long long)nb * 128 + r;
        if (n >= N) break;
        float v[4];
        load4_f32(W + n * K + (long long)g * 128 + 4 * lane, v);
        if (hadamard) fwht128_warp(v, lane);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            tile[r * 128 + 4 * lane + i] = v[i];
            amax = fmaxf(amax, fabsf(v[i]));
        }
    }
    amax = warp_max(amax);
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = red[0];
        for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
        const __nv_bfloat16 b = __float2bfloat16_rn(__fdiv_rn(m, 448.0f));
        red[0] = __bfloat162float(b);
        s[(long long)nb * G + g] = __bfloat16_as_ushort(b);
    }
    __syncthreads();
    const float sf = red[0];
    for (int r = warp; r < 128; r += 8) {
        const long long n = (long long)nb * 128 + r;
        if (n >= N) break;
        uint32_t packed = 0;
        if (sf != 0.0f) {
            const float* v = tile + r * 128 + 4 * lane;
            const __nv_fp8x2_storage_t lo =
                __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(v[0], sf), __fdiv_rn(v[1], sf)), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t hi =
                __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(v[2], sf), __fdiv_rn(v[3], sf)), __NV_SATFINITE, __NV_E4M3);
            packed = (uint32_t)lo | ((uint32_t)hi << 16);
        }
        *reinterpret_cast<uint32_t*>(q + n * K + (long long)g * 128 + 4 * lane) = packed;
    }
}

// Given codes, 8 per thread.  Out-of-range codes are packed as 0 and flagged.
template <int kFmt>
__global__ void k_pack_codes(const uint8_t* in, long long n8, uint8_t* out, unsigned* err) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
        const uint2 raw = reinterpret_cast<const uint2*>(in)[i];
        const uint8_t* b = reinterpret_cast<const uint8_t*>(&raw);
        bool bad = false;
        if (kFmt == QL_I4_G64_BF16) {
            uint32_t w = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                int c = (int8_t)b[j];
                if (c < -8 || c > 7) { bad = true; c = 0; }
                w |= (uint32_t)(c + 8) << (4 * j);
            }
            reinterpret_cast<uint32_t*>(out)[i] = w;
        } else if (kFmt == QL_I5Z_G128_F16) {
            unsigned long long w = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                unsigned c = b[j];
                if (c > 31) { bad = true; c = 0; }
                w |= (unsigned long long)c << (5 * j);
            }
#pragma unroll
            for (int j = 0; j < 5; ++j) out[i * 5 + j] = (uint8_t)(w >> (8 * j));
        } else if (kFmt == QL_FP8_B128_BF16) {
            uint2 o = raw;
            uint8_t* ob = reinterpret_cast<uint8_t*>(&o);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if ((ob[j] & 0x7F) == 0x7F) { bad = true; ob[j] = 0; }  // NaN codes
            reinterpret_cast<uint2*>(out)[i] = o;
        } else {  // int8: -128 is outside the symmetric range
            uint2 o = raw;
            uint8_t* ob = reinterpret_cast<uint8_t*>(&o);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (ob[j] == 0x80) { bad = true; ob[j] = 0; }
            reinterpret_cast<uint2*>(out)[i] = o;
        }
        if (bad) atomicOr(err, (unsigned)QL_DEVERR_CODE_RANGE);
    }
}

__global__ void k_check_zeros(const uint8_t* in, long long n, uint8_t* out, unsigned* err) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        uint8_t z = in[i];
        if (z > 31) { atomicOr(err, (unsigned)QL_DEVERR_CODE_RANGE); z = 0; }
        out[i] = z;
    }
}

int blocks_for(long long items, int threads, int sm_count) {
    long long b = (items + threads - 1) / threads;
    long long cap = (long long)sm_count * 16;
    return (int)(b < 1 ? 1 : (b < cap ? b : cap));
}

}  // namespace

cudaError_t launch_pack_rtn(const float* W, int fmt, int flags, int N, int K, void* codes, void* scales,
                            cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    const int had = (flags & QL_HADAMARD) ? 1 : 0;
    const long long warps = (long long)N * (K / 128);
    const int grid = blocks_for(warps * 32, 256, di.sm_count);
    if (flags & QL_SCALE_SEARCH) {
        switch (fmt) {
        case QL_I8_G128_BF16:
        case QL_I8A8_G128_BF16:
            k_search_i8<false><<<grid, 256, 0, s>>>(W, N, K, had, static_cast<int8_t*>(codes),
                                                    static_cast<uint16_t*>(scales));
            return cudaGetLastError();
        case QL_I8_G128_F16:
            k_search_i8<true><<<grid, 256, 0, s>>>(W, N, K, had, static_cast<int8_t*>(codes),
                                                   static_cast<uint16_t*>(scales));
            return cudaGetLastError();
        default:
            return cudaErrorNotSupported;
        }
    }
    switch (fmt) {
    case QL_I8_G128_BF16:
    case QL_I8A8_G128_BF16:
        k_rtn_i8<false><<<grid, 256, 0, s>>>(W, N, K, had, static_cast<int8_t*>(codes), static_cast<uint16_t*>(scales));
        break;
    case QL_I8_G128_F16:
        k_rtn_i8<true><<<grid, 256, 0, s>>>(W, N, K, had, static_cast<int8_t*>(codes), static_cast<uint16_t*>(scales));
        break;
    case QL_I4_G64_BF16:
        k_rtn_i4<<<grid, 256, 0, s>>>(W, N, K, had, static_cast<uint8_t*>(codes), static_cast<uint16_t*>(scales));
        break;
    case QL_FP8_B128_BF16:
    case QL_FP8A8_B128_BF16: {
        const int smem = 128 * 128 * sizeof(float);
        e = cudaFuncSetAttribute(k_rtn_fp8, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        dim3 grid2((N + 127) / 128, K / 128);
        k_rtn_fp8<<<grid2, 256, smem, s>>>(W, N, K, had, static_cast<uint8_t*>(codes), static_cast<uint16_t*>(scales));
        break;
    }
    default:
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_pack_codes(const void* codes_in, int fmt, int N, int K, void* codes_out, unsigned* err,
                              cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    const long long n8 = (long long)N * K / 8;
    const int grid = blocks_for(n8, 256, di.sm_count);
    const uint8_t* in = static_cast<const uint8_t*>(codes_in);
    uint8_t* out = static_cast<uint8_t*>(codes_out);
    switch (fmt) {
    case QL_I4_G64_BF16: k_pack_codes<QL_I4_G64_BF16><<<grid, 256, 0, s>>>(in, n8, out, err); break;
    case QL_I5Z_G128_F16: k_pack_codes<QL_I5Z_G128_F16><<<grid, 256, 0, s>>>(in, n8, out, err); break;
    case QL_FP8_B128_BF16:
    case QL_FP8A8_B128_BF16: k_pack_codes<QL_FP8_B128_BF16><<<grid, 256, 0, s>>>(in, n8, out, err); break;
    default: k_pack_codes<QL_I8_G128_BF16><<<grid, 256, 0, s>>>(in, n8, out, err); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_check_zeros(const uint8_t* z_in, size_t n, uint8_t* z_out, unsigned* err, cudaStream_t s) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return e;
    k_check_zeros<<<blocks_for((long long)n, 256, di.sm_count), 256, 0, s>>>(z_in, (long long)n, z_out, err);
    return cudaGetLastError();
}

}  // namespace ql
