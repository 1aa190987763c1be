// ql_api.cu -- the C ABI of libqlinear.so (declared in include/qlinear.h):
// argument validation on the host, workspace carving, and the launch order
// of the kernels of each call.  Every check happens before the first launch;
// a rejected call enqueues nothing.
#include <cstring>
#include <new>

#include "ql_internal.h"

namespace ql {

// The per-process device state (one per device context): [0] the error word,
// [2..3] the pipeline wait limit in ns as a 64-bit value (0: the default).
__device__ __align__(16) unsigned g_ql_state[4];

void packed_sizes(int fmt, size_t N, size_t K, size_t* codes, size_t* scales, size_t* zeros) {
    *codes = N * fmt_row_bytes(fmt, K);
    *zeros = fmt == QL_I5Z_G128_F16 ? N * (K / 128) : 0;
    if (fmt_fp8_weights(fmt)) *scales = ((N + 127) / 128) * (K / 128) * 2;
    else *scales = N * (K / fmt_group(fmt)) * 2;
}

cudaError_t device_info(DeviceInfo* out) {
    static DeviceInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && have[dev]) {
        *out = cache[dev];
        return cudaSuccess;
    }
    DeviceInfo d;
    int v = 0;
    if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    d.sm_count = v;
    if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
    d.smem_optin = (size_t)v;
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_ql_state)) != cudaSuccess) return e;
    d.err_word = static_cast<unsigned*>(p);
    if (dev < 64) {
        cache[dev] = d;
        have[dev] = true;
    }
    *out = d;
    return cudaSuccess;
}

// ---- launch trace -------------------------------------------------------------------
namespace {
struct TraceSlot {
    int kind;
    bool ok;  // both events recorded
    cudaEvent_t start, stop;
};
TraceSlot* g_slots = nullptr;
int g_capacity = 0, g_used = 0;

void trace_free() {
    for (int i = 0; i < g_capacity; ++i) {
        cudaEventDestroy(g_slots[i].start);
        cudaEventDestroy(g_slots[i].stop);
    }
    delete[] g_slots;
    g_slots = nullptr;
    g_capacity = g_used = 0;
}
}  // namespace

namespace {
// Under stream capture the record must be an external event node of the graph;
// outside capture it is a plain record.  A failed record is cleared (so it
// cannot surface at the next launch check) and reported as false.
bool trace_record(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
        cudaGetLastError();
        cs = cudaStreamCaptureStatusNone;
    }
    const cudaError_t e = cs == cudaStreamCaptureStatusActive
                              ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
                              : cudaEventRecord(ev, s);
    if (e != cudaSuccess) cudaGetLastError();
    return e == cudaSuccess;
}
}  // namespace

int trace_begin(int kind, cudaStream_t s) {
    if (g_used >= g_capacity) return -1;
    const int slot = g_used++;
    g_slots[slot].kind = kind;
    g_slots[slot].ok = trace_record(g_slots[slot].start, s);
    return slot;
}

void trace_end(int slot, cudaStream_t s) {
    if (slot >= 0) g_slots[slot].ok = trace_record(g_slots[slot].stop, s) && g_slots[slot].ok;
}

}  // namespace ql

using namespace ql;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
thread_local cudaError_t g_last_cuda = cudaSuccess;  // reported by ql_last_cuda_error
int from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return QL_OK;
    g_last_cuda = e;
    return QL_ECUDA;
}

// Activations prepared for the GEMM: f16 [M][K] + factors [M] (A16), or
// int8 [M][K] + fp32 scales [M][K/128] (W8A8); for the tensor-core W8A8 GEMM
// the scales are stored transposed, [K/128][M padded to the tile], followed by
// the GEMM's own scratch.
struct FwdWs {
    size_t x_bytes, f_bytes, g_bytes;
    size_t total() const { return x_bytes + f_bytes + g_bytes; }
};
FwdWs forward_ws(int fmt, size_t M, size_t N, size_t K) {
    FwdWs w;
    w.g_bytes = 0;
    if (fmt == QL_FP8A8_B128_BF16 && M >= (size_t)kPrefillMinM) {
        // E4M3 codes, transposed scales, the GEMM's weight scales
        w.x_bytes = align_up(M * K, 256);
        w.f_bytes = align_up((K / 128) * prefill_pad_m((int)M) * 4, 256);
        w.g_bytes = prefill_scratch_bytes((int)N, (int)K);
    } else if (fmt == QL_FP8A8_B128_BF16) {  // decode: E4M3 codes and their scales [M][K/128]
        w.x_bytes = align_up(M * K, 256);
        w.f_bytes = align_up(M * (K / 128) * 4, 256);
    } else if (fmt == QL_I5Z_G128_F16 && M >= (size_t)kW5A8MinM) {
        // int8 activation codes, transposed scales, then the GEMM's weight scales and the
        // weight codes converted to int8 (q - z)
        w.x_bytes = align_up(M * K, 256);
        w.f_bytes = align_up((K / 128) * prefill_pad_m((int)M) * 4, 256);
        w.g_bytes = prefill_scratch_bytes((int)N, (int)K) + align_up(N * K, 256);
    } else if (fmt == QL_I8A8_G128_BF16) {
        w.x_bytes = align_up(M * K, 256);
        if (M >= (size_t)kPrefillMinM) {
            w.f_bytes = align_up((K / 128) * prefill_pad_m((int)M) * 4, 256);
            w.g_bytes = prefill_scratch_bytes((int)N, (int)K);
        } else {
            w.f_bytes = align_up(M * (K / 128) * 4, 256);
        }
    } else {
        w.x_bytes = align_up(M * K * 2, 256);
        w.f_bytes = align_up(M * 4, 256);
        // the tokens' group sums: the int5 zero point, and the int8 / int4 codes' offset in the decode
        // kernel (int4: per 64-group)
        if (fmt == QL_I5Z_G128_F16 || fmt_i8_a16(fmt)) w.g_bytes = align_up(M * (K / 128) * 4, 256);
        if (fmt == QL_I4_G64_BF16) w.g_bytes = align_up(M * (K / 64) * 4, 256);
    }
    return w;
}

int x_order(int fmt) {
    return fmt == QL_I4_G64_BF16 ? XORD_I4 : (fmt == QL_I5Z_G128_F16 ? XORD_I5 : XORD_NATURAL);
}

// The grouped tensor-core GEMM takes over once experts average this many rows.
// The grouped tensor-core path runs format-7 experts only.  The int8 / FP8 experts with 16-bit
// activations had one too (the A16 prefill kernel in grouped mode); it is withdrawn until the cause
// of an intermittent device fault seen with it is found, and those experts take the chunked
// grouped decode kernel at every batch size.
bool moe_grouped(const ql_experts* ex, int T, int topk) {
    return ex->fmt == QL_FP8A8_B128_BF16 && (long long)T * topk >= (long long)kMoePrefillMinRowsPerExpert * ex->E;
}
// Format 7 experts, grouped: the permuted rows' scales [K/128][Mp], with the 132 columns past the last
// row that a tile's 16-byte aligned scale copy may read.
int moe_e4m3_mp(int T, int topk) { return (int)align_up((size_t)T * topk + 132, 4); }
struct MoeWs {
    size_t xs, xf, xsum, counts, offsets, perm, chunks, nch, inv, tiles, sw;
    size_t max_tiles;
    size_t total;
};
MoeWs moe_ws(const ql_experts* ex, int T, int topk) {
    MoeWs w;
    size_t o = 0;
    const bool grp = moe_grouped(ex, T, topk);
    // f16 activations: one row per token (skinny GEMM) or one per (token, slot) in permuted order;
    // format 7: E4M3 codes per token and their scales [T][K/128]
    // (grouped: the permuted rows' scales transposed, [K/128][moe_e4m3_mp]; then the experts' weight
    // scales as fp32 [E][K/128][pad(N)] for the tensor-core GEMM)
    const bool e4 = ex->fmt == QL_FP8A8_B128_BF16;
    const size_t G = (size_t)ex->K / 128;
    w.xs = o; o += align_up((size_t)(grp ? T * topk : T) * ex->K * (e4 ? 1 : 2), 256);
    w.xf = o; o += align_up(e4 ? (grp ? G * moe_e4m3_mp(T, topk) * 4 : (size_t)T * G * 4) : (size_t)T * 4, 256);
    // int8 experts: each token's group sums of its f16 activations [T][K/128] (the codes' offset)
    w.xsum = 0;
    if (fmt_i8_a16(ex->fmt)) { w.xsum = o; o += align_up((size_t)T * G * 4, 256); }
    w.counts = o; o += align_up((size_t)ex->E * 4, 256);
    w.offsets = o; o += align_up(((size_t)ex->E + 1) * 4, 256);
    w.perm = o; o += align_up((size_t)T * topk * 4, 256);
    w.max_tiles = grp ? moe_max_tiles(T, topk, ex->E, kPrefillTileM, (ex->N + kPrefillTileN - 1) / kPrefillTileN) : 0;
    w.sw = 0;
    if (grp) {
        w.inv = o; o += align_up((size_t)T * topk * 4, 256);
        w.tiles = o; o += align_up(w.max_tiles * sizeof(MoeTile), 256);
        w.chunks = 0;
        if (e4) { w.sw = o; o += align_up((size_t)ex->E * G * prefill_pad_n(ex->N) * 4, 256); }
    } else {
        w.inv = w.tiles = 0;
        w.chunks = o; o += align_up(moe_max_chunks(T, topk, ex->E) * sizeof(MoeChunk), 256);
    }
    w.nch = o; o += 256;
    w.total = o;
    return w;
}

int check_experts(const ql_experts* ex) {
    if (!ex) return QL_EINVAL;
    if (ex->E < 1 || ex->E > 1024 || ex->N < 1 || ex->K < 128 || ex->K % 128) return QL_EINVAL;
    if (ex->flags & ~(QL_HADAMARD | QL_SCALE_SEARCH)) return QL_EINVAL;
    if (!fmt_valid(ex->fmt)) return QL_EINVAL;
    if (ex->fmt != QL_I8_G128_BF16 && ex->fmt != QL_I8_G128_F16 && ex->fmt != QL_FP8_B128_BF16 &&
        ex->fmt != QL_FP8A8_B128_BF16)
        return QL_EUNSUPPORTED;
    if (ex->K > QL_A16_MAX_K) return QL_EUNSUPPORTED;
    if (!ex->codes || !ex->scales) return QL_EINVAL;
    if (!aligned16(ex->codes) || !aligned16(ex->scales)) return QL_EALIGN;
    return QL_OK;
}

// moe_down_combine's workspace: the activation planes, then the permutation and either the
// weight-streaming kernel's chunks or (prefill batches) the grouped GEMM's tiles.
bool down_grouped(const ql_down_experts* ex, int T, int topk) {
    return (long long)T * topk >= (long long)kMoePrefillMinRowsPerExpert * ex->E;
}
struct DownWs {
    size_t act, counts, offsets, perm, chunks, inv, tiles, nch, max_tiles, total;
};
DownWs down_ws(const ql_down_experts* ex, int T, int topk) {
    DownWs w;
    size_t o = 0;
    const size_t P = (size_t)T * topk;
    const bool grp = down_grouped(ex, T, topk);
    w.act = o; o += align_up(P * 3 * ex->I * 2, 256);
    w.counts = o; o += align_up((size_t)ex->E * 4, 256);
    w.offsets = o; o += align_up(((size_t)ex->E + 1) * 4, 256);
    w.perm = o; o += align_up(P * 4, 256);
    w.max_tiles = grp ? moe_max_tiles(T, topk, ex->E, kDownTileRows, (ex->K + 127) / 128) : 0;
    if (grp) {
        w.chunks = 0;
        w.inv = o; o += align_up(P * 4, 256);
        w.tiles = o; o += align_up(w.max_tiles * sizeof(MoeTile), 256);
    } else {
        w.inv = w.tiles = 0;
        w.chunks = o; o += align_up(moe_max_chunks(T, topk, ex->E) * sizeof(MoeChunk), 256);
    }
    w.nch = o; o += 256;
    w.total = o;
    return w;
}

int check_down_experts(const ql_down_experts* ex) {
    if (!ex) return QL_EINVAL;
    if (ex->E < 1 || ex->E > 1024 || ex->K < 1 || ex->I < 64 || ex->I % 64) return QL_EINVAL;
    if (!ex->weights) return QL_EINVAL;
    if (!aligned16(ex->weights)) return QL_EALIGN;
    return QL_OK;
}

}  // namespace

extern "C" {

const char* ql_status_string(int status) {
    switch (status) {
    case QL_OK: return "ok";
    case QL_EINVAL: return "invalid argument";
    case QL_EUNSUPPORTED: return "unsupported format or mode";
    case QL_EALIGN: return "device pointer not 16-byte aligned";
    case QL_EWORKSPACE: return "workspace missing or too small";
    case QL_ECUDA: return "CUDA runtime error";
    case QL_EDEVICE: return "device error word set";
    }
    return "unknown status";
}

int qlinear_packed_sizes(int fmt, int N, int K, size_t* codes_bytes, size_t* scales_bytes, size_t* zeros_bytes) {
    if (!fmt_valid(fmt) || N < 1 || K < 128 || K % 128 || !codes_bytes || !scales_bytes || !zeros_bytes)
        return QL_EINVAL;
    packed_sizes(fmt, (size_t)N, (size_t)K, codes_bytes, scales_bytes, zeros_bytes);
    return QL_OK;
}

int qlinear_pack(const float* W, const void* codes_in, const void* scales_in, const uint8_t* zeros_in, int fmt,
                 int flags, int N, int K, void* codes_out, void* scales_out, uint8_t* zeros_out, void* stream) {
    if (!fmt_valid(fmt) || N < 1 || K < 128 || K % 128 || (flags & ~(QL_HADAMARD | QL_SCALE_SEARCH)))
        return QL_EINVAL;
    if (!codes_out || !scales_out) return QL_EINVAL;
    if ((W == nullptr) == (codes_in == nullptr)) return QL_EINVAL;  // exactly one source
    if (flags & QL_SCALE_SEARCH) {  // a rule for quantising W, int8 formats only
        if (!W) return QL_EINVAL;
        if (fmt != QL_I8_G128_BF16 && fmt != QL_I8_G128_F16 && fmt != QL_I8A8_G128_BF16) return QL_EUNSUPPORTED;
    }
    if (!aligned16(codes_out) || !aligned16(scales_out)) return QL_EALIGN;
    if (fmt == QL_I5Z_G128_F16) {
        if (!zeros_out) return QL_EINVAL;
        if (!aligned16(zeros_out)) return QL_EALIGN;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    size_t cb, sb, zb;
    packed_sizes(fmt, N, K, &cb, &sb, &zb);
    if (W) {
        if (!aligned16(W)) return QL_EALIGN;
        if (fmt == QL_I5Z_G128_F16) return QL_EUNSUPPORTED;
        const int t = trace_begin(QL_KIND_PACK, s);
        const cudaError_t e = launch_pack_rtn(W, fmt, flags, N, K, codes_out, scales_out, s);
        trace_end(t, s);
        return from_cuda(e);
    }
    if (!scales_in) return QL_EINVAL;
    if (!aligned16(codes_in) || !aligned16(scales_in)) return QL_EALIGN;
    if (fmt == QL_I5Z_G128_F16) {
        if (!zeros_in) return QL_EINVAL;
        if (!aligned16(zeros_in)) return QL_EALIGN;
    }
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return from_cuda(e);
    int t = trace_begin(QL_KIND_PACK, s);
    e = launch_pack_codes(codes_in, fmt, N, K, codes_out, di.err_word, s);
    trace_end(t, s);
    if (e != cudaSuccess) return from_cuda(e);
    if ((e = cudaMemcpyAsync(scales_out, scales_in, sb, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
        return from_cuda(e);
    if (fmt == QL_I5Z_G128_F16) {
        t = trace_begin(QL_KIND_PACK, s);
        e = launch_check_zeros(zeros_in, zb, zeros_out, di.err_word, s);
        trace_end(t, s);
        return from_cuda(e);
    }
    return QL_OK;
}

int qlinear_workspace_size(int fmt, int flags, int M, int N, int K, size_t* bytes) {
    if (!fmt_valid(fmt) || M < 1 || N < 1 || K < 128 || K % 128 || (flags & ~(QL_HADAMARD | QL_SCALE_SEARCH)) ||
        !bytes)
        return QL_EINVAL;
    *bytes = forward_ws(fmt, M, N, K).total();
    return QL_OK;
}

int qlinear_forward(const void* x, const void* W_packed, const void* scales, const uint8_t* zeros, int fmt,
                    int flags, int M, int N, int K, float* y, void* ws, size_t ws_bytes, void* stream) {
    if (!fmt_valid(fmt) || M < 1 || N < 1 || K < 128 || K % 128 || (flags & ~(QL_HADAMARD | QL_SCALE_SEARCH)))
        return QL_EINVAL;
    if (!x || !W_packed || !scales || !y) return QL_EINVAL;
    if (fmt == QL_I5Z_G128_F16 && !zeros) return QL_EINVAL;
    const bool a8 = fmt == QL_I8A8_G128_BF16 || fmt == QL_FP8A8_B128_BF16 || (fmt == QL_I5Z_G128_F16 && M >= kW5A8MinM);
    if (!a8 && K > QL_A16_MAX_K) return QL_EUNSUPPORTED;
    if (!aligned16(x) || !aligned16(W_packed) || !aligned16(scales) || !aligned16(y) ||
        (zeros && !aligned16(zeros)))
        return QL_EALIGN;
    const FwdWs w = forward_ws(fmt, M, N, K);
    if (!ws || ws_bytes < w.total()) return QL_EWORKSPACE;
    if (!aligned16(ws)) return QL_EALIGN;
    if (skinny_max_k(fmt) < 128) return QL_ECUDA;
    // One decode launch per 16-row block covers the whole K: the kernel orders its
    // units by K part and each CTA stages only the parts its unit range touches.
    const int kmax = K;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int G = K / 128;
    const int rot = (flags & QL_HADAMARD) ? 1 : 0;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    void* xs = wsb;
    float* xf = reinterpret_cast<float*>(wsb + w.x_bytes);
    cudaError_t e;
    if (fmt == QL_FP8A8_B128_BF16 && M >= kPrefillMinM) {  // E4M3 activations, the tensor-core E4M3 GEMM
        int t = trace_begin(QL_KIND_ACT_QUANT, s);
        e = launch_act_quant_e4m3(x, M, K, rot, static_cast<uint8_t*>(xs), nullptr, xf, prefill_pad_m(M), nullptr, 0, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        uint8_t* const gs = wsb + w.x_bytes + w.f_bytes;
        t = trace_begin(QL_KIND_PREFILL_PREP, s);
        e = launch_prefill_prep_blk(static_cast<const uint16_t*>(scales), N, K, gs, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        t = trace_begin(QL_KIND_PREFILL, s);
        e = launch_prefill_w8a8(static_cast<const int8_t*>(xs), xf, static_cast<const int8_t*>(W_packed), M, N, K, y,
                                N, nullptr, gs, s, true);
        trace_end(t, s);
        return from_cuda(e);
    }
    if (fmt == QL_I5Z_G128_F16 && M >= kW5A8MinM) {  // W5A8: int8 activations, the W8A8 tensor-core GEMM
        int t = trace_begin(QL_KIND_ACT_QUANT, s);
        e = launch_act_quant(x, M, K, rot, static_cast<int8_t*>(xs), nullptr, xf, prefill_pad_m(M), nullptr, 0, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        uint8_t* const gs = wsb + w.x_bytes + w.f_bytes;
        int8_t* const q8 = reinterpret_cast<int8_t*>(gs + prefill_scratch_bytes(N, K));
        t = trace_begin(QL_KIND_PREFILL_PREP, s);
        e = launch_prefill_prep(static_cast<const uint16_t*>(scales), N, K, gs, s, true);
        if (e == cudaSuccess) e = launch_prefill_i5_codes(static_cast<const uint8_t*>(W_packed), zeros, N, K, q8, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        t = trace_begin(QL_KIND_PREFILL, s);
        e = launch_prefill_w8a8(static_cast<const int8_t*>(xs), xf, q8, M, N, K, y, N, nullptr, gs, s);
        trace_end(t, s);
        return from_cuda(e);
    }
    if (fmt == QL_I8A8_G128_BF16 && M >= kPrefillMinM) {  // tensor-core GEMM, y written directly
        int t = trace_begin(QL_KIND_ACT_QUANT, s);
        e = launch_act_quant(x, M, K, rot, static_cast<int8_t*>(xs), nullptr, xf, prefill_pad_m(M), nullptr, 0, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        uint8_t* const gs = wsb + w.x_bytes + w.f_bytes;
        t = trace_begin(QL_KIND_PREFILL_PREP, s);
        e = launch_prefill_prep(static_cast<const uint16_t*>(scales), N, K, gs, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        t = trace_begin(QL_KIND_PREFILL, s);
        e = launch_prefill_w8a8(static_cast<const int8_t*>(xs), xf, static_cast<const int8_t*>(W_packed), M, N, K, y,
                                N, nullptr, gs, s);
        trace_end(t, s);
        return from_cuda(e);
    }
    if (M >= kPrefillMinM && prefill_a16_supported(fmt)) {  // tensor-core GEMM, y written directly
        int t = trace_begin(QL_KIND_PREP_A16, s);
        e = launch_prep_a16(x, M, K, rot, XORD_NATURAL, static_cast<__half*>(xs), xf, nullptr, 0, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        t = trace_begin(QL_KIND_PREFILL, s);
        e = launch_prefill_a16(fmt, static_cast<const __half*>(xs), xf, static_cast<const uint8_t*>(W_packed), scales,
                               M, N, K, y, N, s);
        trace_end(t, s);
        return from_cuda(e);
    }
    const long long ny = (long long)M * N;  // the prologue zeroes y for the accumulating GEMM
    float* const xsum = (fmt == QL_I5Z_G128_F16 || fmt == QL_I4_G64_BF16 || fmt_i8_a16(fmt))
                            ? reinterpret_cast<float*>(wsb + w.x_bytes + w.f_bytes)
                            : nullptr;
    if (fmt == QL_I8A8_G128_BF16) {
        const int t = trace_begin(QL_KIND_ACT_QUANT, s);
        e = launch_act_quant(x, M, K, rot, static_cast<int8_t*>(xs), xf, nullptr, 0, y, ny, s);
        trace_end(t, s);
    } else if (fmt == QL_FP8A8_B128_BF16) {
        const int t = trace_begin(QL_KIND_ACT_QUANT, s);
        e = launch_act_quant_e4m3(x, M, K, rot, static_cast<uint8_t*>(xs), xf, nullptr, 0, y, ny, s);
        trace_end(t, s);
    } else {
        const int t = trace_begin(QL_KIND_PREP_A16, s);
        e = launch_prep_a16(x, M, K, rot, x_order(fmt), static_cast<__half*>(xs), xf, y, ny, s, xsum);
        trace_end(t, s);
    }
    if (e != cudaSuccess) return from_cuda(e);

    const bool act8 = fmt == QL_I8A8_G128_BF16 || fmt == QL_FP8A8_B128_BF16;  // byte activations, scales [M][G]
    const size_t xelem = act8 ? 1 : 2;
    for (int m0 = 0; m0 < M; m0 += 16) {
        for (int k0 = 0; k0 < K; k0 += kmax) {
            const int kc = K - k0 < kmax ? K - k0 : kmax;
            SkinnyArgs a;
            a.W = static_cast<const uint8_t*>(W_packed) + fmt_row_bytes(fmt, k0);
            a.scales = scales;
            a.zeros = zeros;
            a.xs = static_cast<const uint8_t*>(xs) + ((size_t)m0 * K + k0) * xelem;
            a.xf = act8 ? xf + (size_t)m0 * G : xf + m0;
            a.xsum = xsum ? xsum + (size_t)m0 * G * (fmt == QL_I4_G64_BF16 ? 2 : 1) : nullptr;
            a.y = y + (size_t)m0 * N;
            a.acc = nullptr;
            a.M = M - m0 < 16 ? M - m0 : 16;
            a.N = N;
            a.G = kc / 128;
            a.g0 = k0 / 128;
            a.Gtot = G;
            a.ldw = (long long)fmt_row_bytes(fmt, K);
            a.ldx = K;
            a.ldy = N;
            a.pdl = 1;  // preceded by this call's prologue (or the previous K chunk)
            const int t = trace_begin(QL_KIND_SKINNY, s);
            e = launch_skinny(fmt, a, s);
            trace_end(t, s);
            if (e != cudaSuccess) return from_cuda(e);
        }
    }
    return QL_OK;
}

int qlinear_forward_i8_acc(const int8_t* qx, const int8_t* qw, int M, int N, int K, int32_t* acc, void* stream) {
    if (M < 1 || N < 1 || K < 128 || K % 128 || !qx || !qw || !acc) return QL_EINVAL;
    if (!aligned16(qx) || !aligned16(qw) || !aligned16(acc)) return QL_EALIGN;
    if (skinny_max_k(QL_I8A8_G128_BF16) < 128) return QL_ECUDA;
    const int kmax = K;  // one launch per 16-row block (see qlinear_forward)
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int G = K / 128;
    if (M >= kPrefillMinM) {  // the same tensor-core GEMM qlinear_forward runs at this M
        const int t = trace_begin(QL_KIND_PREFILL, s);
        const cudaError_t e = launch_prefill_w8a8(qx, nullptr, qw, M, N, K, nullptr, N, acc, nullptr, s);
        trace_end(t, s);
        return from_cuda(e);
    }
    for (int m0 = 0; m0 < M; m0 += 16) {
        for (int k0 = 0; k0 < K; k0 += kmax) {
            const int kc = K - k0 < kmax ? K - k0 : kmax;
            SkinnyArgs a;
            std::memset(&a, 0, sizeof a);
            a.W = reinterpret_cast<const uint8_t*>(qw) + k0;
            a.xs = qx + (size_t)m0 * K + k0;
            a.xf = nullptr;
            a.acc = acc + (size_t)m0 * N * G;
            a.M = M - m0 < 16 ? M - m0 : 16;
            a.N = N;
            a.G = kc / 128;
            a.g0 = k0 / 128;
            a.Gtot = G;
            a.ldw = K;
            a.ldx = K;
            a.ldy = N;
            const int t = trace_begin(QL_KIND_SKINNY, s);
            cudaError_t e = launch_skinny(QL_I8A8_G128_BF16, a, s);
            trace_end(t, s);
            if (e != cudaSuccess) return from_cuda(e);
        }
    }
    return QL_OK;
}

int qlinear_gemm_a8(const void* qx, const float* sx, const void* W_packed, const void* scales, int fmt, int M, int N,
                    int K, float* y, int accumulate, void* stream) {
    if ((fmt != QL_I8A8_G128_BF16 && fmt != QL_FP8A8_B128_BF16) || M < 1 || N < 1 || K < 128 || K % 128)
        return QL_EINVAL;
    if (!qx || !sx || !W_packed || !scales || !y) return QL_EINVAL;
    if (M > 16) return QL_EUNSUPPORTED;
    if (!aligned16(qx) || !aligned16(sx) || !aligned16(W_packed) || !aligned16(scales) || !aligned16(y))
        return QL_EALIGN;
    if (skinny_max_k(fmt) < 128) return QL_ECUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!accumulate) {
        const cudaError_t e = cudaMemsetAsync(y, 0, (size_t)M * N * sizeof(float), s);
        if (e != cudaSuccess) return from_cuda(e);
    }
    const int G = K / 128;
    SkinnyArgs a;
    a.W = static_cast<const uint8_t*>(W_packed);
    a.scales = scales;
    a.zeros = nullptr;
    a.xs = qx;
    a.xf = sx;
    a.y = y;
    a.acc = nullptr;
    a.M = M;
    a.N = N;
    a.G = G;
    a.g0 = 0;
    a.Gtot = G;
    a.ldw = K;
    a.ldx = K;
    a.ldy = N;
    a.pdl = 1;  // waits for the kernel before it before reading qx, sx or y
    const int t = trace_begin(QL_KIND_SKINNY, s);
    const cudaError_t e = launch_skinny(fmt, a, s);
    trace_end(t, s);
    return from_cuda(e);
}

int act_quant_i8_g128(const void* x, int M, int K, int rotate, int8_t* q, float* s, void* stream) {
    if (M < 1 || K < 128 || K % 128 || !x || !q || !s) return QL_EINVAL;
    if (!aligned16(x) || !aligned16(q) || !aligned16(s)) return QL_EALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int t = trace_begin(QL_KIND_ACT_QUANT, st);
    const cudaError_t e = launch_act_quant(x, M, K, rotate ? 1 : 0, q, s, nullptr, 0, nullptr, 0, st);
    trace_end(t, st);
    return from_cuda(e);
}

int act_quant_e4m3_g128(const void* x, int M, int K, int rotate, uint8_t* q, float* s, void* stream) {
    if (M < 1 || K < 128 || K % 128 || !x || !q || !s) return QL_EINVAL;
    if (!aligned16(x) || !aligned16(q) || !aligned16(s)) return QL_EALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int t = trace_begin(QL_KIND_ACT_QUANT, st);
    const cudaError_t e = launch_act_quant_e4m3(x, M, K, rotate ? 1 : 0, q, s, nullptr, 0, nullptr, 0, st);
    trace_end(t, st);
    return from_cuda(e);
}

int hadamard128_rotate(const void* x, int M, int K, void* y, void* stream) {
    if (M < 1 || K < 128 || K % 128 || !x || !y) return QL_EINVAL;
    if (!aligned16(x) || !aligned16(y)) return QL_EALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int t = trace_begin(QL_KIND_ROTATE, st);
    const cudaError_t e = launch_rotate_bf16(x, M, K, y, st);
    trace_end(t, st);
    return from_cuda(e);
}

int moe_permute(const int32_t* topk_ids, int T, int topk, int E, int32_t* counts, int32_t* offsets, int32_t* perm,
                void* stream) {
    if (T < 1 || topk < 1 || topk > 64 || E < 1 || E > 1024 || !topk_ids || !counts || !offsets || !perm)
        return QL_EINVAL;
    if (!aligned16(topk_ids) || !aligned16(counts) || !aligned16(offsets) || !aligned16(perm)) return QL_EALIGN;
    // Standalone permutation: the chunk table the grouped GEMM uses is not requested.
    DeviceInfo di;
    if (device_info(&di) != cudaSuccess) return QL_ECUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int t = trace_begin(QL_KIND_MOE_PERMUTE, st);
    const cudaError_t e = launch_moe_permute(topk_ids, T, topk, E, counts, offsets, perm, MoePermuteOut{}, di.err_word, st);
    trace_end(t, st);
    return from_cuda(e);
}

int moe_workspace_size(const ql_experts* experts, int T, int topk, size_t* bytes) {
    int st = check_experts(experts);
    if (st != QL_OK) return st;
    if (T < 1 || topk < 1 || topk > 64 || !bytes) return QL_EINVAL;
    *bytes = moe_ws(experts, T, topk).total;
    return QL_OK;
}

int moe_gate_up(const void* x, const int32_t* topk_ids, const float* topk_weights, const ql_experts* experts, int T,
                int topk, float* y, void* ws, size_t ws_bytes, void* stream) {
    (void)topk_weights;  // applied after the down projection, not here
    int st = check_experts(experts);
    if (st != QL_OK) return st;
    if (T < 1 || topk < 1 || topk > 64 || !x || !topk_ids || !y) return QL_EINVAL;
    if (!aligned16(x) || !aligned16(topk_ids) || !aligned16(y)) return QL_EALIGN;
    const MoeWs w = moe_ws(experts, T, topk);
    if (!ws || ws_bytes < w.total) return QL_EWORKSPACE;
    if (!aligned16(ws)) return QL_EALIGN;
    DeviceInfo di;
    if (device_info(&di) != cudaSuccess) return QL_ECUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* b = static_cast<uint8_t*>(ws);
    __half* xs = reinterpret_cast<__half*>(b + w.xs);
    float* xf = reinterpret_cast<float*>(b + w.xf);
    float* xsum = fmt_i8_a16(experts->fmt) ? reinterpret_cast<float*>(b + w.xsum) : nullptr;
    int32_t* counts = reinterpret_cast<int32_t*>(b + w.counts);
    int32_t* offsets = reinterpret_cast<int32_t*>(b + w.offsets);
    int32_t* perm = reinterpret_cast<int32_t*>(b + w.perm);
    MoeChunk* chunks = reinterpret_cast<MoeChunk*>(b + w.chunks);
    int* nch = reinterpret_cast<int*>(b + w.nch);
    const int K = experts->K, N = experts->N;
    const int rot = (experts->flags & QL_HADAMARD) ? 1 : 0;
    cudaError_t e;
    if (moe_grouped(experts, T, topk)) {  // format 7
        // permute; E4M3 codes and scales straight into permuted order; the experts' weight scales
        // as fp32; the grouped E4M3 tensor-core GEMM with the un-permute in its stores
        MoePermuteOut po;
        po.inv = reinterpret_cast<int32_t*>(b + w.inv);
        po.tiles = reinterpret_cast<MoeTile*>(b + w.tiles);
        po.n_tiles = nch;
        po.tile_rows = kPrefillTileM;
        po.wblocks = (N + kPrefillTileN - 1) / kPrefillTileN;
        po.yz = y;  // rows of pairs with a bad expert id are zeroed
        po.N = N;
        int t = trace_begin(QL_KIND_MOE_PERMUTE, s);
        e = launch_moe_permute(topk_ids, T, topk, experts->E, counts, offsets, perm, po, di.err_word, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        const int Mp = moe_e4m3_mp(T, topk);
        t = trace_begin(QL_KIND_ACT_QUANT, s);
        e = launch_act_quant_e4m3(x, T, K, rot, reinterpret_cast<uint8_t*>(xs), nullptr, xf, Mp, nullptr, 0, s,
                                  po.inv, topk);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        float* swT = reinterpret_cast<float*>(b + w.sw);
        t = trace_begin(QL_KIND_PREFILL_PREP, s);
        e = launch_prefill_prep_blk(static_cast<const uint16_t*>(experts->scales), N, K, swT, s, experts->E);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        t = trace_begin(QL_KIND_MOE_GEMM, s);
        e = launch_prefill_e4m3_grouped(reinterpret_cast<const uint8_t*>(xs), xf, Mp,
                                        static_cast<const uint8_t*>(experts->codes), swT, experts->E, N, K, T * topk,
                                        po.tiles, nch, (int)w.max_tiles, perm, y, s);
        trace_end(t, s);
        return from_cuda(e);
    }
    int t;
    if (experts->fmt == QL_FP8A8_B128_BF16) {  // rotation, E4M3 codes and scales per token, the zeroing of y
        t = trace_begin(QL_KIND_ACT_QUANT, s);
        e = launch_act_quant_e4m3(x, T, K, rot, reinterpret_cast<uint8_t*>(xs), xf, nullptr, 0, y,
                                  (long long)T * topk * N, s);
    } else {  // rotation, f16 staging, and the zeroing of y
        t = trace_begin(QL_KIND_PREP_A16, s);
        e = launch_prep_a16(x, T, K, rot, XORD_NATURAL, xs, xf, y, (long long)T * topk * N, s, xsum);
    }
    trace_end(t, s);
    if (e != cudaSuccess) return from_cuda(e);
    // Small batches: the expert GEMM ranks the ids itself (no permute launch).
    const bool fused = (long long)T * topk <= kMoeFusedMaxPairs;
    if (!fused) {
        t = trace_begin(QL_KIND_MOE_PERMUTE, s);
        MoePermuteOut po;
        po.chunks = chunks;
        po.n_chunks = nch;
        e = launch_moe_permute(topk_ids, T, topk, experts->E, counts, offsets, perm, po, di.err_word, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
    }
    MoeArgs a;
    a.codes = static_cast<const uint8_t*>(experts->codes);
    a.scales = experts->scales;
    a.xs = xs;
    a.xf = xf;
    a.xsum = xsum;
    a.perm = perm;
    a.chunks = chunks;
    a.n_chunks = nch;
    a.ids = fused ? topk_ids : nullptr;
    a.y = y;
    a.fmt = experts->fmt;
    a.T = T;
    a.topk = topk;
    a.E = experts->E;
    a.N = N;
    a.K = K;
    a.max_chunks = (long long)moe_max_chunks(T, topk, experts->E);
    t = trace_begin(QL_KIND_MOE_GEMM, s);
    e = launch_moe_skinny(a, s);
    trace_end(t, s);
    return from_cuda(e);
}

int moe_down_workspace_size(const ql_down_experts* experts, int T, int topk, size_t* bytes) {
    const int st = check_down_experts(experts);
    if (st != QL_OK) return st;
    if (T < 1 || topk < 1 || topk > 64 || !bytes) return QL_EINVAL;
    *bytes = down_ws(experts, T, topk).total;
    return QL_OK;
}

int moe_down_combine(const float* h, const int32_t* topk_ids, const float* topk_weights,
                     const ql_down_experts* experts, int T, int topk, float* out, void* ws, size_t ws_bytes,
                     void* stream) {
    int st = check_down_experts(experts);
    if (st != QL_OK) return st;
    if (T < 1 || topk < 1 || topk > 64 || !h || !topk_ids || !topk_weights || !out) return QL_EINVAL;
    if (!aligned16(h) || !aligned16(topk_ids) || !aligned16(topk_weights) || !aligned16(out)) return QL_EALIGN;
    const DownWs w = down_ws(experts, T, topk);
    if (!ws || ws_bytes < w.total) return QL_EWORKSPACE;
    if (!aligned16(ws)) return QL_EALIGN;
    DeviceInfo di;
    if (device_info(&di) != cudaSuccess) return QL_ECUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* b = static_cast<uint8_t*>(ws);
    __nv_bfloat16* act = reinterpret_cast<__nv_bfloat16*>(b + w.act);
    int32_t* counts = reinterpret_cast<int32_t*>(b + w.counts);
    int32_t* offsets = reinterpret_cast<int32_t*>(b + w.offsets);
    int32_t* perm = reinterpret_cast<int32_t*>(b + w.perm);
    MoeChunk* chunks = reinterpret_cast<MoeChunk*>(b + w.chunks);
    int* nch = reinterpret_cast<int*>(b + w.nch);
    const int P = T * topk;
    if (down_grouped(experts, T, topk)) {
        // permute into tiles of up to 160 rows; the planes straight into permuted order (and out
        // zeroed); the grouped bf16 tensor-core GEMM adds each pair's share into its token's row
        MoePermuteOut po;
        po.inv = reinterpret_cast<int32_t*>(b + w.inv);
        po.tiles = reinterpret_cast<MoeTile*>(b + w.tiles);
        po.n_tiles = nch;
        po.tile_rows = kDownTileRows;
        po.wblocks = (experts->K + 127) / 128;
        int t = trace_begin(QL_KIND_MOE_PERMUTE, s);
        cudaError_t e = launch_moe_permute(topk_ids, T, topk, experts->E, counts, offsets, perm, po, di.err_word, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        t = trace_begin(QL_KIND_MOE_ACT, s);
        e = launch_moe_act(h, topk_ids, P, experts->E, experts->I, act, out, (long long)T * experts->K, s, po.inv);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
        t = trace_begin(QL_KIND_MOE_DOWN, s);
        e = launch_down_grouped(act, static_cast<const uint16_t*>(experts->weights), experts->E, experts->K,
                                experts->I, P, po.tiles, nch, (int)w.max_tiles, perm, topk, topk_weights, out, s);
        trace_end(t, s);
        return from_cuda(e);
    }
    // gelu(gate) * up as three bf16 planes, and the zeroing of out
    int t = trace_begin(QL_KIND_MOE_ACT, s);
    cudaError_t e = launch_moe_act(h, topk_ids, P, experts->E, experts->I, act, out, (long long)T * experts->K, s);
    trace_end(t, s);
    if (e != cudaSuccess) return from_cuda(e);
    // Small batches: the expert GEMM ranks the ids itself (no permute launch).
    const bool fused = P <= kMoeFusedMaxPairs;
    if (!fused) {
        MoePermuteOut po;
        po.chunks = chunks;
        po.n_chunks = nch;
        t = trace_begin(QL_KIND_MOE_PERMUTE, s);
        e = launch_moe_permute(topk_ids, T, topk, experts->E, counts, offsets, perm, po, di.err_word, s);
        trace_end(t, s);
        if (e != cudaSuccess) return from_cuda(e);
    }
    MoeArgs a;
    a.codes = static_cast<const uint8_t*>(experts->weights);
    a.scales = nullptr;
    a.xs = act;
    a.xf = nullptr;
    a.perm = perm;
    a.chunks = chunks;
    a.n_chunks = nch;
    a.ids = fused ? topk_ids : nullptr;
    a.y = out;
    a.wts = topk_weights;
    a.fmt = 0;
    a.T = T;
    a.topk = topk;
    a.E = experts->E;
    a.N = experts->K;
    a.K = experts->I;
    a.max_chunks = (long long)moe_max_chunks(T, topk, experts->E);
    t = trace_begin(QL_KIND_MOE_DOWN, s);
    e = launch_moe_down(a, s);
    trace_end(t, s);
    return from_cuda(e);
}

int ql_trace_enable(int capacity) {
    if (capacity < 0 || capacity > (1 << 20)) return QL_EINVAL;
    trace_free();
    if (capacity == 0) return QL_OK;
    g_slots = new (std::nothrow) TraceSlot[capacity];
    if (!g_slots) return QL_EINVAL;
    for (int i = 0; i < capacity; ++i) {
        if (cudaEventCreate(&g_slots[i].start) != cudaSuccess || cudaEventCreate(&g_slots[i].stop) != cudaSuccess) {
            g_capacity = i;
            trace_free();
            return QL_ECUDA;
        }
    }
    g_capacity = capacity;
    g_used = 0;
    return QL_OK;
}

int ql_trace_read(int* kinds, float* ms, int max, int* count) {
    if (!count || max < 0 || (max > 0 && (!kinds || !ms))) return QL_EINVAL;
    const int n = g_used < max ? g_used : max;
    for (int i = 0; i < n; ++i) {
        float t = -1.0f;  // -1: the slot's events were not recorded
        if (g_slots[i].ok) {
            if (cudaEventSynchronize(g_slots[i].stop) != cudaSuccess) return QL_ECUDA;
            if (cudaEventElapsedTime(&t, g_slots[i].start, g_slots[i].stop) != cudaSuccess) return QL_ECUDA;
        }
        kinds[i] = g_slots[i].kind;
        ms[i] = t;
    }
    *count = g_used;
    return QL_OK;
}

const char* ql_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda); }

int ql_set_wait_limit(unsigned long long ns) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return from_cuda(e);
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return from_cuda(e);
    if ((e = cudaMemcpy(di.err_word + 2, &ns, sizeof ns, cudaMemcpyHostToDevice)) != cudaSuccess) return from_cuda(e);
    return QL_OK;
}

int ql_get_device_error(void* stream, unsigned* bits) {
    DeviceInfo di;
    cudaError_t e = device_info(&di);
    if (e != cudaSuccess) return from_cuda(e);
    if ((e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream))) != cudaSuccess) return from_cuda(e);
    unsigned v = 0;
    if ((e = cudaMemcpy(&v, di.err_word, sizeof v, cudaMemcpyDeviceToHost)) != cudaSuccess) return from_cuda(e);
    if (v) {
        const unsigned zero = 0;
        if ((e = cudaMemcpy(di.err_word, &zero, sizeof zero, cudaMemcpyHostToDevice)) != cudaSuccess)
            return from_cuda(e);
    }
    if (bits) *bits = v;
    return v ? QL_EDEVICE : QL_OK;
}

}  // extern "C"
