// ql_noalloc.cu -- a W8A8 forward for callers that cannot allocate device
// memory.
//
// qlinear_forward needs a workspace for the int8 activations and their
// scales.  Some callers have no way to provide one: a plugin running inside a
// host engine that owns all device memory and forbids cudaMalloc, or a
// latency-critical loop that must never hit cudaMalloc's implicit device
// synchronisation.  This entry point keeps that scratch in a fixed array in the
// library's own device memory instead, so the caller passes only its inputs
// and outputs.
//
// The array holds int8 activations of up to QL_NOALLOC_MAX_M tokens x
// QL_NOALLOC_MAX_K values plus their fp32 scales (270,336 bytes); every GPU
// that loads the library keeps it until the process exits.  All calls share
// it: two calls whose kernels overlap on the GPU (different streams, or
// different host threads) race on it.  Nothing in it has to start at zero --
// every call rewrites the part it reads.
#include "ql_internal.h"

namespace ql {
namespace {

constexpr int kMaxM = QL_NOALLOC_MAX_M;
constexpr int kMaxK = QL_NOALLOC_MAX_K;
constexpr size_t kQxBytes = (size_t)kMaxM * kMaxK;                 // int8 activations
constexpr size_t kSxBytes = (size_t)kMaxM * (kMaxK / 128) * 4;     // fp32 scales
constexpr size_t kScratchBytes = kQxBytes + kSxBytes;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the scratch array on the current device.  In host code
// the symbol g_noalloc_scratch is only a host-side stand-in, so the kernels
// must be given this address instead.  It is looked up on every call (the
// lookup allocates nothing), so no address outlives a device reset and
// concurrent first calls from several host threads need no lock.
cudaError_t scratch_for_current_device(unsigned char** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    *out = static_cast<unsigned char*>(p);
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace ql

using namespace ql;

extern "C" int qlinear_forward_w8a8_noalloc(const void* x, const void* W_packed, const void* scales, int flags, int M,
                                            int N, int K, float* y, void* stream) {
    if (M < 1 || N < 1 || K < 128 || K % 128 || (flags & ~(QL_HADAMARD | QL_SCALE_SEARCH))) return QL_EINVAL;
    if (M > kMaxM || K > kMaxK) return QL_EUNSUPPORTED;  // larger than the fixed scratch
    if (!x || !W_packed || !scales || !y) return QL_EINVAL;
    if (!aligned16(x) || !aligned16(W_packed) || !aligned16(scales) || !aligned16(y)) return QL_EALIGN;
    unsigned char* scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return QL_ECUDA;
    if (skinny_max_k(QL_I8A8_G128_BF16) < 128) return QL_ECUDA;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int G = K / 128;
    int8_t* qx = reinterpret_cast<int8_t*>(scratch);
    float* sx = reinterpret_cast<float*>(scratch + kQxBytes);
    // The quantiser also zeroes y, which the GEMM then accumulates into.
    int t = trace_begin(QL_KIND_ACT_QUANT, s);
    cudaError_t e = launch_act_quant(x, M, K, (flags & QL_HADAMARD) ? 1 : 0, qx, sx, nullptr, 0, y, (long long)M * N,
                                     s);
    trace_end(t, s);
    if (e != cudaSuccess) return QL_ECUDA;
    // One decode launch over the whole K, as qlinear_forward makes it.
    SkinnyArgs a{};
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
    a.pdl = 1;
    t = trace_begin(QL_KIND_SKINNY, s);
    e = launch_skinny(QL_I8A8_G128_BF16, a, s);
    trace_end(t, s);
    return e == cudaSuccess ? QL_OK : QL_ECUDA;
}
