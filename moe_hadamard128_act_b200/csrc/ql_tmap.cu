// ql_tmap.cu -- host-side construction of TMA tensor maps for 2-D byte
// matrices (packed weights, int8 activations), cached by (address, shape, box,
// swizzle) since the same weight is encoded again on every call.
#include <mutex>

#include <cudaTypedefs.h>

#include "ql_internal.h"

namespace ql {
namespace {

struct TmapKey {
    const void* ptr;
    long long rows, width, ld;
    int box_x, box_y, swz;
    bool operator==(const TmapKey& o) const {
        return ptr == o.ptr && rows == o.rows && width == o.width && ld == o.ld && box_x == o.box_x &&
               box_y == o.box_y && swz == o.swz;
    }
};

std::mutex g_mu;
TmapKey g_keys[128];
CUtensorMap g_vals[128];
int g_n = 0, g_next = 0;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

}  // namespace

cudaError_t make_tmap_2d(const void* base, long long rows, long long width_bytes, long long ld_bytes, int box_x,
                         int box_y, int swz, CUtensorMap* out) {
    std::lock_guard<std::mutex> lock(g_mu);
    const TmapKey key{base, rows, width_bytes, ld_bytes, box_x, box_y, swz};
    for (int i = 0; i < g_n; ++i)
        if (g_keys[i] == key) {
            *out = g_vals[i];
            return cudaSuccess;
        }
    if (!g_encode) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
            cudaGetLastError();
            return cudaErrorNotSupported;
        }
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    const cuuint64_t dims[2] = {(cuuint64_t)width_bytes, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ld_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)box_x, (cuuint32_t)box_y};
    const cuuint32_t estr[2] = {1u, 1u};
    CUtensorMap m;
    const CUresult r = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, static_cast<CUtensorMapSwizzle>(swz),
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const int slot = g_n < 128 ? g_n++ : (g_next++ & 127);
    g_keys[slot] = key;
    g_vals[slot] = m;
    *out = m;
    return cudaSuccess;
}

}  // namespace ql
