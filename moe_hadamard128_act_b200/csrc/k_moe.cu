// k_moe.cu -- MoE token permutation for the routed experts' gate_up
// projection ("gemma4-26b-a4b-dflash-i8", table "Weights").
//
// One CTA of 1024 threads groups the T*topk (token, slot) pairs by expert,
// stably (expert, t, j): a shared-memory histogram and scan give the segment
// offsets; then the pairs are placed tile by tile (1024 per tile, in input
// order): inside a warp the peers with the same expert are found with
// __match_any_sync and ranked by lane, the per-warp counts of each expert are
// prefix-summed across the 32 warps, and a running per-expert base carries
// over between tiles.  The same kernel cuts every expert's segment into
// chunks of at most 16 rows, the unit the grouped skinny GEMM consumes.
// Everything stays on the device: the GEMM reads the chunk count itself, so
// no host round trip sits between routing and the expert GEMM.
#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

constexpr int kPermThreads = 1024;

__global__ void __launch_bounds__(kPermThreads) k_moe_permute(const int32_t* ids, int T, int topk, int E,
                                                              int32_t* counts, int32_t* offsets, int32_t* perm,
                                                              MoeChunk* chunks, int* n_chunks, unsigned* err) {
    extern __shared__ int sm[];
    int* cnt = sm;                // [E]
    int* off = cnt + E;           // [E + 1]
    int* run = off + E + 1;       // [E]
    int* whist = run + E;         // [32][E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int P = T * topk;

    for (int e = tid; e < E; e += kPermThreads) cnt[e] = 0;
    __syncthreads();
    int bad = 0;
    for (int i = tid; i < P; i += kPermThreads) {
        const int e = ids[i];
        if (e < 0 || e >= E) ++bad;
        else atomicAdd(&cnt[e], 1);
    }
    if (__syncthreads_or(bad) && tid == 0) atomicOr(err, (unsigned)QL_DEVERR_EXPERT_ID);
    if (tid == 0) {
        int acc = 0, ch = 0;
        for (int e = 0; e < E; ++e) {
            off[e] = acc;
            run[e] = 0;
            const int c = cnt[e];
            for (int s = 0; s < c; s += 16, ++ch)
                if (chunks) chunks[ch] = MoeChunk{e, acc + s, min(16, c - s)};
            acc += c;
        }
        off[E] = acc;
        if (n_chunks) *n_chunks = ch;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kPermThreads) counts[e] = cnt[e];
    for (int e = tid; e <= E; e += kPermThreads) offsets[e] = off[e];
    const int valid = off[E];
    for (int i = valid + tid; i < P; i += kPermThreads) perm[i] = -1;

    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < P; base += kPermThreads) {
        for (int i = tid; i < 32 * E; i += kPermThreads) whist[i] = 0;
        __syncthreads();
        const int i = base + tid;
        int e = (i < P) ? ids[i] : -1;
        if (e >= E) e = -1;
        const unsigned peers = __match_any_sync(kFull, e);
        const int rank = __popc(peers & lt);
        if (e >= 0 && rank == 0) whist[warp * E + e] = __popc(peers);
        __syncthreads();
        // Exclusive prefix over warps, per expert; whist becomes the warp's base.
        for (int x = tid; x < E; x += kPermThreads) {
            int r = run[x];
            for (int w = 0; w < 32; ++w) {
                const int c = whist[w * E + x];
                whist[w * E + x] = r;
                r += c;
            }
            run[x] = r;
        }
        __syncthreads();
        if (e >= 0) perm[off[e] + whist[warp * E + e] + rank] = i;
        __syncthreads();
    }
}

}  // namespace

size_t moe_max_chunks(int T, int topk, int E) { return (size_t)T * topk / 16 + (size_t)E + 1; }

cudaError_t launch_moe_permute(const int32_t* ids, int T, int topk, int E, int32_t* counts, int32_t* offsets,
                               int32_t* perm, MoeChunk* chunks, int* n_chunks, unsigned* err, cudaStream_t s) {
    const size_t smem = (size_t)(3 * E + 1 + 32 * E) * sizeof(int);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_moe_permute, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_moe_permute<<<1, kPermThreads, smem, s>>>(ids, T, topk, E, counts, offsets, perm, chunks, n_chunks, err);
    return cudaGetLastError();
}

}  // namespace ql
