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
// chunks of at most 16 rows, the unit the grouped skinny GEMM consumes, or
// into the (row block, weight block) tiles of the grouped tensor-core GEMM,
// and records each pair's position (the inverse permutation) so that the
// activation staging can write rows straight into permuted order.
// Everything stays on the device: the GEMM reads the chunk count itself, so
// no host round trip sits between routing and the expert GEMM.
#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

constexpr int kPermThreads = 1024;

__global__ void __launch_bounds__(kPermThreads) k_moe_permute(const int32_t* ids, int T, int topk, int E,
                                                              int32_t* counts, int32_t* offsets, int32_t* perm,
                                                              const MoePermuteOut o, unsigned* err) {
    extern __shared__ int sm[];
    int* cnt = sm;                // [E]
    int* off = cnt + E;           // [E + 1]
    int* run = off + E + 1;       // [E]
    int* whist = run + E;         // [32][E]
    int* coff = whist + 32 * E;   // [E] first chunk of each expert
    int* toff = coff + E;         // [E] first tile of each expert
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int P = T * topk;

    for (int e = tid; e < E; e += kPermThreads) cnt[e] = 0;
    __syncthreads();
    int bad = 0;
    for (int i = tid; i < P; i += kPermThreads) {
        const int e = ids[i];
        if (e < 0 || e >= E) {
            ++bad;
            if (o.inv) o.inv[i] = -1;
            if (o.yz)  // the pair is skipped: its output row is zero
                for (int n = 0; n < o.N; ++n) o.yz[(long long)i * o.N + n] = 0.0f;
        } else {
            atomicAdd(&cnt[e], 1);
        }
    }
    if (__syncthreads_or(bad) && tid == 0) atomicOr(err, (unsigned)QL_DEVERR_EXPERT_ID);
    if (tid == 0) {  // exclusive scans over experts: rows, chunks, tiles
        int acc = 0, ch = 0, nt = 0;
        for (int e = 0; e < E; ++e) {
            const int c = cnt[e];
            off[e] = acc;
            run[e] = 0;
            coff[e] = ch;
            toff[e] = nt;
            acc += c;
            ch += (c + 15) / 16;
            if (o.tiles) nt += (c + o.tile_rows - 1) / o.tile_rows * o.wblocks;
        }
        off[E] = acc;
        if (o.n_chunks) *o.n_chunks = ch;
        if (o.n_tiles) *o.n_tiles = nt;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kPermThreads) {  // each expert's chunks and tiles, in parallel
        const int c = cnt[e], r0 = off[e];
        if (o.chunks)
            for (int s = 0, ch = coff[e]; s < c; s += 16, ++ch) o.chunks[ch] = MoeChunk{e, r0 + s, min(16, c - s)};
        if (o.tiles) {  // weight-block-major within the expert: its row blocks share each weight block
            int nt = toff[e];
            for (int wb = 0; wb < o.wblocks; ++wb)
                for (int s = 0; s < c; s += o.tile_rows, ++nt) o.tiles[nt] = MoeTile{e, r0 + s, min(o.tile_rows, c - s), wb};
        }
    }
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
        if (e >= 0) {
            const int pos = off[e] + whist[warp * E + e] + rank;
            perm[pos] = i;
            if (o.inv) o.inv[i] = pos;
        }
        __syncthreads();
    }
}

}  // namespace

size_t moe_max_chunks(int T, int topk, int E) { return (size_t)T * topk / 16 + (size_t)E + 1; }
size_t moe_max_tiles(int T, int topk, int E, int tile_rows, int wblocks) {
    return ((size_t)T * topk / tile_rows + (size_t)E + 1) * (size_t)wblocks;
}

cudaError_t launch_moe_permute(const int32_t* ids, int T, int topk, int E, int32_t* counts, int32_t* offsets,
                               int32_t* perm, const MoePermuteOut& out, unsigned* err, cudaStream_t s) {
    const size_t smem = (size_t)(5 * E + 1 + 32 * E) * sizeof(int);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_moe_permute, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_moe_permute<<<1, kPermThreads, smem, s>>>(ids, T, topk, E, counts, offsets, perm, out, err);
    return cudaGetLastError();
}

}  // namespace ql
