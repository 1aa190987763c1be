// k_moe.cu -- MoE token permutation for the routed experts' gate_up
// projection ("gemma4-26b-a4b-dflash-i8", table "Weights").
//
// The T*topk (token, slot) pairs are grouped by expert, stably in (expert, t,
// j) order, by one CTA per expert, so no CTA waits for another.  Every CTA
// reads all pair ids once (they stay in L2), with each thread owning a
// contiguous span: a shared-memory histogram of all experts gives the CTA its
// segment offset and its first chunk and tile, and the thread's own count of
// the CTA's expert, scanned across the block, gives where its pairs go.  The
// threads that hold such pairs read their span again to write them.
// Each CTA also writes its expert's count and offset, its entries of the
// inverse permutation, and its chunks of at most 16 rows (the unit of the
// grouped skinny GEMM) or its (row block, weight block) tiles (the grouped
// tensor-core GEMM).  One more CTA takes the pairs whose id is outside
// [0, E): it flags them, marks them in the inverse permutation, zeroes their
// output rows when asked, fills the tail of perm with -1, and writes the
// totals.  Everything stays on the device: the GEMMs read the chunk or tile
// count themselves, so no host round trip sits between routing and the
// expert GEMM.
#include "ql_device.cuh"
#include "ql_internal.h"

namespace ql {
namespace {

constexpr int kPermThreads = 512;

// Sum of v over the block; every thread gets the result.  red holds a slot per warp.
__device__ __forceinline__ int block_sum(int v, int* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int t = 0;
    for (int w = 0; w < kPermThreads / 32; ++w) t += red[w];
    return t;
}

__global__ void __launch_bounds__(kPermThreads) k_moe_permute(const int32_t* ids, int T, int topk, int E,
                                                              int32_t* counts, int32_t* offsets, int32_t* perm,
                                                              const MoePermuteOut o, unsigned* err) {
    extern __shared__ int hist[];  // [E]
    __shared__ int s_red[kPermThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int P = T * topk;
    const int e = blockIdx.x;  // this CTA's expert; e == E: the bad ids and the totals

    for (int x = tid; x < E; x += kPermThreads) hist[x] = 0;
    __syncthreads();

    // Each thread owns a contiguous span of ids (a multiple of 4 long, so the
    // 16-byte loads stay aligned), which keeps the compaction in input order
    // with a single scan of per-thread counts.
    const int S = ((P + kPermThreads - 1) / kPermThreads + 3) & ~3;
    const int b0 = tid * S, b1 = min(P, b0 + S);
    const bool vec = (P & 3) == 0;  // ids are 16-byte aligned (checked on the host)
    int mine = 0;
#pragma unroll 4
    for (int i = b0; i < b1; i += 4) {
        int xs[4];
        if (vec) {
            const int4 q = __ldg(reinterpret_cast<const int4*>(ids + i));
            xs[0] = q.x; xs[1] = q.y; xs[2] = q.z; xs[3] = q.w;
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) xs[j] = i + j < b1 ? __ldg(ids + i + j) : 0;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (i + j >= b1) break;
            const int x = xs[j];
            if (x >= 0 && x < E) {
                atomicAdd(&hist[x], 1);
                mine += x == e;
            } else if (e == E) {  // a pair routed to no expert: flagged, its output row zero
                ++mine;
                if (o.inv) o.inv[i + j] = -1;
                if (o.yz)
                    for (int n = 0; n < o.N; ++n) o.yz[(long long)(i + j) * o.N + n] = 0.0f;
            }
        }
    }
    __syncthreads();

    // Exclusive sums over the experts before e of rows, chunks and tiles (for
    // e == E: the totals), each thread taking every 512th expert.
    int r = 0, ch = 0, nt = 0;
    for (int x = tid; x < e; x += kPermThreads) {
        const int c = hist[x];
        r += c;
        ch += (c + 15) >> 4;
        if (o.tiles) nt += (c + o.tile_rows - 1) / o.tile_rows * o.wblocks;
    }
    const int r0 = block_sum(r, s_red);
    const int coff = block_sum(ch, s_red);
    const int toff = block_sum(nt, s_red);

    if (e == E) {  // ---- bad ids, the tail of perm, the totals ----
        if (__syncthreads_or(mine) && tid == 0) atomicOr(err, (unsigned)QL_DEVERR_EXPERT_ID);
        for (int i = r0 + tid; i < P; i += kPermThreads) perm[i] = -1;
        if (tid == 0) {
            offsets[E] = r0;
            if (o.n_chunks) *o.n_chunks = coff;
            if (o.n_tiles) *o.n_tiles = toff;
        }
        return;
    }

    const int c = hist[e];
    if (tid == 0) {
        counts[e] = c;
        offsets[e] = r0;
    }
    // Exclusive scan of the per-thread counts: shuffles within the warp, warp totals across.
    int incl = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int up = __shfl_up_sync(kFull, incl, d);
        if (lane >= d) incl += up;
    }
    __syncthreads();
    if (lane == 31) s_red[warp] = incl;
    __syncthreads();
    int pos = r0 + incl - mine;
    for (int w = 0; w < warp; ++w) pos += s_red[w];
    if (mine > 0)  // second read of the span, now in L1/L2
        for (int i = b0; i < b1; ++i)
            if (__ldg(ids + i) == e) {
                perm[pos] = i;
                if (o.inv) o.inv[i] = pos;
                ++pos;
            }

    if (o.chunks)
        for (int k = tid; 16 * k < c; k += kPermThreads) o.chunks[coff + k] = MoeChunk{e, r0 + 16 * k, min(16, c - 16 * k)};
    if (o.tiles) {  // weight-block-major within the expert: its row blocks share each weight block
        const int nrb = (c + o.tile_rows - 1) / o.tile_rows;
        for (int k = tid; k < nrb * o.wblocks; k += kPermThreads) {
            const int wb = k / nrb, rb = k - wb * nrb;
            o.tiles[toff + k] = MoeTile{e, r0 + rb * o.tile_rows, min(o.tile_rows, c - rb * o.tile_rows), wb};
        }
    }
}

}  // namespace

size_t moe_max_chunks(int T, int topk, int E) { return (size_t)T * topk / 16 + (size_t)E + 1; }
size_t moe_max_tiles(int T, int topk, int E, int tile_rows, int wblocks) {
    return ((size_t)T * topk / tile_rows + (size_t)E + 1) * (size_t)wblocks;
}

cudaError_t launch_moe_permute(const int32_t* ids, int T, int topk, int E, int32_t* counts, int32_t* offsets,
                               int32_t* perm, const MoePermuteOut& out, unsigned* err, cudaStream_t s) {
    const size_t smem = (size_t)E * sizeof(int);
    if (smem > 48 * 1024) return cudaErrorInvalidValue;  // E <= 1024 (checked by the caller)
    k_moe_permute<<<E + 1, kPermThreads, smem, s>>>(ids, T, topk, E, counts, offsets, perm, out, err);
    return cudaGetLastError();
}

}  // namespace ql
