// ql_internal.h -- host-side interface between the C-ABI layer (ql_api.cu)
// and the kernel translation units.  Nothing here is exported.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/qlinear.h"

namespace ql {

// ---- format arithmetic -------------------------------------------------------
inline bool fmt_valid(int f) { return f >= QL_I8_G128_BF16 && f <= QL_FP8A8_B128_BF16; }
// FP8 E4M3 weights with 128 x 128 block scales (formats 6 and 7 pack alike).
inline bool fmt_fp8_weights(int f) { return f == QL_FP8_B128_BF16 || f == QL_FP8A8_B128_BF16; }
inline bool fmt_scale_f16(int f) { return f == QL_I8_G128_F16 || f == QL_I5Z_G128_F16; }
// int8 codes with 16-bit activations (formats 1 and 2).
inline bool fmt_i8_a16(int f) { return f == QL_I8_G128_BF16 || f == QL_I8_G128_F16; }
inline int fmt_group(int f) { return f == QL_I4_G64_BF16 ? 64 : 128; }
// Bytes of one packed row of K codes.
inline size_t fmt_row_bytes(int f, size_t K) {
    switch (f) {
    case QL_I4_G64_BF16: return K / 2;
    case QL_I5Z_G128_F16: return K * 5 / 8;
    default: return K;
    }
}
void packed_sizes(int fmt, size_t N, size_t K, size_t* codes, size_t* scales, size_t* zeros);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// A TMA tensor map over a 2-D byte matrix: `rows` rows of `width_bytes` bytes,
// `ld_bytes` apart, box [box_y rows][box_x bytes], swizzle as CUtensorMapSwizzle.
cudaError_t make_tmap_2d(const void* base, long long rows, long long width_bytes, long long ld_bytes, int box_x,
                         int box_y, int swz, CUtensorMap* out);

// Per-device facts, cached on first use.
struct DeviceInfo {
    int sm_count;
    size_t smem_optin;   // max dynamic shared memory per block (opt-in)
    unsigned* err_word;  // device address of the error word; the wait limit follows it (see wait_limit)
};
cudaError_t device_info(DeviceInfo* out);

// ---- activations ---------------------------------------------------------------
// Prepared activations for the weight-only (A16) skinny GEMM: f16 copy of x
// scaled per token by a power of two, in the element order the format's MMA
// fragments want; xf[t] = the inverse power of two.
enum XOrder { XORD_NATURAL = 0, XORD_I4 = 1, XORD_I5 = 2 };
cudaError_t launch_rotate_bf16(const void* x, int M, int K, void* y, cudaStream_t s);
// The act-quant and prep kernels also zero y[0 .. nz) (yz may be null), so the
// skinny GEMM that follows can accumulate into it without a separate launch.
// act quant writes the scales [M][K/128] to sx and/or transposed, [K/128][Mp],
// to sxT (either may be null).
cudaError_t launch_act_quant(const void* x, int M, int K, int rotate, int8_t* q, float* sx, float* sxT, int Mp,
                             float* yz, long long nz, cudaStream_t s);
// The same rule with E4M3 codes (448 for 127), written as bytes.  With inv != null, token t's codes
// and scales go to rows inv[t * topk + j] of q and sxT (the permuted order of the grouped expert GEMM).
cudaError_t launch_act_quant_e4m3(const void* x, int M, int K, int rotate, uint8_t* q, float* sx, float* sxT, int Mp,
                                  float* yz, long long nz, cudaStream_t s, const int32_t* inv = nullptr,
                                  int topk = 0);
// XORD_I5 also writes xsum [M][K/128] (each group's sum of the f16 activations, for the zero
// point) and puts 2^24 into xf (the int5 codes enter the MMAs as exact subnormals u * 2^-24);
// so does any other order given an xsum, but XORD_I4: it stages the activations of odd k (the
// high nibbles) divided by 16, writes the sums per 64-group, [M][K/64], and no 2^24 (the int4
// kernel that uses the sums puts that factor into its scales).
cudaError_t launch_prep_a16(const void* x, int M, int K, int rotate, int order, __half* xs, float* xf, float* yz,
                            long long nz, cudaStream_t s, float* xsum = nullptr);

// ---- packing ---------------------------------------------------------------------
cudaError_t launch_pack_rtn(const float* W, int fmt, int flags, int N, int K, void* codes, void* scales,
                            cudaStream_t s);
cudaError_t launch_pack_codes(const void* codes_in, int fmt, int N, int K, void* codes_out, unsigned* err,
                              cudaStream_t s);
cudaError_t launch_check_zeros(const uint8_t* z_in, size_t n, uint8_t* z_out, unsigned* err, cudaStream_t s);

// ---- skinny GEMM (M <= 16 per launch) -----------------------------------------------
struct SkinnyArgs {
    CUtensorMap tmap;      // filled by launch_skinny: W as [N rows][G units], box [16][unit bytes]
    const uint8_t* W;      // packed codes, row stride ldw bytes; already offset to group g0
    const void* scales;    // [N][Gtot] (fp8: [N/128][Gtot]); indexed with g0 + g
    const uint8_t* zeros;  // int5: [N][Gtot]
    const void* xs;        // prepared activations, row stride ldx elements; offset to group g0
    const float* xf;       // A16: [M] inverse token factors; W8A8: sx [M][Gtot]
    const float* xsum = nullptr;  // int5, int8 A16: each token's sums of its f16 activations per group [M][Gtot];
                                  // int4: per 64-group [M][2 Gtot]
    float* y;              // [M][ldy]
    int32_t* acc;          // optional W8A8 group sums [M][N][Gtot]
    unsigned* err;         // device error word (filled by launch_skinny)
    int M, N, G, g0, Gtot;
    int GP, XG;            // K-part size and staged groups (filled by launch_skinny)
    int pdl;               // launched right after this library's activation prologue: may overlap it
    long long ldw, ldx, ldy;
};
cudaError_t launch_skinny(int fmt, const SkinnyArgs& a, cudaStream_t s);
// Largest K (multiple of 128) one skinny launch stages in shared memory.
int skinny_max_k(int fmt);

// ---- prefill GEMM (tcgen05) ----------------------------------------------------------------
// y[M][ldy] (fp32, overwritten) = W8A8 product of int8 activations qx [M][K] with
// scales sxT [K/128][Mp] (transposed, Mp = prefill_pad_m(M)) and int8
// weights qw [N][K] with bf16 scales sw [N][K/128].  `scratch` holds
// prefill_scratch_bytes(N, K) bytes (the weight scales, transposed to fp32).
// With acc != null, writes the int32 group sums [M][N][K/128] instead of y;
// then sxT, sw and scratch are not used.
#ifndef QL_PF_N
#define QL_PF_N 192
#endif
constexpr int kPrefillTileM = 128, kPrefillTileN = QL_PF_N;  // output tile; scale arrays are padded to it
inline int prefill_pad_m(int v) { return (v + kPrefillTileM - 1) / kPrefillTileM * kPrefillTileM; }
inline int prefill_pad_n(int v) { return (v + kPrefillTileN - 1) / kPrefillTileN * kPrefillTileN; }
static_assert(kPrefillTileN % 32 == 0, "weight-scale padding is a whole number of 32-wide transpose tiles");
inline size_t prefill_scratch_bytes(int N, int K) { return align_up((size_t)(K / 128) * prefill_pad_n(N) * 4, 256); }
// e4m3: qx and qw hold E4M3 codes (format 7), the MMAs run kind::f8f6f4.
cudaError_t launch_prefill_w8a8(const int8_t* qx, const float* sxT, const int8_t* qw, int M, int N, int K,
                                float* y, long long ldy, int32_t* acc, const void* scratch, cudaStream_t s,
                                bool e4m3 = false);
// Fills the scratch: bf16 (f16) weight scales [N][K/128] -> fp32 [K/128][pad(N)].
cudaError_t launch_prefill_prep(const uint16_t* sw, int N, int K, void* scratch, cudaStream_t s, bool f16 = false);
// int5 codes [N][5K/8] and zero points [N][K/128] -> int8 q - z [N][K] (for the W5A8 path).
cudaError_t launch_prefill_i5_codes(const uint8_t* codes, const uint8_t* zeros, int N, int K, int8_t* out,
                                    cudaStream_t s);
// From this many rows on, the int5 format takes int8 activations ("keptn/gemma4-31b-w5",
// table "Format": f16 activations up to 64 rows, int8 per token per 128 above).
constexpr int kW5A8MinM = 65;
// The same from bf16 block scales [ceil(N/128)][K/128] (each row takes its block's scale); for E
// stacked experts, E consecutive scale arrays in, E consecutive [K/128][pad(N)] blocks out.
cudaError_t launch_prefill_prep_blk(const uint16_t* sw, int N, int K, void* scratch, cudaStream_t s, int E = 1);
constexpr int kPrefillMinM = 17;  // from this many tokens on, W8A8 runs on the tcgen05 GEMM

// The same for the formats with 16-bit activations (int8 g128 with bf16 or f16
// scales, fp8 128x128): y[M][ldy] (fp32, overwritten) from the f16 activations
// xs [M][K] (natural order, token factors xf [M], as launch_prep_a16 makes
// them) and the packed codes and scales.  Weight rows are the MMA's M, tokens
// its N (kPrefillA16Tokens per tile).
#ifndef QL_A16_TN
#define QL_A16_TN 192
#endif
constexpr int kPrefillA16Tokens = QL_A16_TN;
bool prefill_a16_supported(int fmt);
cudaError_t launch_prefill_a16(int fmt, const __half* xs, const float* xf, const uint8_t* codes, const void* scales,
                               int M, int N, int K, float* y, long long ldy, cudaStream_t s);

// ---- MoE -----------------------------------------------------------------------------------
struct MoeChunk {
    int expert, start, count;  // rows perm[start .. start+count) of the permuted order
};
size_t moe_max_chunks(int T, int topk, int E);
// One tile of a grouped expert GEMM: `rows` permuted rows from `row0` (all
// of one expert) against weight block wb of that expert (blocks of the GEMM's
// height: 128 rows for the A16 and down-projection kernels, 192 for the E4M3
// one).
struct MoeTile {
    int expert, row0, rows, wb;
};
// Optional outputs beyond counts/offsets/perm (each may be null):
//   chunks / n_chunks: segments cut into <= 16-row chunks (the skinny GEMM's unit);
//   inv: inv[t * topk + j] = position of the pair in perm, -1 for a bad id;
//   tiles / n_tiles: segments cut into tile_rows-row blocks x wblocks weight blocks;
//   yz: the rows y[t * topk + j][0 .. N) of pairs with a bad id are zeroed.
struct MoePermuteOut {
    MoeChunk* chunks = nullptr;
    int* n_chunks = nullptr;
    int32_t* inv = nullptr;
    MoeTile* tiles = nullptr;
    int* n_tiles = nullptr;
    int tile_rows = 0, wblocks = 0;
    float* yz = nullptr;
    int N = 0;
};
size_t moe_max_tiles(int T, int topk, int E, int tile_rows, int wblocks);
// Format 7 experts on the E4M3 tensor-core GEMM, grouped: qx the E4M3 codes of the permuted rows
// [rows_total][K] with their scales sxT [K/128][Mp] (Mp % 4 == 0, at least 132 columns past the last
// row), swT the experts' weight scales from launch_prefill_prep_blk (E blocks), tiles of
// kPrefillTileM permuted rows x kPrefillTileN weight rows from the permute.
cudaError_t launch_prefill_e4m3_grouped(const uint8_t* qx, const float* sxT, int Mp, const uint8_t* codes,
                                        const float* swT, int E, int N, int K, int rows_total, const MoeTile* tiles,
                                        const int* n_tiles, int max_tiles, const int32_t* perm, float* y,
                                        cudaStream_t s);
// The experts' bf16 down projection on the grouped tensor-core GEMM (k_down.cu): act holds each
// pair's activation as three bf16 planes [rows_total][3 I] in permuted order, wd the stacked bf16
// weights [E * N][I]; tiles of at most kDownTileRows permuted rows x 128 weight rows from the
// permute; row r of a tile is added into out[perm[r] / topk][0 .. N) scaled by wts[perm[r]], the
// whole 3 I accumulated in tensor memory.
constexpr int kDownTileRows = 160;
cudaError_t launch_down_grouped(const __nv_bfloat16* act, const uint16_t* wd, int E, int N, int I, int rows_total,
                                const MoeTile* tiles, const int* n_tiles, int max_tiles, const int32_t* perm,
                                int topk, const float* wts, float* out, cudaStream_t s);
// From this many (token, slot) pairs per expert on average, moe_gate_up runs the grouped tensor-core GEMM.
constexpr int kMoePrefillMinRowsPerExpert = 8;
cudaError_t launch_moe_permute(const int32_t* ids, int T, int topk, int E, int32_t* counts, int32_t* offsets,
                               int32_t* perm, const MoePermuteOut& out, unsigned* err, cudaStream_t s);
struct MoeArgs {
    CUtensorMap tmap;      // filled by launch_moe_skinny: codes as [E * N rows][K bytes], box [16][128 B]
    unsigned* err;         // device error word (filled by launch_moe_skinny)
    const uint8_t* codes;  // [E][N][K]
    const void* scales;    // [E][...] per the format
    const void* xs;        // prepared activations [T][K]: f16 in natural order, or E4M3 codes (format 7)
    const float* xf;       // [T] inverse token factors, or (format 7) activation scales [T][K/128]
    const float* xsum = nullptr;  // int8 codes: each token's sums of its f16 activations per group [T][K/128]
    const int32_t* perm;   // [T*topk]
    const MoeChunk* chunks;
    const int* n_chunks;
    const int32_t* ids = nullptr;  // [T*topk] routing ids: when set (T*topk <= kMoeFusedMaxPairs), every CTA
                           // builds the permutation and chunk table itself and perm / chunks are unused
    float* y;              // [T*topk][N] (down projection: [T][N])
    const float* wts = nullptr;  // down projection: routing weights [T*topk]
    int fmt, T, topk, E, N, K;
    long long max_chunks;
};
constexpr int kMoeFusedMaxPairs = 128;
cudaError_t launch_moe_skinny(const MoeArgs& a, cudaStream_t s);
// The experts' bf16 down projection with the routing-weighted combine: codes are the stacked bf16
// weights [E][N][K] (N = hidden size, K = intermediate size, K % 64 == 0), xs the pairs'
// activations as three bf16 planes [T*topk][3][K]; y [T][N] (zeroed before) gets
// sum_j wts[t*topk+j] * (act of (t, j)) . W_e^T.  Chunks / fused ranking as launch_moe_skinny.
cudaError_t launch_moe_down(const MoeArgs& a, cudaStream_t s);
// gelu(gate) * up of each pair's gate_up row h [P][2 I] (fp32), split into three bf16 planes
// act [P][3][I] whose sum is the fp32 value (pair p to row inv[p] when inv is given, the permuted
// order); pairs with an id outside [0, E) are skipped.  Also zeroes out[0 .. nz).
cudaError_t launch_moe_act(const float* h, const int32_t* ids, int P, int E, int I, __nv_bfloat16* act, float* out,
                           long long nz, cudaStream_t s, const int32_t* inv = nullptr);

// ---- launch trace (ql_trace_enable / ql_trace_read) --------------------------------------
// trace_begin records a start event for one library launch when tracing is on
// and returns its slot (or -1); trace_end records the matching stop event.
int trace_begin(int kind, cudaStream_t s);
void trace_end(int slot, cudaStream_t s);

}  // namespace ql
