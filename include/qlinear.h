/*
 * qlinear.h -- C ABI of libqlinear.so: the group-scaled low-bit quantized
 * linear layer y = x . dequant(W)^T on NVIDIA B200 (sm_100a), and its use as
 * the routed experts' gate_up projection of a mixture-of-experts block.
 *
 * Formats (one enum value each), as the model cards define them:
 *   QL_I8_G128_BF16   int8 codes -127..127, one bf16 scale per row per 128 of
 *                     K ("gemma4-26b-a4b-dflash-i8" README, table "Weights";
 *                     "keptn/gemma4-12b-i8g", table "Format").  x is bf16.
 *   QL_I8_G128_F16    the same codes with an f16 scale (the drafter linears
 *                     of "gemma4-26b-a4b-dflash-i8", recipe lines dflash.*).
 *   QL_I8A8_G128_BF16 W8A8: the int8 weights above, and the activations
 *                     quantised to int8 with one scale per token per 128
 *                     values ("keptn/gemma4-12b-i8g", table "Format").
 *   QL_I4_G64_BF16    symmetric int4 [-8,7], one bf16 scale per row per 64
 *                     of K ("Gemma4-26B-CIRU-AMD-STRIX-vLLM", "What is in the
 *                     release"); x is bf16.
 *   QL_I5Z_G128_F16   int5 codes [0,31] with a u8 zero point and one f16 scale
 *                     per row per 128 of K: w = s * (q - z) ("keptn/gemma4-31b-w5",
 *                     table "Format"); x is bf16 up to 64 rows (M <= 64).  From
 *                     65 rows on, as that card's activations do, x is quantised
 *                     to int8 per token per 128 like W8A8's and each group's
 *                     integer dot product sum qx * (q - z) is exact before s_x * s
 *                     is applied (W5A8).
 *   QL_FP8_B128_BF16  FP8 E4M3 codes with one bf16 scale per 128 (rows) x 128
 *                     (K) block ("gemma4-26b-a4b-dflash-fp8" README, table
 *                     "Weights" and its recipe); x is bf16.
 *   QL_FP8A8_B128_BF16  the same packed weights with E4M3 activations: x is
 *                     quantised per token per 128 values as
 *                     act_quant_e4m3_g128 does (the int8 activation rule of
 *                     "keptn/gemma4-12b-i8g" with E4M3 codes; a reading, no card
 *                     ships it), and every 128-group's products are summed
 *                     before both scales are applied.  M <= 16 runs
 *                     the weight-streaming decode kernel on E4M3 mma.sync,
 *                     M >= 17 the tensor-core E4M3 GEMM.
 * Flag QL_HADAMARD: the weights live in the 128-wide Walsh-Hadamard domain
 * ("transform=fwht128" in the recipe of "gemma4-26b-a4b-dflash-i8"); the
 * forward pass rotates each 128-block of x by the same orthonormal transform
 * first, so that (H x) . (H w) = x . w.
 *
 * Packed layouts (all row-major, W is [N, K] with K contiguous):
 *   int8 / fp8 codes: one byte per code, [N][K] (formats 6 and 7 pack alike).
 *   int4 codes: [N][K/2] bytes, code k of a row in byte k/2, low nibble for
 *     even k, stored offset-binary (q + 8).
 *   int5 codes: [N][5K/8] bytes, each row a least-significant-bit-first bit
 *     stream with code k in stream bits 5k..5k+4.
 *   scales: [N][K/g] of bf16 or f16 (g = 128, or 64 for int4); fp8 block
 *     scales [ceil(N/128)][K/128] bf16.  zeros (int5 only): [N][K/128] u8.
 *
 * Conventions for every call:
 *   - All data pointers are DEVICE pointers owned by the caller, except the
 *     size outputs of the *_size calls, which are host pointers.  The library
 *     keeps no reference to any buffer after a call returns and allocates no
 *     device memory: scratch space is the caller's workspace.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     enqueue work and return; none synchronises except ql_get_device_error.
 *   - K must be a multiple of 128, M, N, T >= 1, every device pointer 16-byte
 *     aligned.  Violations return a status before anything is launched.
 *   - Errors found on the device (an expert id outside [0, E), a code out of
 *     its range given to the packer, a copy into shared memory that did not
 *     complete within 200 ms) never trap: the offending item is skipped (a
 *     timed-out kernel stops early, leaving its output incomplete) and a bit is
 *     set in a per-process device error word that ql_get_device_error reads and
 *     clears.
 *   - No C++ exception crosses this interface.
 */
#ifndef QLINEAR_H
#define QLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QL_OK = 0,
    QL_EINVAL = 1,        /* bad size, null pointer or unknown format/flag        */
    QL_EUNSUPPORTED = 2,  /* valid request this library does not implement        */
    QL_EALIGN = 3,        /* a device pointer is not 16-byte aligned               */
    QL_EWORKSPACE = 4,    /* workspace missing or smaller than *_workspace_size   */
    QL_ECUDA = 5,         /* a CUDA runtime call failed                           */
    QL_EDEVICE = 6        /* the device error word was set (see ql_get_device_error) */
} ql_status;

typedef enum {
    QL_I8_G128_BF16 = 1,
    QL_I8_G128_F16 = 2,
    QL_I8A8_G128_BF16 = 3,
    QL_I4_G64_BF16 = 4,
    QL_I5Z_G128_F16 = 5,
    QL_FP8_B128_BF16 = 6,
    QL_FP8A8_B128_BF16 = 7
} ql_fmt;

/* QL_SCALE_SEARCH: a rule for qlinear_pack's mode (a), int8 formats (1, 2, 3)
 * only -- see qlinear_pack.  The packed result has the same layout, so other
 * calls accept the flag and ignore it. */
enum { QL_HADAMARD = 1, QL_SCALE_SEARCH = 2 };

/* Bits of the device error word.  QL_DEVERR_BOUNDS: a kernel found an index it
 * reads from device memory (a routing table entry or a permuted row) outside its
 * buffers and skipped it; the results of that call are incomplete. */
enum { QL_DEVERR_EXPERT_ID = 1, QL_DEVERR_CODE_RANGE = 2, QL_DEVERR_TIMEOUT = 4, QL_DEVERR_BOUNDS = 8 };

/* Human-readable name of a status. Never NULL. */
const char* ql_status_string(int status);

/* Byte sizes of the packed codes, scales and zeros of an [N, K] weight in
 * format `fmt` (zeros is 0 except for int5).  Host pointers. */
int qlinear_packed_sizes(int fmt, int N, int K, size_t* codes_bytes, size_t* scales_bytes,
                         size_t* zeros_bytes);

/* qlinear_pack -- build the packed weight ("rtn ... group=128 scale=bf16
 * [transform=fwht128] clamp=sym" and its siblings in the recipes of the
 * "gemma4-26b-a4b-dflash-i8" and "-fp8" READMEs).
 *
 * Two modes:
 *  (a) W != NULL, codes_in == NULL: round-to-nearest quantisation of the fp32
 *      weight W [N, K] (device).  With QL_HADAMARD each 128-block of each row
 *      is first rotated by the fp32 Walsh-Hadamard transform (butterfly
 *      strides 1..64, then x fp32(1/sqrt(128))).  int8 formats: per row per
 *      128, s = scale_fmt(fp32(amax/127)), q = clamp(rne(w/s), -127, 127);
 *      int4: s = bf16(fp32(amax/7)), q = clamp(rne(w/s), -8, 7); fp8: per
 *      128x128 block, s = bf16(fp32(amax/448)), q = e4m3_rne_satfinite(w/s).
 *      An all-zero group gets s = 0 and q = 0.  int5 is rejected
 *      (QL_EUNSUPPORTED): its codes come from a calibrated quantiser.
 *      With QL_SCALE_SEARCH (int8 formats; others QL_EUNSUPPORTED) each group
 *      takes the best of 21 scales instead ("round to nearest with a scale
 *      search", rule=search, in the "gemma4-26b-a4b-dflash-i8" README; the
 *      card names the search, the candidates and measure are a reading):
 *      r = fp32(amax/127); for i = 0..20, s_i = scale_fmt(fp32(r *
 *      fp32((100 - i)/100))), codes by the round-to-nearest rule with s_i, and
 *      the squared error sum_k (w_k - s_i q_k)^2 over k = 0..127 in order, each
 *      operation rounded to fp64; the least error wins, the smaller i on a
 *      tie (i = 0 is the plain round-to-nearest result).
 *  (b) codes_in != NULL: pack given codes.  codes_in is int8 [N, K] (uint8 for
 *      int5, e4m3 bytes for fp8), scales_in the scales in the output layout,
 *      zeros_in the int5 zero points; they are copied / bit-packed.  A code
 *      outside its format's range is packed as 0 and flags QL_DEVERR_CODE_RANGE.
 *      QL_SCALE_SEARCH with given codes is QL_EINVAL.
 * Outputs: codes_out, scales_out and (int5) zeros_out, sized by
 * qlinear_packed_sizes. */
int qlinear_pack(const float* W, const void* codes_in, const void* scales_in, const uint8_t* zeros_in, int fmt,
                 int flags, int N, int K, void* codes_out, void* scales_out, uint8_t* zeros_out, void* stream);

/* Workspace bytes qlinear_forward needs for these sizes (may be 0). */
int qlinear_workspace_size(int fmt, int flags, int M, int N, int K, size_t* bytes);

/* qlinear_forward -- y[M, N] (fp32) = x~ . dequant(W)^T.
 *   x: bf16 [M, K] (device).  x~ is x, or with QL_HADAMARD its per-128-block
 *      rotation rounded to bf16 (as hadamard128_rotate); for W8A8, x~ is the
 *      int8 quantisation of (rotated) x, one fp32 scale per token per 128
 *      (as act_quant_i8_g128), and each 128-group's integer dot product is
 *      exact in int32 before its two scales are applied; the same for int5
 *      with M >= 65 (W5A8, codes q - z).
 *   W_packed, scales, zeros: the packed weight (zeros only for int5).
 *   ws, ws_bytes: caller's device workspace, at least qlinear_workspace_size.
 * y is overwritten.  The floating-point sums may be accumulated in any order;
 * they are not bit-reproducible across calls.
 * Calls whose activations stay 16-bit (all formats but W8A8 and format 7, and
 * int5 up to 64 rows) stage one token row, in fp32 and f16, in shared memory:
 * they take K <= QL_A16_MAX_K and return QL_EUNSUPPORTED above it
 * (moe_gate_up likewise). */
enum { QL_A16_MAX_K = 32768 };
int qlinear_forward(const void* x, const void* W_packed, const void* scales, const uint8_t* zeros, int fmt,
                    int flags, int M, int N, int K, float* y, void* ws, size_t ws_bytes, void* stream);

/* W8A8 integer core, for checking: acc[m, n, g] (int32, [M, N, K/128]) =
 * sum over k in group g of qx[m, k] * qw[n, k], with qx int8 [M, K] and qw int8
 * [N, K] (device).  Runs the same integer MMA path as qlinear_forward. */
int qlinear_forward_i8_acc(const int8_t* qx, const int8_t* qw, int M, int N, int K, int32_t* acc, void* stream);

/* qlinear_gemm_a8 -- the decode GEMM alone, on activations that are already
 * quantised per token per 128 values ("keptn/gemma4-12b-i8g", table "Format":
 * int8 activations with one scale per token per 128), for callers whose
 * previous kernel emits them:
 *   y[m, n] (+)= sum_g sx[m, g] * s_w[n, g] * sum_{k in g} qx[m, k] * qw[n, k].
 * fmt QL_I8A8_G128_BF16: qx int8 [M, K] as act_quant_i8_g128 makes it, each
 * group's integer sum exact; fmt QL_FP8A8_B128_BF16: qx E4M3 bytes [M, K] as
 * act_quant_e4m3_g128 makes it, s_w the weight's 128 x 128 block scale.  sx
 * fp32 [M, K/128].  W_packed, scales: the packed weight.  M <= 16 (the decode
 * shapes; larger M returns QL_EUNSUPPORTED).  accumulate != 0 adds the product
 * to y; accumulate == 0 overwrites y.  No workspace; y fp32 [M, N]. */
int qlinear_gemm_a8(const void* qx, const float* sx, const void* W_packed, const void* scales, int fmt, int M, int N,
                    int K, float* y, int accumulate, void* stream);

/* act_quant_i8_g128 -- per token per 128 values ("keptn/gemma4-12b-i8g",
 * table "Format"): on the fp32 group v (rotated as hadamard128_rotate but
 * NOT rounded to bf16 when rotate != 0), amax = max|v|, s = fp32(amax/127),
 * q = clamp(rne(fp32(v * fp32(127/amax))), -127, 127); amax = 0 gives s = 0,
 * q = 0.  x bf16 [M, K]; q int8 [M, K]; s fp32 [M, K/128]. */
int act_quant_i8_g128(const void* x, int M, int K, int rotate, int8_t* q, float* s, void* stream);

/* act_quant_e4m3_g128 -- the same rule with E4M3 codes (QL_FP8A8_B128_BF16's
 * activations): s = fp32(amax/448), q = e4m3(fp32(v * fp32(448/amax))) rounded
 * to nearest even and saturated to +-448 (448 is the largest finite E4M3
 * value); amax = 0 gives s = 0, q = 0.  x bf16 [M, K]; q E4M3 bytes [M, K];
 * s fp32 [M, K/128]. */
int act_quant_e4m3_g128(const void* x, int M, int K, int rotate, uint8_t* q, float* s, void* stream);

/* hadamard128_rotate -- y = per-128-block orthonormal Walsh-Hadamard
 * transform of x along K, Sylvester order (the "attention join" of
 * "gemma4-26b-a4b-dflash-i8" writes the experts' input in this domain).
 * fp32 butterflies with strides 1, 2, ..., 64, then x fp32(1/sqrt(128)),
 * rounded to bf16.  x, y bf16 [M, K]; y may equal x (in place). */
int hadamard128_rotate(const void* x, int M, int K, void* y, void* stream);

/* Stacked expert weights of one MoE gate_up projection. */
typedef struct {
    int E;              /* number of experts                                    */
    int N;              /* output rows per expert (gate and up halves together) */
    int K;              /* hidden size, multiple of 128                          */
    int fmt;            /* QL_I8_G128_BF16, QL_I8_G128_F16, QL_FP8_B128_BF16 or
                           QL_FP8A8_B128_BF16 (the fp8 experts with E4M3
                           activations, quantised once per token)            */
    int flags;          /* QL_HADAMARD when the experts are in the rotated domain */
    const void* codes;  /* device, [E] consecutive packed weights of [N, K]      */
    const void* scales; /* device, [E] consecutive scale arrays                  */
} ql_experts;

/* moe_permute -- group the T*topk (token, slot) pairs by expert: counts[E],
 * offsets[E+1] (exclusive prefix sum) and perm[T*topk], the flat pair index
 * t*topk + j in (expert, t, j) order.  Ids outside [0, E) are left out of
 * every segment (perm is then shorter than T*topk; its tail holds -1) and set
 * QL_DEVERR_EXPERT_ID.  All arrays device int32. */
int moe_permute(const int32_t* topk_ids, int T, int topk, int E, int32_t* counts, int32_t* offsets,
                int32_t* perm, void* stream);

/* Workspace bytes moe_gate_up needs. */
int moe_workspace_size(const ql_experts* experts, int T, int topk, size_t* bytes);

/* moe_gate_up -- the routed experts' gate_up projection
 * ("gemma4-26b-a4b-dflash-i8", table "Weights"): for every pair (t, j),
 * y[t, j, :] = x~[t, :] . dequant(W_{topk_ids[t, j]})^T, where x~ is x
 * rotated once per token (bf16) when the experts carry QL_HADAMARD.  With
 * QL_FP8A8_B128_BF16 experts ("gemma4-26b-a4b-dflash-fp8" README, table
 * "Weights", with E4M3 activations) x~ is instead each token quantised once
 * as act_quant_e4m3_g128 does (rotated first with QL_HADAMARD), and
 * y[t, j, n] = sum_g sx[t, g] * s_w[n / 128, g] * sum_{k in g} qx * qw.
 * x bf16 [T, K]; topk_ids int32 [T, topk]; y fp32 [T, topk, N], overwritten.
 * topk_weights (fp32 [T, topk], may be NULL) is accepted but not applied:
 * the routing weight belongs after the down projection.  Internally:
 * rotate, permute, grouped expert GEMM, and un-permute fused into the GEMM's
 * output stores.  `experts` is a host pointer. */
int moe_gate_up(const void* x, const int32_t* topk_ids, const float* topk_weights, const ql_experts* experts,
                int T, int topk, float* y, void* ws, size_t ws_bytes, void* stream);

/* Stacked bf16 down-projection weights of the routed experts. */
typedef struct {
    int E;               /* number of experts                                  */
    int K;               /* hidden size: output rows of each down weight       */
    int I;               /* intermediate size: the gate and up halves' width,  */
                         /* multiple of 64                                      */
    const void* weights; /* device, bf16 [E][K][I] (row-major, I contiguous)    */
} ql_down_experts;

/* Workspace bytes moe_down_combine needs. */
int moe_down_workspace_size(const ql_down_experts* experts, int T, int topk, size_t* bytes);

/* moe_down_combine -- the step after moe_gate_up: the routed experts' down
 * projections, bf16 as the checkpoint ships them ("gemma4-26b-a4b-dflash-i8"
 * README, table "Weights"), and the routing-weighted sum over each token's
 * slots.  The cards give neither the activation nor the combine; this library
 * takes the Gemma family's gated MLP:
 *   a[t, j, i] = gelu(h[t, j, i]) * h[t, j, I + i],
 *     gelu(v) = 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))),
 *   out[t, n]  = sum_j topk_weights[t, j] * sum_i a[t, j, i] * W_{topk_ids[t, j]}[n, i].
 * h fp32 [T, topk, 2I]: the gate_up output (gate half first, as moe_gate_up
 * writes it); topk_ids int32 [T, topk]; topk_weights fp32 [T, topk], applied
 * as given; out fp32 [T, K], overwritten.  a is formed in fp32 and the products
 * keep fp32 precision (the bf16 tensor cores see a as three bf16 parts); the
 * sums are accumulated in any order.  Pairs with an id outside [0, E) add
 * nothing and set QL_DEVERR_EXPERT_ID.  `experts` is a host pointer. */
int moe_down_combine(const float* h, const int32_t* topk_ids, const float* topk_weights,
                     const ql_down_experts* experts, int T, int topk, float* out, void* ws, size_t ws_bytes,
                     void* stream);

/* qlinear_forward_w8a8_noalloc -- the W8A8 forward of qlinear_forward
 * (fmt QL_I8A8_G128_BF16) for callers that cannot allocate device memory,
 * such as a plugin inside a host engine that owns all device memory and
 * forbids cudaMalloc, or a latency-critical loop that must avoid cudaMalloc's
 * implicit synchronisation.  The model cards have no counterpart: this is an
 * interface choice of this library.
 *
 * Same arguments and result as qlinear_forward with fmt = QL_I8A8_G128_BF16,
 * minus the workspace: the int8 activations and their scales go to a fixed
 * array inside the library's device memory, sized for M <= QL_NOALLOC_MAX_M
 * and K <= QL_NOALLOC_MAX_K (270,336 bytes, held on every GPU that loads the
 * library until the process exits).  Larger M or K return QL_EUNSUPPORTED
 * before anything is launched.  The call allocates nothing.
 * Every call looks up the array's device address on the current device
 * (cudaGetSymbolAddress, which allocates nothing).  The first call on each
 * device also sets the decode kernel's launch attributes once; make that first
 * call before any stream capture.
 * All calls share the array: calls whose kernels may overlap on the GPU
 * (other streams, other host threads) race on it and must be serialised by
 * the caller.  Nothing in the array needs to start at zero; each call
 * rewrites what it reads. */
enum { QL_NOALLOC_MAX_M = 16, QL_NOALLOC_MAX_K = 16384 };
int qlinear_forward_w8a8_noalloc(const void* x, const void* W_packed, const void* scales, int flags, int M, int N,
                                 int K, float* y, void* stream);

/* Launch trace.  Every kernel the library launches can be bracketed by a pair
 * of CUDA events recorded on the caller's stream (also inside stream capture,
 * where they become event nodes of the graph).  ql_trace_enable(capacity)
 * creates `capacity` event pairs and starts recording from slot 0 (any
 * earlier trace is dropped); 0 stops tracing and destroys the events.  Once
 * all slots are used, further launches go unrecorded.  ql_trace_read waits
 * for the recorded stop events and returns, per slot in launch order, the
 * kind of launch (QL_KIND_*) and its duration in milliseconds (-1 if its
 * events could not be recorded); *count is the number of slots used.
 * Host-side state only: not thread safe. */
enum {
    QL_KIND_ROTATE = 1,      /* hadamard128_rotate                              */
    QL_KIND_ACT_QUANT = 2,   /* activation quantiser (also zeroes y for W8A8)   */
    QL_KIND_PREP_A16 = 3,    /* activation staging for A16 (also zeroes y)      */
    QL_KIND_SKINNY = 4,      /* decode skinny GEMM                              */
    QL_KIND_MOE_PERMUTE = 5, /* expert permutation and chunk table              */
    QL_KIND_MOE_GEMM = 6,    /* grouped expert GEMM with fused un-permute        */
    QL_KIND_PACK = 7,        /* weight packing                                  */
    QL_KIND_PREFILL = 8,     /* tensor-core prefill GEMM                        */
    QL_KIND_PREFILL_PREP = 9, /* weight scales transposed for the prefill GEMM  */
    QL_KIND_MOE_ACT = 10,     /* gelu(gate) * up ahead of the down projection   */
    QL_KIND_MOE_DOWN = 11     /* experts' down projection with the combine       */
};
int ql_trace_enable(int capacity);
int ql_trace_read(int* kinds, float* ms, int max, int* count);

/* Text of the last CUDA runtime error behind a QL_ECUDA status returned to
 * this host thread ("no error" if there was none).  Never NULL. */
const char* ql_last_cuda_error(void);

/* Bound every wait of the library's kernels for a copy, an MMA or another
 * warp's work to `ns` nanoseconds on the current device (0 restores the
 * default, 200 ms).  A wait that runs out sets QL_DEVERR_TIMEOUT, and its
 * kernel stops early, letting the copies and MMAs it already started finish
 * (those waits keep the default bound) and freeing its tensor memory; the
 * call's output is then incomplete.  For testing that path: a limit of 1 makes
 * nearly every pipeline wait run out.  Synchronises the device; host state
 * only per device, not per stream. */
int ql_set_wait_limit(unsigned long long ns);

/* Synchronise `stream`, then read and clear the device error word.
 * Returns QL_OK when it was clear, QL_EDEVICE otherwise (with *bits, if not
 * NULL, set to its QL_DEVERR_* bits), QL_ECUDA if a CUDA call failed. */
int ql_get_device_error(void* stream, unsigned* bits);

#ifdef __cplusplus
}
#endif

#endif /* QLINEAR_H */
