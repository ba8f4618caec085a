/*
 * moe.h — C ABI of the routed, weight-quantized Mixture-of-Experts layer for NVIDIA B200
 * (sm_100a): softmax top-k router, token-to-expert alignment, W4A16 and block-FP8 grouped
 * expert GEMMs with a fused SiLU*up epilogue, and a deterministic weighted combine.
 *
 * Where the operations are defined (titles of the pages that describe the method):
 *  - "AWS Details H200 Kernel Optimizations for MoE Inference", section "Three bottlenecks
 *    require different fixes": a fused MoE operator combines token routing, data movement
 *    and expert calculations (moe_route, moe_align, moe_w4a16_forward).
 *  - "Chord Rewrites the INT4 MoE Kernel for Kimi K2.x ...", second paragraph: W4A16 =
 *    BF16 inputs, INT4 weights dequantized with one BF16 scale per group of 32 weights, gate /
 *    up / down projections, scheduling from each expert's actual token count
 *    (moe_w4a16_forward, moe_w4a16_gemm).
 *  - "Helion Brings Autotuned GEMM Kernels to vLLM ...", section "Scope: Hopper and
 *    quantized formats": Block_FP8 = FP8 with 1x128 activation scaling and 128x128 weight
 *    scaling (moe_blockfp8_forward).
 *  - "[Performance] W4A8 MoE GEMM significantly slower than W4A16 on H200" (Humming issue),
 *    opening report: W4A8 = MXFP4 weights x FP8 activations in K groups (moe_w4a8_forward).
 *  The router (softmax, top-k, renormalised weights), SiLU*up activation and top-k-weighted
 *  combine are not written out on those pages; this library takes the textbook readings
 *  stated with each call below.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major, 16-byte aligned.
 *    The library never allocates, frees or synchronises inside these calls; all scratch
 *    memory is the caller's workspace (size from the matching *_workspace_size call), except
 *    for moe_align_noalloc, whose scratch is a fixed array inside the library (see there).
 *  - Work is enqueued on `stream` and returns immediately; no host reads of device data, so
 *    the calls that take a workspace may be captured in a CUDA graph.
 *  - Argument, shape and alignment errors return an error code synchronously with nothing
 *    enqueued.  A failed kernel launch returns MOE_ERR_CUDA.
 *  - Faults the GPU detects (an expert id outside [0,E), a wait that timed out) are recorded
 *    in a per-device status word that moe_get_device_status() reads.
 *  - There is no CPU fallback: without a usable sm_100 GPU the calls return MOE_ERR_CUDA or
 *    MOE_ERR_UNSUPPORTED.
 *  - Shape limits: 1 <= k <= E <= 1024, T >= 1, H and I multiples of 128, T*k < 2^31.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size */
  MOE_ERR_UNSUPPORTED = 2,  /* shape outside the limits above, or no sm_100 device */
  MOE_ERR_WORKSPACE = 3,    /* workspace smaller than the *_workspace_size value */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed */
  MOE_ERR_TIMEOUT = 5,      /* (device status) a bounded in-kernel wait gave up */
  MOE_ERR_DEVICE_CHECK = 6  /* (device status) an input failed a device-side check */
} moe_status_t;

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status_t s);

/* ------------------------------------------------------------------ a1: router
 * Per token t: the k experts with the largest logits, ordered by (logit descending, expert
 * index ascending); slot s holds the s-th.  Weights are the softmax of the logits over all
 * E experts restricted to the winners, renormalised to sum to 1 when `renormalize` != 0 (then
 * w_s = exp(l_s - l_max) / sum_{s'} exp(l_s' - l_max)), otherwise the plain softmax
 * probabilities.  Logits must be finite.
 *   logits   fp32  [T, E]   (in)
 *   topk_ids int32 [T, k]   (out)
 *   topk_w   fp32  [T, k]   (out)
 * One warp per token; no workspace. */
moe_status_t moe_route(const float* logits, int T, int E, int k, int renormalize, int32_t* topk_ids,
                       float* topk_w, cudaStream_t stream);

/* ------------------------------------------------------------------ a2: alignment
 * Stable counting sort of the T*k (token, slot) pairs by expert.  Pair p = t*k + s.
 *   expert_counts  int32 [E]     pairs routed to each expert
 *   expert_offsets int32 [E+1]   offsets[0] = 0, offsets[e+1] = offsets[e] +
 *                                ceil(counts[e]/align)*align
 *   sorted_ids     int32 [moe_align_capacity()]  sorted_ids[offsets[e] + r] = r-th pair of
 *                  expert e in ascending p; the padding of each expert's run holds the
 *                  sentinel T*k; entries at and beyond offsets[E] are left untouched
 *   inv_pos        int32 [T*k]   row of pair p in sorted_ids (-1 for a pair whose id is out of
 *                  range; such pairs are skipped and MOE_ERR_DEVICE_CHECK is recorded)
 * align >= 1.  ws: moe_align_workspace_size(T, k, E) bytes. */
size_t moe_align_capacity(int T, int k, int E, int align); /* T*k + E*(align-1) entries */
size_t moe_align_workspace_size(int T, int k, int E);
moe_status_t moe_align(const int32_t* topk_ids, int T, int k, int E, int align, int32_t* expert_counts,
                       int32_t* expert_offsets, int32_t* sorted_ids, int32_t* inv_pos, void* ws, size_t ws_bytes,
                       cudaStream_t stream);

/* moe_align_noalloc: the same alignment as moe_align, for callers that cannot allocate device
 * memory and have no workspace to pass (e.g. a plugin inside a host framework that owns all
 * device buffers, or a deployment with a device memory budget fixed at start-up).  The pages
 * describing the method have no counterpart of this call; it exists for those callers.
 * The scratch lives in a fixed 512 KiB array inside the library (131072 int32, kept on every
 * GPU that loads the library until the process exits); a call needs ceil(T*k/512)*E of them and
 * returns MOE_ERR_UNSUPPORTED when that is more.  It allocates nothing.  Each call outside stream
 * capture looks up the array's device address on the current device (cudaGetSymbolAddress, no
 * allocation) and remembers it; a call on a stream that is being captured uses the remembered
 * address, so make the first call on each device before any stream capture.  Every call
 * reuses the same array and overwrites each entry it reads, so earlier contents never leak
 * into a result; calls that overlap on the GPU race on the array and must be serialised by the
 * caller.  Arguments and outputs otherwise as moe_align. */
moe_status_t moe_align_noalloc(const int32_t* topk_ids, int T, int k, int E, int align, int32_t* expert_counts,
                               int32_t* expert_offsets, int32_t* sorted_ids, int32_t* inv_pos, cudaStream_t stream);

/* ------------------------------------------------------------------ a2..a8: W4A16 layer
 * out[t] = sum_{s<k} topk_w[t,s] * y_{t,s},   y = h . W2[e]^T,   h_j = SiLU(g_j) * g_{I+j},
 * g = x[t] . W13[e]^T,   e = topk_ids[t,s],   SiLU(v) = v / (1 + e^-v),
 * with dequantized weights W[n][c] = int4(q) * bf16(scale of (n, c/32)).
 *   x      bf16  [T, H]
 *   w13_q  int32 [E, 2I, H/8]  rows 0..I-1 = gate, I..2I-1 = up; word c/8 of row n holds K
 *                              indices 8*(c/8)..+7, nibble j (bits 4j..4j+3) = index 8w+j,
 *                              two's complement in [-8, 7]
 *   w13_s  bf16  [E, 2I, H/32] one scale per 32 K elements per output row
 *   w2_q   int32 [E, H, I/8],  w2_s bf16 [E, H, I/32]   (down projection, same packing)
 *   out    bf16  [T, H] (RNE of the fp32 result), or fp32 [T, H] when out_fp32 != 0
 * Numerics: each expert runs on one of two GEMMs, chosen per expert from its token count (every
 * expert on the first when T <= 64; for larger T an expert with at most 8 rows on the first and
 * one with more on the second):
 *   int8 GEMM: the INT4 values meet 16-bit fixed-point activations on the int8 tensor cores:
 *     per (row, 128-K block) s = max(|x|max, 1e-30) / 16383 and X = rint(x / s); each 32-K
 *     group's sum of q*X is exact in int32 and is scaled by (weight scale * s) and
 *     accumulated in fp32; h is stored the same way (one scale per token per 128 rows of I).
 *     The only rounding besides fp32 accumulation is X (at most s / 2 per element); any finite
 *     x is taken.
 *   fp16 GEMM: activations and dequantized weights are fed to the tensor cores in fp16 with fp32
 *     accumulation.  Each permuted row of x is multiplied by an exact power of two 2^-c (c >= 0
 *     the smallest that brings the row's largest magnitude inside fp16, so c = 0 for every row
 *     already inside it) and the row's accumulators are multiplied by 2^c, so any finite x is
 *     taken; the conversion is exact for values inside the fp16 normal range after that
 *     scaling.  The dequantized weights q*s are exact in fp16 while |q*s| is inside its normal
 *     range.  h is rounded to fp16; a value of h beyond fp16 is stored times 2^-16 and its row
 *     is then brought to one power-of-two scale 2^-c (c >= 1) before the down projection,
 *     which multiplies that row's accumulators by 2^c.  An h beyond even that (|h| >= 65520 *
 *     2^16, about 4.3e9) and a non-finite x record MOE_ERR_DEVICE_CHECK.
 * The combine sums the k slots in fp32 in slot order, so the result is deterministic run to
 * run.
 * ws: moe_w4a16_workspace_size(T, H, I, E, k) bytes. */
typedef struct {
  const void* x;
  const int32_t* topk_ids;
  const float* topk_w;
  const int32_t* w13_q;
  const void* w13_s;
  const int32_t* w2_q;
  const void* w2_s;
  int T, H, I, E, k;
  void* out;
  int out_fp32;
} moe_w4a16_args;

size_t moe_w4a16_workspace_size(int T, int H, int I, int E, int k);
moe_status_t moe_w4a16_forward(const moe_w4a16_args* args, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------ a9: block-FP8 layer
 * Same layer with e4m3 (OCP E4M3FN) operands:
 *   x      e4m3 [T, H] with fp32 scales xs [T, H/128]        (x = q * xs[t][c/128])
 *   w13    e4m3 [E, 2I, H] with fp32 scales [E, 2I/128, H/128] (W = q * s[n/128][c/128])
 *   w2     e4m3 [E, H, I]  with fp32 scales [E, H/128, I/128]
 * The intermediate h = SiLU(gate) * up (fp32) is requantized per (pair, 128-column group):
 * s = max(amax, 1e-10) / 448, q = e4m3_rne_satfinite(h / s), before the down projection.
 * out bf16 [T, H] or fp32 when out_fp32 != 0.
 * ws: moe_blockfp8_workspace_size(T, H, I, E, k) bytes. */
typedef struct {
  const uint8_t* x;
  const float* xs;
  const int32_t* topk_ids;
  const float* topk_w;
  const uint8_t* w13;
  const float* w13_s;
  const uint8_t* w2;
  const float* w2_s;
  int T, H, I, E, k;
  void* out;
  int out_fp32;
} moe_blockfp8_args;

size_t moe_blockfp8_workspace_size(int T, int H, int I, int E, int k);
moe_status_t moe_blockfp8_forward(const moe_blockfp8_args* args, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Diagnostic view of the block-FP8 layer's requantized intermediate: given the workspace `ws`
 * of a moe_blockfp8_forward call with the same (T, H, I, E, k), returns device pointers into
 * it (nothing is enqueued or read):
 *   inv_pos    int32 [T*k]          row r of pair p = t*k + s (as moe_align's inv_pos)
 *   h          e4m3  [T*k, I]       row r = the e4m3 codes of the pair's requantized h
 *   h_scale_t  fp32  [I/128, T*k]   h_scale_t[g][r] = the scale of row r's 128-column group g
 * so that h of pair p, column j, is e4m3(h[r][j]) * h_scale_t[j/128][r] with r = inv_pos[p].
 * The contents are valid once that call's work on its stream has completed and until the next
 * call that uses the workspace.  Shape errors MOE_ERR_UNSUPPORTED, a null or misaligned
 * argument MOE_ERR_INVALID_ARG. */
moe_status_t moe_blockfp8_intermediate(const void* ws, int T, int H, int I, int E, int k, const int32_t** inv_pos,
                                       const uint8_t** h, const float** h_scale_t);

/* ------------------------------------------------------------------ W4A8 layer
 * The W4A8 configuration of "[Performance] W4A8 MoE GEMM significantly slower than W4A16 on
 * H200" (Humming issue, opening report): MXFP4 weights and FP8 activations quantized in groups
 * of 32 along K.  The same routed layer as moe_w4a16_forward with
 *   W[e][n][c] = e2m1(code) * 2^(sf - 127)
 * where code is the 4-bit E2M1 element (sign, 2 exponent bits with bias 1, 1 mantissa bit;
 * magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6) and sf the E8M0 scale code of the 32-element K group.
 * The activations (x, then h = SiLU(gate) * up held in fp32) are quantized per token and 32-K
 * group to E4M3 with an E8M0 scale (the microscaling reading of the report's group-32 FP8):
 * 2^X is the smallest power of two, X in [-127, 127], with amax <= 448 * 2^X, and the codes are
 * e4m3_rne(v * 2^-X).  The tensor cores apply both scales per 32 K (tcgen05 block-scaled MMA)
 * and accumulate the whole reduction in fp32.
 *   x        bf16 [T, H]
 *   topk_ids int32 [T, k], topk_w fp32 [T, k] (as moe_route returns them)
 *   w13      uint8 [E, 2I, H/2]: two E2M1 codes per byte along K, even K index in the low
 *            nibble; gate rows [0, I), up rows [I, 2I); 32-byte aligned
 *   w13_sf   uint8 [E, H/128, 2I, 4]: w13_sf[e][b][n][j] = E8M0 code of row n's K group 4b + j
 *   w2       uint8 [E, H, I/2], w2_sf uint8 [E, I/128, H, 4] (same packing); 32-byte aligned
 *   out      bf16 [T, H] or fp32 when out_fp32 != 0
 * An inf or NaN in x or h is flagged in the device status word (MOE_ERR_DEVICE_CHECK).
 * ws: moe_w4a8_workspace_size(T, H, I, E, k) bytes. */
typedef struct {
  const void* x;
  const int32_t* topk_ids;
  const float* topk_w;
  const uint8_t* w13;
  const uint8_t* w13_sf;
  const uint8_t* w2;
  const uint8_t* w2_sf;
  int T, H, I, E, k;
  void* out;
  int out_fp32;
} moe_w4a8_args;

size_t moe_w4a8_workspace_size(int T, int H, int I, int E, int k);
moe_status_t moe_w4a8_forward(const moe_w4a8_args* args, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Diagnostic view of the W4A8 layer's quantized intermediate, like moe_blockfp8_intermediate:
 *   inv_pos  int32 [T*k]               row r of pair p = t*k + s
 *   h        e4m3  [T*k, I]            row r = the codes of the pair's quantized h
 *   h_sf     uint8 [I/128, T*k, 4]     h_sf[b][r][j] = E8M0 code of row r's column group 4b + j
 * so that h of pair p, column j, is e4m3(h[r][j]) * 2^(h_sf[j/128][r][(j/32)%4] - 127). */
moe_status_t moe_w4a8_intermediate(const void* ws, int T, int H, int I, int E, int k, const int32_t** inv_pos,
                                   const uint8_t** h, const uint8_t** h_sf);

/* ------------------------------------------------------------------ grouped W4A16 GEMM
 * No activation: rows [expert_offsets[e], expert_offsets[e+1]) of a are multiplied by
 * expert e's dequantized weights:  out[m][n] = sum_c a[m][c] * W[e][n][c].
 *   a              bf16 (a_is_bf16 != 0) or fp16 [M, K]
 *   w_q            int32 [E, N, K/8], w_s bf16 [E, N, K/32] (packing as in moe_w4a16_forward)
 *   expert_offsets int32 [E+1] (device), non-decreasing, offsets[0] >= 0, offsets[E] <= M;
 *                  rows outside every range are not written
 *   out            bf16 or fp32 (out_fp32 != 0) [M, N]
 * K and N multiples of 128.  M <= 64 runs the int8 tensor-core path and M > 64 the fp16 path,
 * with the numerics described at moe_w4a16_forward.  When the shape has few work items
 * (N/128 x ceil(M/tile rows), 8 or 256 rows per tile, well below the SM count) the K range is
 * split and the fp32 partial sums are added in a fixed order, so results stay identical run
 * to run.
 * ws: moe_w4a16_gemm_workspace_size(M, K, N, E) bytes (includes the partial sums). */
size_t moe_w4a16_gemm_workspace_size(int M, int K, int N, int E);
moe_status_t moe_w4a16_gemm(const void* a, int a_is_bf16, const int32_t* w_q, const void* w_s,
                            const int32_t* expert_offsets, int M, int K, int N, int E, void* out, int out_fp32,
                            void* ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------ status, diagnostics
 * moe_get_device_status: synchronises `stream`, returns the device status word of the
 * current device (MOE_OK if no kernel recorded a fault) and clears it. */
moe_status_t moe_get_device_status(cudaStream_t stream);

/* Test hook: launches one CTA that waits on an mbarrier nothing will ever arrive on, with a
 * bound of `limit_ns` nanoseconds (1 <= limit_ns <= 10^9).  The wait gives up, the kernel
 * records MOE_ERR_TIMEOUT in the status word and returns normally. */
moe_status_t moe_debug_wait_timeout(int64_t limit_ns, cudaStream_t stream);

/* Per-kernel timing for benchmarks: while enabled, every kernel launch of this library is
 * bracketed by a pair of CUDA events on its stream.  moe_timing_read synchronises the
 * device, writes for up to `max` kernel names the summed milliseconds and launch counts
 * since the last read (names are static strings), returns how many kernel names there are,
 * and resets the sums.  Not thread-safe; keep disabled outside benchmarks. */
moe_status_t moe_timing_enable(int enable);
int moe_timing_read(const char** names, double* ms, int* launches, int max);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
