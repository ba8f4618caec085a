// Host-side declarations shared by the library's translation units (not part of the ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Launches `kernel` on stream s with programmatic stream serialization: the kernel may be
// dispatched while the previous kernel on the stream still runs, and orders itself after it with
// grid_dependency_wait (common.cuh) once its setup is done.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Kernel launch bookkeeping (per-kernel event timing for benchmarks).
void timing_before(const char* name, cudaStream_t s);
void timing_after(const char* name, cudaStream_t s);

// Scheduler outputs for the grouped GEMMs.  Expert e owns activation / output rows
// [row_start[e], row_start[e] + row_count[e]); those rows are cut into tile_prefix[e+1] -
// tile_prefix[e] token tiles of `chunk[e]` rows (the last may be shorter); a GEMM over
// m_tiles weight tiles per expert then has m_tiles * tile_prefix[E] work items.
struct TileSched {
  const int32_t* row_start;
  const int32_t* row_count;
  const int32_t* tile_prefix;  // [E+1]
  const int32_t* chunk;        // [E]
};

// route / align / scheduler (route_align.cu)
cudaError_t launch_route(const float* logits, int T, int E, int k, int renormalize, int32_t* ids, float* w,
                         cudaStream_t s);
int align_blocks(int T, int k);
// Token-tile schedules the alignment builds from each expert's count.  The main schedule cuts
// an expert's rows into balanced tiles of at most nmax rows.  With thin_tile_prefix given, an
// expert with at most thin_rows rows goes to the thin schedule instead (tiles of at most
// thin_nmax rows), and each schedule's row_count holds the expert's rows in that schedule (0 in
// the other).
struct SchedOut {
  int nmax = 0;
  int32_t* tile_prefix = nullptr;  // [E+1]
  int32_t* chunk = nullptr;        // [E]
  int32_t* row_count = nullptr;    // [E], or null: the main schedule takes every expert (= counts)
  int thin_rows = 0;
  int thin_nmax = 0;
  int32_t* thin_tile_prefix = nullptr;
  int32_t* thin_chunk = nullptr;
  int32_t* thin_row_count = nullptr;
  int32_t* thin_row_prefix = nullptr;  // [E+1] exclusive scan of thin_row_count
};
// blockcnt: [align_blocks * E] int32 scratch.  sched may be null (no scheduler).
cudaError_t launch_align(const int32_t* ids, int T, int k, int E, int align, int32_t* counts, int32_t* offsets,
                         int32_t* sorted_ids, int32_t* inv_pos, int32_t* blockcnt, const SchedOut* sched,
                         cudaStream_t s);
// Scheduler for the public grouped GEMM: from expert_offsets [E+1] (arbitrary row counts).
cudaError_t launch_sched_from_offsets(const int32_t* offsets, int E, int M, int nmax, int32_t* row_count,
                                      int32_t* tile_prefix, int32_t* chunk, cudaStream_t s);

// permute / combine (permute_combine.cu)
// x rows -> expert-sorted interleaved fp16 rows for every pair p (or, with ids / cls_rows given,
// for the pairs whose expert has cls_rows[ids[p]] > 0): row r = inv_pos[p] holds
// fp16(x[p/k] * 2^-x_exp[r]) with x_exp[r] >= 0 the smallest exponent that fits the row into
// fp16.  For every placed pair ovf_flag[r] is cleared, and for the converted rows the I/32 words
// of ovf_mask too (the gated GEMM's overflow marks).
cudaError_t launch_permute_w4(const uint16_t* x_bf16, const int32_t* inv_pos, const int32_t* ids,
                              const int32_t* cls_rows, int T, int k, int H, __half* x_perm, int32_t* x_exp,
                              int32_t* ovf_flag, uint32_t* ovf_mask, int I, cudaStream_t s);
// rows of a (bf16 or fp16) -> interleaved fp16 rows out[r] = fp16(a[r] * 2^-x_exp[r]), x_exp[r]
// the smallest exponent >= 0 that fits the row into fp16
cudaError_t launch_convert_rows(const uint16_t* a, int a_is_bf16, int M, int K, __half* out, int32_t* x_exp,
                                cudaStream_t s);
cudaError_t launch_combine(const float* y_perm, const int32_t* inv_pos, const float* topk_w, int T, int k, int H,
                           void* out, int out_fp32, cudaStream_t s);

// W4A16 grouped GEMM (gemm_w4a16.cu): token tiles of at most this many rows (the accumulators
// and the A ring share tensor memory)
constexpr int kWideTileRows = 192;
enum OutKind { OUT_H_F16_INTERLEAVED = 0, OUT_F32 = 1, OUT_BF16 = 2, OUT_PLANES = 3 };
struct W4GemmProblem {
  const int32_t* w_q;  // [E, rows_per_expert, K/8]
  const uint16_t* w_s; // [E, rows_per_expert, K/32]
  const __half* act;   // [act_rows, K] fp16, K interleaved in groups of 8
  int act_rows;
  int K, E, rows_per_expert;
  bool gated;          // gate rows [0, I), up rows [I, 2I); output h [*, I]
  int I;               // gated only
  TileSched sched;
  int nmax;
  void* out;
  int out_ld;          // elements per output row
  OutKind out_kind;
  int splits = 1;          // plain outputs: K split this many ways into `part`, then reduce_splits
  float* part = nullptr;   // [splits, act_rows, out_ld] fp32
  // Range handling of the fp16 operands (exact power-of-two scalings):
  const int32_t* acc_exp = nullptr;  // per act row e (or null): accumulators times 2^e before the epilogue
  int32_t* ovf_flag = nullptr;       // gated (required): [act_rows], set to 1 for a row with an h value
                                     // beyond fp16, which is then stored as h * 2^-16 ...
  uint32_t* ovf_mask = nullptr;      // ... and marked in this [act_rows, I/32] bit mask (by stored
                                     // position); launch_h_rescale rescales such rows
};
cudaError_t launch_w4a16_gemm(const W4GemmProblem& p, cudaStream_t s);
// After a gated fp16 GEMM: every row r with ovf_flag[r] set is rescaled in place to
// h * 2^-c with the smallest c >= 1 that fits the row into fp16 (h_exp[r] = c), the others get
// h_exp[r] = 0.  Clears nothing; the rows' flags and masks are cleared by launch_permute_w4.
cudaError_t launch_h_rescale(__half* h, int rows, int I, const int32_t* ovf_flag, const uint32_t* ovf_mask,
                             int32_t* h_exp, cudaStream_t s);

// W4A16 grouped GEMM for decode-sized experts on the int8 tensor cores (gemm_w4i8.cu).
// Activations as 16-bit fixed-point planes: per (row, 128-K block) scale s, X = rint(x/s)
// = 256*hi + lo.  Plane matrix int8 [2*rows, K]: row 2r holds hi of row r, row 2r+1 its lo,
// with K in the order (0,2,4,6,1,3,5,7) inside every 8-group; |X| <= kFixMax.  Meta int32
// [rows, ceil(K/256), 12]: per 256-K stage, for each of its eight 32-K groups kFixBias - 8 *
// (sum of X over the group), then the scales of its two 128-K blocks (fp32 bits), then two
// unused words.  kFixBias is the fp32 bit pattern of 1.5 * 2^23: adding an integer v with
// |v| < 2^22 to it gives the bits of the float 1.5 * 2^23 + v, an exact int-to-float step.
constexpr int kFixMax = 16383;
constexpr int32_t kFixBias = 0x4B400000;
constexpr float kFixBiasF = 12582912.0f;
constexpr int kMetaWords = 12;
__host__ __device__ inline int meta_words_per_row(int K) { return (K + 255) / 256 * kMetaWords; }
struct W4I8Problem {
  const int32_t* w_q;   // [E, rows_per_expert, K/8]
  const uint16_t* w_s;  // [E, rows_per_expert, K/32]
  const int8_t* act;    // planes [2*act_rows, K]
  const int32_t* act_meta;
  int act_rows;
  int K, E, rows_per_expert;
  bool gated;  // output planes of h [2*act_rows, I]
  int I;
  TileSched sched;
  OutKind out_kind;  // OUT_PLANES (gated), OUT_F32 or OUT_BF16
  void* out;
  int32_t* out_meta;  // planes only: meta of h
  int out_ld;         // OUT_F32/OUT_BF16: elements per output row (planes: I)
  int splits = 1;     // plain outputs: K split this many ways into `part`, then reduce_splits
  float* part = nullptr;  // [splits, act_rows, out_ld] fp32
};
constexpr int kI8TileRows = 8;  // token rows per tile of the int8 GEMM
cudaError_t launch_w4i8_gemm(const W4I8Problem& p, cudaStream_t s);
// 128-row weight tiles per work item of the int8 GEMM: 2 (gate and up, or two adjacent output
// tiles when the rows come in 256s), else 1
int w4i8_tiles_per_item(bool gated, int rows_per_expert);
// 128-row weight tiles per work item of the fp16 GEMM's plain (down) form: 2 when the output rows
// come in 256s, else 1
int w4a16_tiles_per_item(int rows_per_expert);
// out[r][n] = sum over s = 0..splits-1 (in that order) of part[s][r][n] for the rows of every
// expert e, [row_start[e], row_start[e] + row_count[e]), stored as fp32 (out_fp32) or bf16 (RNE)
cudaError_t launch_reduce_splits(const float* part, int splits, int rows, int N, const int32_t* row_start,
                                 const int32_t* row_count, int E, void* out, int out_fp32, cudaStream_t s);
// Planes of the K-vectors x_src: plane row r takes source row r (inv_pos == null, k == 1),
// or for every pair p plane row inv_pos[p] takes source row p / k.
// Alignment (align = 1) with the int8 GEMM's tile schedule and the fixed-point planes of every
// pair's row, in one launch, for batches where fused_align_planes_ok(T, k, E).
bool fused_align_planes_ok(int T, int k, int E);
cudaError_t launch_align_planes(const int32_t* ids, int T, int k, int E, const uint16_t* x_bf16, int K,
                                int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* inv_pos,
                                int32_t* tile_prefix, int32_t* chunk, int nmax, int8_t* planes, int32_t* meta,
                                cudaStream_t s);
cudaError_t launch_planes(const uint16_t* a, int a_is_bf16, const int32_t* inv_pos, int n_pairs, int k, int K,
                          int8_t* planes, int32_t* meta, cudaStream_t s);
// Planes of the rows of the thin schedule's experts: row_prefix [E+1] is the exclusive scan of
// their row counts, and list row j < row_prefix[E] <= max_rows is row j - row_prefix[e] of expert
// e; its sorted row offsets[e] + j - row_prefix[e] takes source row sorted_ids[that row] / k.
cudaError_t launch_planes_list(const uint16_t* x_bf16, const int32_t* row_prefix, const int32_t* offsets,
                               const int32_t* sorted_ids, int E, int k, int max_rows, int K, int8_t* planes,
                               int32_t* meta, cudaStream_t s);

// block-FP8 grouped GEMM (gemm_fp8.cu)
struct F8GemmProblem {
  const uint8_t* w;        // e4m3 [E, rows_per_expert, K]
  const float* w_scale;    // [E, rows_per_expert/128, K/128]
  const uint8_t* act;      // e4m3 [act_rows, K]
  const float* x_scale;    // transposed activation scales [K/128, act_rows]
  int act_rows;
  int K, E, rows_per_expert;
  bool gated;              // gate rows [0, I), up rows [I, 2I); output e4m3 h [*, I] + h_scale
  int I;
  TileSched sched;
  void* out;
  int out_ld;
  float* h_scale;          // gated: [I/128, act_rows]
  int nmax;                // token rows per tile: 32 or 64 (the cap the schedule was built with)
};
cudaError_t launch_fp8_gemm(const F8GemmProblem& p, cudaStream_t s);
cudaError_t launch_permute_fp8(const uint8_t* x, const float* xs, const int32_t* inv_pos, int T, int k, int H,
                               uint8_t* x_perm, float* xs_t, int P, cudaStream_t s);

// W4A8 grouped GEMM (gemm_mx.cu): MXFP4 weights x e4m3 activations with E8M0 scales per 32 K
struct MxGemmProblem {
  const uint8_t* w;        // E2M1 codes [E, rows_per_expert, K/2] (even K in the low nibble), 32-byte aligned
  const uint8_t* w_sf;     // E8M0 [E, K/128, rows_per_expert, 4]
  const uint8_t* act;      // e4m3 [act_rows, K]
  const uint32_t* x_sf;    // [K/128, act_rows]: byte j = E8M0 code of the row's K group 4*blk + j
  int act_rows;
  int K, E, rows_per_expert;
  bool gated;              // gate rows [0, I), up rows [I, 2I); output e4m3 h [*, I] + h_sf
  int I;
  TileSched sched;
  void* out;
  int out_ld;
  uint8_t* h_sf;           // gated: [I/128, act_rows, 4] (the x_sf layout of the down GEMM's input)
  int nmax;                // token rows per tile: 32 or 112 (the cap the schedule was built with)
};
cudaError_t launch_mx_gemm(const MxGemmProblem& p, cudaStream_t s);
// the single grouped GEMM's schedule from caller offsets and its rows' activation planes, one launch
cudaError_t launch_sched_planes(const int32_t* offsets, int E, int nmax, int32_t* row_count, int32_t* tile_prefix,
                                int32_t* chunk, const uint16_t* a, int a_is_bf16, int M, int K, int8_t* planes,
                                int32_t* meta, cudaStream_t s);
cudaError_t launch_permute_mx(const uint16_t* x, const int32_t* inv_pos, int T, int k, int H, uint8_t* x_perm,
                              uint32_t* x_sf, int P, cudaStream_t s);

// driver entry point for tensor maps (api.cu)
// 2-D tiled tensor map over a row-major [rows, cols] tensor at `base` (zero fill out of bounds).
CUresult encode_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows,
                        uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz);
int sm_count();
uint64_t wait_limit_ns();

}  // namespace moe
