// The C ABI (include/moe.h): argument checks, workspace carving, tensor-map encoding,
// launch sequencing, the device status word and the benchmark timing hooks.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace moe {


// ------------------------------------------------------------------ device facts
namespace {
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
int g_cc_major[kMaxDevices];
std::mutex g_mu;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}
bool device_facts(int d) {
  if (d < 0 || d >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sm_count[d] > 0) return true;
  int sms = 0, major = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess) return false;
  g_cc_major[d] = major;
  g_sm_count[d] = sms;
  return true;
}

// sm_100 family only: the kernels are built for sm_100a
moe_status_t check_device() {
  const int d = current_device();
  if (!device_facts(d)) return MOE_ERR_CUDA;
  return g_cc_major[d] == 10 ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

bool aligned(const void* p, size_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Sub-allocates a caller workspace; with a null base it only measures.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(size_t n) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += n * sizeof(T);
    return p;
  }
};
}  // namespace

int sm_count() {
  const int d = current_device();
  return device_facts(d) ? g_sm_count[d] : 148;
}

uint64_t wait_limit_ns() { return 1000000000ull; }  // 1 s per barrier wait

// ------------------------------------------------------------------ tensor maps
CUresult encode_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows,
                        uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!fn) {
      void* ptr = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !ptr)
        return CUDA_ERROR_NOT_FOUND;
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
  }
  const cuuint64_t gdim[2] = {cols, rows};
  const cuuint64_t gstride[1] = {row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// ------------------------------------------------------------------ timing hooks
namespace {
bool g_timing_on = false;
struct Rec {
  const char* name;
  cudaEvent_t a, b;
};
struct Agg {
  const char* name;
  double ms;
  int n;
};
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_free_ev;
std::vector<Agg> g_agg;
cudaEvent_t get_event() {
  if (!g_free_ev.empty()) {
    cudaEvent_t e = g_free_ev.back();
    g_free_ev.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

// Every kernel launch sits between these two calls.  They open and close an NVTX range named
// after the kernel (a timeline tool attached to the process shows which launch each range
// enqueued; without one the calls do nothing) and, while moe_timing_enable(1) is in effect,
// bracket the launch with CUDA events for moe_timing_read.
void timing_before(const char* name, cudaStream_t s) {
  nvtxRangePushA(name);
  if (!g_timing_on) return;
  Rec r{name, get_event(), get_event()};
  cudaEventRecord(r.a, s);
  g_recs.push_back(r);
}
void timing_after(const char*, cudaStream_t s) {
  nvtxRangePop();
  if (!g_timing_on || g_recs.empty()) return;
  cudaEventRecord(g_recs.back().b, s);
}

// ------------------------------------------------------------------ workspace layouts
namespace {
// Decode-sized problems (no expert can get more than 64 rows) run entirely on the int8
// tensor-core GEMM with activations as 16-bit fixed-point planes.
bool use_i8(int max_rows_per_expert) { return max_rows_per_expert <= 64; }

// Larger layer calls choose per expert, from its actual token count: an expert with at most
// kThinRows rows runs on the int8 GEMM (8-row token tiles; its cost is streaming the weights
// plus a promotion step per live token), one with more on the fp16 GEMM (tiles of up to 192
// rows, where dequantizing a weight tile once serves many tokens, but a tile of few tokens
// costs as much dequantization as a full one).  Measured on the 384-expert model with skewed
// routing at T = 128 ... 8192: switch points of 4, 8 and 16 rows (once both GEMMs had their
// current form; earlier, 16 against 32, 48 and 64), 8 fastest or within 4% of the fastest at
// every T (T = 8192: 4-6% faster than 16; T = 128 and 512: 20% faster) - one int8 tile of 8
// rows, where an expert of 9-16 rows took two passes over its weights.
#ifndef MOE_THIN_ROWS
#define MOE_THIN_ROWS 8
#endif
constexpr int kThinRows = MOE_THIN_ROWS;

// 16-bit fixed-point planes of an activation matrix [rows, K]
struct Planes {
  int8_t* x;      // [2*rows, K]: hi and lo rows interleaved
  int32_t* meta;  // [rows, meta_words_per_row(K)]: group sums and block scales
};
Planes take_planes(Carver& c, size_t rows, int K) {
  Planes q;
  q.x = c.take<int8_t>(2 * rows * K);
  q.meta = c.take<int32_t>(rows * meta_words_per_row(K));
  return q;
}

struct FwdWs {
  int32_t *counts, *offsets, *sorted, *inv, *blockcnt;
  int32_t *tile_prefix, *chunk, *row_count;                  // fp16 GEMM schedule (wide experts)
  int32_t *thin_tile_prefix, *thin_chunk, *thin_row_count, *thin_row_prefix;  // int8 GEMM schedule
  __half *x_perm, *h;  // fp16 path rows
  int32_t *x_exp, *h_exp, *ovf_flag;  // fp16 path: per-row exponents and h overflow flags
  uint32_t* ovf_mask;                 // fp16 path: [P, I/32] h overflow marks
  Planes xq, hq;       // int8 path rows
  float* y;
  size_t bytes;
};
FwdWs carve_w4_forward(void* ws, int T, int H, int I, int E, int k) {
  Carver c(ws);
  FwdWs w{};
  const size_t P = (size_t)T * k;
  w.counts = c.take<int32_t>(E);
  w.offsets = c.take<int32_t>(E + 1);
  w.sorted = c.take<int32_t>(P);
  w.inv = c.take<int32_t>(P);
  w.blockcnt = c.take<int32_t>((size_t)align_blocks(T, k) * E);
  w.thin_tile_prefix = c.take<int32_t>(E + 1);
  w.thin_chunk = c.take<int32_t>(E);
  w.xq = take_planes(c, P, H);
  w.hq = take_planes(c, P, I);
  if (!use_i8(T)) {  // some experts may have more than kThinRows rows
    w.tile_prefix = c.take<int32_t>(E + 1);
    w.chunk = c.take<int32_t>(E);
    w.row_count = c.take<int32_t>(E);
    w.thin_row_count = c.take<int32_t>(E);
    w.thin_row_prefix = c.take<int32_t>(E + 1);
    w.x_perm = c.take<__half>(P * H);
    w.h = c.take<__half>(P * I);
    w.x_exp = c.take<int32_t>(P);
    w.h_exp = c.take<int32_t>(P);
    w.ovf_flag = c.take<int32_t>(P);
    w.ovf_mask = c.take<uint32_t>(P * (I / 32));
  }
  w.y = c.take<float>(P * H);
  w.bytes = c.off + 256;
  return w;
}
// K splits of the single grouped GEMM: when even the fewest work items the shape can have (all
// M rows in one expert) leave most of the 148 SMs of a B200 idle, each item's K range is split
// so that items x splits ~ 148 (at least one 256-K stage per split, at most 32 splits); a
// shape-only rule, so the workspace size needs no device.
int gemm_splits(int M, int K, int N) {
  const int tile_rows = use_i8(M) ? kI8TileRows : kWideTileRows;
  const int weight_rows = 128 * (use_i8(M) ? w4i8_tiles_per_item(false, N) : w4a16_tiles_per_item(N));  // per item
  const int nkb = (K + 255) / 256;
  const int items = (N / weight_rows) * ((M + tile_rows - 1) / tile_rows);
  int s = 148 / (items > 0 ? items : 1);
  if (s > nkb) s = nkb;
  if (s > 32) s = 32;
  return s < 1 ? 1 : s;
}

struct GemmWs {
  int32_t *row_count, *tile_prefix, *chunk;
  __half* a;       // fp16 path
  int32_t* a_exp;  // fp16 path: per-row exponents
  Planes aq;       // int8 path
  float* part;  // with K splits: [splits, M, N] fp32 partial sums
  size_t bytes;
};
GemmWs carve_gemm(void* ws, int M, int K, int N, int E) {
  Carver c(ws);
  GemmWs w{};
  w.row_count = c.take<int32_t>(E);
  w.tile_prefix = c.take<int32_t>(E + 1);
  w.chunk = c.take<int32_t>(E);
  if (use_i8(M)) {
    w.aq = take_planes(c, M, K);
  } else {
    w.a = c.take<__half>((size_t)M * K);
    w.a_exp = c.take<int32_t>(M);
  }
  const int sp = gemm_splits(M, K, N);
  if (sp > 1) w.part = c.take<float>((size_t)sp * M * N);
  w.bytes = c.off + 256;
  return w;
}
struct F8Ws {
  int32_t *counts, *offsets, *sorted, *inv, *blockcnt, *tile_prefix, *chunk;
  uint8_t *x_perm, *h;
  float *xs_t, *hs_t, *y;
  size_t bytes;
};
F8Ws carve_fp8_forward(void* ws, int T, int H, int I, int E, int k) {
  Carver c(ws);
  F8Ws w;
  const size_t P = (size_t)T * k;
  w.counts = c.take<int32_t>(E);
  w.offsets = c.take<int32_t>(E + 1);
  w.sorted = c.take<int32_t>(P);
  w.inv = c.take<int32_t>(P);
  w.blockcnt = c.take<int32_t>((size_t)align_blocks(T, k) * E);
  w.tile_prefix = c.take<int32_t>(E + 1);
  w.chunk = c.take<int32_t>(E);
  w.x_perm = c.take<uint8_t>(P * H);
  w.xs_t = c.take<float>((size_t)(H / 128) * P);
  w.h = c.take<uint8_t>(P * I);
  w.hs_t = c.take<float>((size_t)(I / 128) * P);
  w.y = c.take<float>(P * H);
  w.bytes = c.off + 256;
  return w;
}
struct MxWs {
  int32_t *counts, *offsets, *sorted, *inv, *blockcnt, *tile_prefix, *chunk;
  uint8_t *x_perm, *h;
  uint32_t *x_sf, *h_sf;
  float* y;
  size_t bytes;
};
MxWs carve_w4a8_forward(void* ws, int T, int H, int I, int E, int k) {
  Carver c(ws);
  MxWs w;
  const size_t P = (size_t)T * k;
  w.counts = c.take<int32_t>(E);
  w.offsets = c.take<int32_t>(E + 1);
  w.sorted = c.take<int32_t>(P);
  w.inv = c.take<int32_t>(P);
  w.blockcnt = c.take<int32_t>((size_t)align_blocks(T, k) * E);
  w.tile_prefix = c.take<int32_t>(E + 1);
  w.chunk = c.take<int32_t>(E);
  w.x_perm = c.take<uint8_t>(P * H);
  w.x_sf = c.take<uint32_t>((size_t)(H / 128) * P);
  w.h = c.take<uint8_t>(P * I);
  w.h_sf = c.take<uint32_t>((size_t)(I / 128) * P);
  w.y = c.take<float>(P * H);
  w.bytes = c.off + 256;
  return w;
}
// token-tile height cap of the single grouped GEMM's kernel
int pick_nmax(int max_rows_per_expert) { return use_i8(max_rows_per_expert) ? kI8TileRows : kWideTileRows; }

bool shape_ok(int T, int H, int I, int E, int k) {
  if (T < 1 || k < 1 || E < k || E > 1024) return false;
  if (H < 128 || I < 128 || H % 128 || I % 128) return false;
  if ((int64_t)T * k >= (1ll << 31) || (int64_t)E * 2 * I >= (1ll << 31) || (int64_t)E * H >= (1ll << 31)) return false;
  return true;
}
}  // namespace

}  // namespace moe

using namespace moe;

// ================================================================== C ABI
extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
  }
  return "MOE_ERR_UNKNOWN";
}

moe_status_t moe_route(const float* logits, int T, int E, int k, int renormalize, int32_t* topk_ids, float* topk_w,
                       cudaStream_t stream) {
  if (T < 1 || k < 1 || E < k || E > 1024) return MOE_ERR_UNSUPPORTED;
  if (!aligned(logits, 4) || !aligned(topk_ids, 4) || !aligned(topk_w, 4)) return MOE_ERR_INVALID_ARG;
  if (moe_status_t st = check_device()) return st;
  return launch_route(logits, T, E, k, renormalize, topk_ids, topk_w, stream) == cudaSuccess ? MOE_OK
                                                                                               : MOE_ERR_CUDA;
}

size_t moe_align_capacity(int T, int k, int E, int align) {
  if (T < 1 || k < 1 || E < 1 || align < 1) return 0;
  return (size_t)T * k + (size_t)E * (align - 1);
}

size_t moe_align_workspace_size(int T, int k, int E) {
  if (T < 1 || k < 1 || E < 1) return 0;
  return (size_t)align_blocks(T, k) * E * sizeof(int32_t) + 256;
}

moe_status_t moe_align(const int32_t* topk_ids, int T, int k, int E, int align, int32_t* expert_counts,
                       int32_t* expert_offsets, int32_t* sorted_ids, int32_t* inv_pos, void* ws, size_t ws_bytes,
                       cudaStream_t stream) {
  if (T < 1 || k < 1 || E < 1 || E > 1024 || align < 1 || (int64_t)T * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)moe_align_capacity(T, k, E, align) >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(topk_ids, 4) || !aligned(expert_counts, 4) || !aligned(expert_offsets, 4) || !aligned(sorted_ids, 4) ||
      !aligned(inv_pos, 4) || !aligned(ws, 16))
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_align_workspace_size(T, k, E)) return MOE_ERR_WORKSPACE;
  if (moe_status_t st = check_device()) return st;
  const cudaError_t e = launch_align(topk_ids, T, k, E, align, expert_counts, expert_offsets, sorted_ids, inv_pos,
                                     static_cast<int32_t*>(ws), nullptr, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

size_t moe_w4a16_workspace_size(int T, int H, int I, int E, int k) {
  if (!shape_ok(T, H, I, E, k)) return 0;
  return carve_w4_forward(nullptr, T, H, I, E, k).bytes;
}

moe_status_t moe_w4a16_forward(const moe_w4a16_args* a, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!a) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(a->T, a->H, a->I, a->E, a->k)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(a->x, 16) || !aligned(a->topk_ids, 4) || !aligned(a->topk_w, 4) || !aligned(a->w13_q, 16) ||
      !aligned(a->w13_s, 16) || !aligned(a->w2_q, 16) || !aligned(a->w2_s, 16) || !aligned(a->out, 16) ||
      !aligned(ws, 256))
    return MOE_ERR_INVALID_ARG;
  const int T = a->T, H = a->H, I = a->I, E = a->E, k = a->k;
  if (ws_bytes < moe_w4a16_workspace_size(T, H, I, E, k)) return MOE_ERR_WORKSPACE;
  if (moe_status_t st = check_device()) return st;
  const FwdWs w = carve_w4_forward(ws, T, H, I, E, k);
  const int P = T * k;
  const bool mixed = !use_i8(T);  // per-expert choice between the two GEMMs
  SchedOut so;
  if (mixed) {
    so.nmax = kWideTileRows;
    so.tile_prefix = w.tile_prefix;
    so.chunk = w.chunk;
    so.row_count = w.row_count;
    so.thin_rows = kThinRows;
    so.thin_nmax = kI8TileRows;
    so.thin_tile_prefix = w.thin_tile_prefix;
    so.thin_chunk = w.thin_chunk;
    so.thin_row_count = w.thin_row_count;
    so.thin_row_prefix = w.thin_row_prefix;
  } else {  // every expert on the int8 GEMM: its schedule is the main one, row counts = counts
    so.nmax = kI8TileRows;
    so.tile_prefix = w.thin_tile_prefix;
    so.chunk = w.thin_chunk;
  }
  const uint16_t* x = static_cast<const uint16_t*>(a->x);
  const uint16_t* w13_s = static_cast<const uint16_t*>(a->w13_s);
  const uint16_t* w2_s = static_cast<const uint16_t*>(a->w2_s);
  cudaError_t e = cudaSuccess;
  if (!mixed && fused_align_planes_ok(T, k, E)) {
    // a decode-sized batch: alignment, schedule and planes in one launch
    e = launch_align_planes(a->topk_ids, T, k, E, x, H, w.counts, w.offsets, w.sorted, w.inv, so.tile_prefix,
                            so.chunk, so.nmax, w.xq.x, w.xq.meta, stream);
  } else {
    e = launch_align(a->topk_ids, T, k, E, 1, w.counts, w.offsets, w.sorted, w.inv, w.blockcnt, &so, stream);
    // activations of each class of experts in the form its GEMM reads
    if (e == cudaSuccess) {
      if (mixed)  // the rows of the thin experts only: at most kThinRows per expert
        e = launch_planes_list(x, w.thin_row_prefix, w.offsets, w.sorted, E, k, std::min(P, kThinRows * E), H,
                               w.xq.x, w.xq.meta, stream);
      else
        e = launch_planes(x, 1, w.inv, P, k, H, w.xq.x, w.xq.meta, stream);
    }
  }
  const TileSched thin{w.offsets, mixed ? w.thin_row_count : w.counts, w.thin_tile_prefix, w.thin_chunk};
  const TileSched wide{w.offsets, w.row_count, w.tile_prefix, w.chunk};
  if (e == cudaSuccess && mixed)
    e = launch_permute_w4(x, w.inv, a->topk_ids, w.row_count, T, k, H, w.x_perm, w.x_exp, w.ovf_flag, w.ovf_mask, I,
                          stream);
  // gate/up with SiLU*up, then down, each on both GEMMs (an empty schedule makes a kernel exit)
  if (e == cudaSuccess) {
    W4I8Problem g{a->w13_q, w13_s, w.xq.x, w.xq.meta, P, H, E, 2 * I, true, I, thin, OUT_PLANES, w.hq.x, w.hq.meta, I};
    e = launch_w4i8_gemm(g, stream);
  }
  if (e == cudaSuccess && mixed) {
    W4GemmProblem g{a->w13_q, w13_s, w.x_perm, P, H, E, 2 * I, true, I, wide, kWideTileRows, w.h, I,
                    OUT_H_F16_INTERLEAVED};
    g.acc_exp = w.x_exp;
    g.ovf_flag = w.ovf_flag;
    g.ovf_mask = w.ovf_mask;
    e = launch_w4a16_gemm(g, stream);
  }
  // rows with an h beyond fp16 (rare) are brought to one power-of-two scale before the down GEMM
  if (e == cudaSuccess && mixed) e = launch_h_rescale(w.h, P, I, w.ovf_flag, w.ovf_mask, w.h_exp, stream);
  if (e == cudaSuccess) {
    W4I8Problem g{a->w2_q, w2_s, w.hq.x, w.hq.meta, P, I, E, H, false, 0, thin, OUT_F32, w.y, nullptr, H};
    e = launch_w4i8_gemm(g, stream);
  }
  if (e == cudaSuccess && mixed) {
    W4GemmProblem g{a->w2_q, w2_s, w.h, P, I, E, H, false, 0, wide, kWideTileRows, w.y, H, OUT_F32};
    g.acc_exp = w.h_exp;
    e = launch_w4a16_gemm(g, stream);
  }
  if (e == cudaSuccess) e = launch_combine(w.y, w.inv, a->topk_w, T, k, H, a->out, a->out_fp32, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

size_t moe_blockfp8_workspace_size(int T, int H, int I, int E, int k) {
  if (!shape_ok(T, H, I, E, k)) return 0;
  return carve_fp8_forward(nullptr, T, H, I, E, k).bytes;
}

moe_status_t moe_blockfp8_forward(const moe_blockfp8_args* a, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!a) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(a->T, a->H, a->I, a->E, a->k)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(a->x, 16) || !aligned(a->xs, 4) || !aligned(a->topk_ids, 4) || !aligned(a->topk_w, 4) ||
      !aligned(a->w13, 16) || !aligned(a->w13_s, 4) || !aligned(a->w2, 16) || !aligned(a->w2_s, 4) ||
      !aligned(a->out, 16) || !aligned(ws, 256))
    return MOE_ERR_INVALID_ARG;
  const int T = a->T, H = a->H, I = a->I, E = a->E, k = a->k;
  if (ws_bytes < moe_blockfp8_workspace_size(T, H, I, E, k)) return MOE_ERR_WORKSPACE;
  if (moe_status_t st = check_device()) return st;
  const F8Ws w = carve_fp8_forward(ws, T, H, I, E, k);
  const int P = T * k;
  // token tile of the FP8 GEMM: 64 rows once experts can get that many tokens (halves the
  // weight re-reads and doubles the tokens per MMA), else 32 (a deeper copy pipeline)
  const int nmax = T > 512 ? 64 : 32;
  SchedOut so;
  so.nmax = nmax;
  so.tile_prefix = w.tile_prefix;
  so.chunk = w.chunk;
  cudaError_t e = launch_align(a->topk_ids, T, k, E, 1, w.counts, w.offsets, w.sorted, w.inv, w.blockcnt, &so, stream);
  if (e == cudaSuccess) e = launch_permute_fp8(a->x, a->xs, w.inv, T, k, H, w.x_perm, w.xs_t, P, stream);
  const TileSched sched{w.offsets, w.counts, w.tile_prefix, w.chunk};
  if (e == cudaSuccess) {
    F8GemmProblem g{a->w13, a->w13_s, w.x_perm, w.xs_t, P, H, E, 2 * I, true, I, sched, w.h, I, w.hs_t, nmax};
    e = launch_fp8_gemm(g, stream);
  }
  if (e == cudaSuccess) {
    F8GemmProblem g{a->w2, a->w2_s, w.h, w.hs_t, P, I, E, H, false, 0, sched, w.y, H, nullptr, nmax};
    e = launch_fp8_gemm(g, stream);
  }
  if (e == cudaSuccess) e = launch_combine(w.y, w.inv, a->topk_w, T, k, H, a->out, a->out_fp32, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

size_t moe_w4a8_workspace_size(int T, int H, int I, int E, int k) {
  if (!shape_ok(T, H, I, E, k)) return 0;
  return carve_w4a8_forward(nullptr, T, H, I, E, k).bytes;
}

moe_status_t moe_w4a8_forward(const moe_w4a8_args* a, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!a) return MOE_ERR_INVALID_ARG;
  if (!shape_ok(a->T, a->H, a->I, a->E, a->k)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(a->x, 16) || !aligned(a->topk_ids, 4) || !aligned(a->topk_w, 4) || !aligned(a->w13, 32) ||
      !aligned(a->w13_sf, 16) || !aligned(a->w2, 32) || !aligned(a->w2_sf, 16) || !aligned(a->out, 16) ||
      !aligned(ws, 256))
    return MOE_ERR_INVALID_ARG;
  const int T = a->T, H = a->H, I = a->I, E = a->E, k = a->k;
  if (ws_bytes < moe_w4a8_workspace_size(T, H, I, E, k)) return MOE_ERR_WORKSPACE;
  if (moe_status_t st = check_device()) return st;
  const MxWs w = carve_w4a8_forward(ws, T, H, I, E, k);
  const int P = T * k;
  // token tile of the W4A8 GEMM: 112 rows once experts get that many tokens - two accumulator
  // tiles of 2 x 112 columns and four stages' scale blocks fill the 512 TMEM columns; each
  // MMA's shared-memory operand bytes per flop fall with the tile's width (measured at T = 8192:
  // 64 rows 6550 us, 96 rows 5890, 112 rows 5380-5480) - else 32 (16 measured the same at T = 64)
  const int nmax = T > 512 ? 112 : 32;
  SchedOut so;
  so.nmax = nmax;
  so.tile_prefix = w.tile_prefix;
  so.chunk = w.chunk;
  cudaError_t e = launch_align(a->topk_ids, T, k, E, 1, w.counts, w.offsets, w.sorted, w.inv, w.blockcnt, &so, stream);
  if (e == cudaSuccess)
    e = launch_permute_mx(reinterpret_cast<const uint16_t*>(a->x), w.inv, T, k, H, w.x_perm, w.x_sf, P, stream);
  const TileSched sched{w.offsets, w.counts, w.tile_prefix, w.chunk};
  if (e == cudaSuccess) {
    MxGemmProblem g{a->w13, a->w13_sf, w.x_perm, w.x_sf, P, H, E, 2 * I, true, I, sched,
                    w.h, I, reinterpret_cast<uint8_t*>(w.h_sf), nmax};
    e = launch_mx_gemm(g, stream);
  }
  if (e == cudaSuccess) {
    MxGemmProblem g{a->w2, a->w2_sf, w.h, w.h_sf, P, I, E, H, false, 0, sched, w.y, H, nullptr, nmax};
    e = launch_mx_gemm(g, stream);
  }
  if (e == cudaSuccess) e = launch_combine(w.y, w.inv, a->topk_w, T, k, H, a->out, a->out_fp32, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_w4a8_intermediate(const void* ws, int T, int H, int I, int E, int k, const int32_t** inv_pos,
                                   const uint8_t** h, const uint8_t** h_sf) {
  if (!shape_ok(T, H, I, E, k)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(ws, 256) || !inv_pos || !h || !h_sf) return MOE_ERR_INVALID_ARG;
  const MxWs w = carve_w4a8_forward(const_cast<void*>(ws), T, H, I, E, k);
  *inv_pos = w.inv;
  *h = w.h;
  *h_sf = reinterpret_cast<const uint8_t*>(w.h_sf);
  return MOE_OK;
}

moe_status_t moe_blockfp8_intermediate(const void* ws, int T, int H, int I, int E, int k, const int32_t** inv_pos,
                                       const uint8_t** h, const float** h_scale_t) {
  if (!shape_ok(T, H, I, E, k)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(ws, 256) || !inv_pos || !h || !h_scale_t) return MOE_ERR_INVALID_ARG;
  const F8Ws w = carve_fp8_forward(const_cast<void*>(ws), T, H, I, E, k);
  *inv_pos = w.inv;
  *h = w.h;
  *h_scale_t = w.hs_t;
  return MOE_OK;
}

size_t moe_w4a16_gemm_workspace_size(int M, int K, int N, int E) {
  if (M < 1 || K < 128 || N < 128 || K % 128 || N % 128 || E < 1 || E > 1024) return 0;
  return carve_gemm(nullptr, M, K, N, E).bytes;
}

moe_status_t moe_w4a16_gemm(const void* a, int a_is_bf16, const int32_t* w_q, const void* w_s,
                            const int32_t* expert_offsets, int M, int K, int N, int E, void* out, int out_fp32,
                            void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (M < 1 || K < 128 || N < 128 || K % 128 || N % 128 || E < 1 || E > 1024) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)E * N >= (1ll << 31) || (int64_t)M * K >= (1ll << 40)) return MOE_ERR_UNSUPPORTED;
  if (!aligned(a, 16) || !aligned(w_q, 16) || !aligned(w_s, 16) || !aligned(expert_offsets, 4) || !aligned(out, 16) ||
      !aligned(ws, 256))
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_w4a16_gemm_workspace_size(M, K, N, E)) return MOE_ERR_WORKSPACE;
  if (moe_status_t st = check_device()) return st;
  const GemmWs w = carve_gemm(ws, M, K, N, E);
  const int nmax = pick_nmax(M);
  const TileSched sched{expert_offsets, w.row_count, w.tile_prefix, w.chunk};
  if (use_i8(M)) {
    cudaError_t e = launch_sched_planes(expert_offsets, E, nmax, w.row_count, w.tile_prefix, w.chunk,
                                        static_cast<const uint16_t*>(a), a_is_bf16, M, K, w.aq.x, w.aq.meta, stream);
    const int sp = gemm_splits(M, K, N);
    if (e == cudaSuccess) {
      W4I8Problem g{w_q, static_cast<const uint16_t*>(w_s), w.aq.x, w.aq.meta, M, K, E, N, false, 0, sched,
                    out_fp32 ? OUT_F32 : OUT_BF16, out, nullptr, N, sp, w.part};
      e = launch_w4i8_gemm(g, stream);
    }
    if (e == cudaSuccess && sp > 1) e = launch_reduce_splits(w.part, sp, M, N, expert_offsets, w.row_count, E, out, out_fp32, stream);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  cudaError_t e = launch_sched_from_offsets(expert_offsets, E, M, nmax, w.row_count, w.tile_prefix, w.chunk, stream);
  if (e == cudaSuccess)
    e = launch_convert_rows(static_cast<const uint16_t*>(a), a_is_bf16, M, K, w.a, w.a_exp, stream);
  const int sp = gemm_splits(M, K, N);
  if (e == cudaSuccess) {
    W4GemmProblem g{w_q, static_cast<const uint16_t*>(w_s), w.a, M, K, E, N, false, 0, sched, nmax, out, N,
                    out_fp32 ? OUT_F32 : OUT_BF16, sp, w.part};
    g.acc_exp = w.a_exp;
    e = launch_w4a16_gemm(g, stream);
  }
  if (e == cudaSuccess && sp > 1) e = launch_reduce_splits(w.part, sp, M, N, expert_offsets, w.row_count, E, out, out_fp32, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_get_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return static_cast<moe_status_t>(v);
}

moe_status_t moe_timing_enable(int enable) {
  g_timing_on = enable != 0;
  return MOE_OK;
}

int moe_timing_read(const char** names, double* ms, int* launches, int max) {
  cudaDeviceSynchronize();
  for (const Rec& r : g_recs) {
    float t = 0.f;
    cudaEventElapsedTime(&t, r.a, r.b);
    auto it = std::find_if(g_agg.begin(), g_agg.end(), [&](const Agg& a) { return std::strcmp(a.name, r.name) == 0; });
    if (it == g_agg.end()) {
      g_agg.push_back(Agg{r.name, 0.0, 0});
      it = g_agg.end() - 1;
    }
    it->ms += t;
    it->n += 1;
    g_free_ev.push_back(r.a);
    g_free_ev.push_back(r.b);
  }
  g_recs.clear();
  const int n = (int)g_agg.size();
  for (int i = 0; i < n && i < max; ++i) {
    if (names) names[i] = g_agg[i].name;
    if (ms) ms[i] = g_agg[i].ms;
    if (launches) launches[i] = g_agg[i].n;
  }
  g_agg.clear();
  return n;
}

}  // extern "C"

// ------------------------------------------------------------------ debug: a wait that must time out
namespace moe {
__global__ void debug_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns);  // nothing ever arrives
}
}  // namespace moe

extern "C" moe_status_t moe_debug_wait_timeout(int64_t limit_ns, cudaStream_t stream) {
  if (limit_ns < 1 || limit_ns > 1000000000ll) return MOE_ERR_INVALID_ARG;
  if (moe_status_t st = check_device()) return st;
  moe::debug_wait_kernel<<<1, 32, 0, stream>>>((uint64_t)limit_ns);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
