// a4 permute (x rows -> expert-sorted fp16 rows) and a8 combine (weighted sum of each token's
// k expert outputs, in slot order, fp32).
//
// Activation rows that feed the W4A16 tensor-core GEMMs are stored in fp16 with the K index
// interleaved inside every group of 8: position (0..7) holds K offset (0,4,1,5,2,6,3,7).
// That is the order in which one packed INT4 word dequantizes with two-nibbles-per-lane
// bit tricks, so the GEMM never has to shuffle weights; applying the same permutation to
// both operands of a dot product leaves it unchanged.
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ uint4 f16x8_interleave(uint4 v) {
  // halves: v.x=(k0,k1) v.y=(k2,k3) v.z=(k4,k5) v.w=(k6,k7)
  const uint32_t a = __byte_perm(v.x, v.z, 0x5410);  // (k0,k4)
  const uint32_t b = __byte_perm(v.x, v.z, 0x7632);  // (k1,k5)
  const uint32_t c = __byte_perm(v.y, v.w, 0x5410);  // (k2,k6)
  const uint32_t d = __byte_perm(v.y, v.w, 0x7632);  // (k3,k7)
  return make_uint4(a, b, c, d);
}

// 2^e as a float for an exponent e in [-126, 127]
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// The smallest c >= 0 with amax * 2^-c <= 65504 (the largest finite fp16): scaling a row by
// 2^-c is exact and fits it into the fp16 operand of the tensor cores.
__device__ __forceinline__ int fit_exp(float amax) {
  if (!(amax > 65504.0f) || !(amax <= 3.402823466e38f)) return 0;  // fits, or not finite (flagged)
  int c = (__float_as_int(amax) >> 23) - 126 - 16;                   // amax < 2^(c + 16)
  if (c < 0) c = 0;
  if (amax * exp2i(-c) > 65504.0f) ++c;
  return c;
}

// largest magnitude field (bits & 0x7FFF) of 8 packed 16-bit floats: for bf16 and fp16 alike the
// field orders finite magnitudes, and infinities and NaNs compare above all of them
__device__ __forceinline__ uint32_t mag16x8_max(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) m = max(m, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
  return m;
}
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// 8 bf16 (k0..k7 in order) times 2^-c -> 8 fp16 in the interleaved order
__device__ __forceinline__ uint4 bf16x8_scaled_to_f16x8_interleaved(uint4 v, float sc) {
  const float f0 = bf16lo(v.x) * sc, f1 = bf16hi(v.x) * sc, f2 = bf16lo(v.y) * sc, f3 = bf16hi(v.y) * sc;
  const float f4 = bf16lo(v.z) * sc, f5 = bf16hi(v.z) * sc, f6 = bf16lo(v.w) * sc, f7 = bf16hi(v.w) * sc;
  return make_uint4(pack_h2(f0, f4), pack_h2(f1, f5), pack_h2(f2, f6), pack_h2(f3, f7));
}

// One warp per (token, slot) pair p placed at row r = inv_pos[p]: clears the row's overflow flag
// (both classes of experts), then, for a pair whose expert runs on the fp16 GEMM, scans the token's
// bf16 row for its largest magnitude, picks the row exponent c (0 unless a value is beyond fp16)
// and writes x_perm[r] = interleave(fp16(x * 2^-c)), x_exp[r] = c, and clears the row's overflow
// mask.  A non-finite input is recorded as MOE_ERR_DEVICE_CHECK.  The second pass over the row
// reads it again from L1.
__global__ void __launch_bounds__(256) permute_w4_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ inv_pos,
                                                         const int32_t* __restrict__ ids,
                                                         const int32_t* __restrict__ cls_rows, int P, int k, int H8,
                                                         uint4* __restrict__ x_perm, int32_t* __restrict__ x_exp,
                                                         int32_t* __restrict__ ovf_flag, uint32_t* __restrict__ ovf_mask,
                                                         int mask_words) {
  grid_dependency_sync();  // see common.cuh
  const int p = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (p >= P) return;
  const int r = inv_pos[p];
  if (r < 0) return;  // an out-of-range id (inv_pos -1): then ids[p] is not read
  if (lane == 0 && ovf_flag) ovf_flag[r] = 0;
  if (cls_rows && __ldg(cls_rows + __ldg(ids + p)) == 0) return;  // the expert runs on the other GEMM
  const uint4* src = x + (size_t)(p / k) * H8;
  uint4* dst = x_perm + (size_t)r * H8;
  uint32_t m = 0;
  for (int c = lane; c < H8; c += 32) m = max(m, mag16x8_max(__ldg(src + c)));
  m = warp_max_u32(m);
  const float amax = __uint_as_float(m << 16);
  if (lane == 0 && !(amax <= 3.402823466e38f)) set_status(MOE_ERR_DEVICE_CHECK);
  const int e = fit_exp(amax);
  const float sc = exp2i(-e);
  for (int c = lane; c < H8; c += 32) dst[c] = bf16x8_scaled_to_f16x8_interleaved(__ldg(src + c), sc);
  if (lane == 0) x_exp[r] = e;
  if (ovf_mask)
    for (int w = lane; w < mask_words; w += 32) ovf_mask[(size_t)r * mask_words + w] = 0;
}

cudaError_t launch_permute_w4(const uint16_t* x_bf16, const int32_t* inv_pos, const int32_t* ids,
                              const int32_t* cls_rows, int T, int k, int H, __half* x_perm, int32_t* x_exp,
                              int32_t* ovf_flag, uint32_t* ovf_mask, int I, cudaStream_t s) {
  const int P = T * k;
  timing_before("permute", s);
  (void)launch_kernel(permute_w4_kernel, dim3(ceil_div(P, 8)), dim3(256), 0, s, reinterpret_cast<const uint4*>(x_bf16), inv_pos, ids, cls_rows, P,
                                                  k, H / 8, reinterpret_cast<uint4*>(x_perm), x_exp, ovf_flag, ovf_mask,
                                                  I / 32);
  timing_after("permute", s);
  return cudaGetLastError();
}

// One warp per row r of the gated GEMM's h [rows, I] (fp16, interleaved positions): a row with
// its overflow flag set holds some values stored as h * 2^-16, marked in its mask by position.
// The row is brought to one scale: c >= 1 the smallest exponent that fits max|h| into fp16, every
// value rewritten as fp16(h * 2^-c) (exact power-of-two rescaling of the stored values), and
// h_exp[r] = c for the down GEMM, which multiplies the row's accumulators by 2^c.  Other rows
// get h_exp[r] = 0 and are not touched.
__global__ void __launch_bounds__(256) h_rescale_kernel(uint4* __restrict__ h, int rows, int I8,
                                                        const int32_t* __restrict__ ovf_flag,
                                                        const uint32_t* __restrict__ ovf_mask,
                                                        int32_t* __restrict__ h_exp) {
  grid_dependency_sync();  // see common.cuh
  const int lane = threadIdx.x & 31;
  const int mask_words = I8 / 4;
  for (int r = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5); r < rows;
       r += (int)((gridDim.x * blockDim.x) >> 5)) {
    if (__ldg(ovf_flag + r) == 0) {
      if (lane == 0) h_exp[r] = 0;
      continue;
    }
    uint4* row = h + (size_t)r * I8;
    const uint32_t* mrow = ovf_mask + (size_t)r * mask_words;
    float amax = 0.f;
    for (int c = lane; c < I8; c += 32) {  // chunk c = stored positions 8c .. 8c+7
      const uint4 v = row[c];
      const uint32_t bits = (__ldg(mrow + c / 4) >> (8 * (c & 3))) & 0xFFu;
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 hh = *reinterpret_cast<const __half2*>(&w[j]);
        amax = fmaxf(amax, fabsf(__low2float(hh)) * ((bits >> (2 * j)) & 1 ? 65536.0f : 1.0f));
        amax = fmaxf(amax, fabsf(__high2float(hh)) * ((bits >> (2 * j + 1)) & 1 ? 65536.0f : 1.0f));
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    int e = fit_exp(amax);
    if (e < 1) e = 1;
    const float s_plain = exp2i(-e), s_marked = exp2i(16 - e);
    for (int c = lane; c < I8; c += 32) {
      const uint4 v = row[c];
      const uint32_t bits = (__ldg(mrow + c / 4) >> (8 * (c & 3))) & 0xFFu;
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 hh = *reinterpret_cast<const __half2*>(&w[j]);
        const float lo = __low2float(hh) * ((bits >> (2 * j)) & 1 ? s_marked : s_plain);
        const float hi = __high2float(hh) * ((bits >> (2 * j + 1)) & 1 ? s_marked : s_plain);
        w[j] = pack_h2(lo, hi);
      }
      row[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (lane == 0) h_exp[r] = e;
  }
}

cudaError_t launch_h_rescale(__half* h, int rows, int I, const int32_t* ovf_flag, const uint32_t* ovf_mask,
                             int32_t* h_exp, cudaStream_t s) {
  const size_t want = ((size_t)rows + 7) / 8;
  const unsigned blocks = (unsigned)std::min<size_t>(want, (size_t)sm_count() * 16);
  timing_before("h_rescale", s);
  (void)launch_kernel(h_rescale_kernel, dim3(blocks), dim3(256), 0, s, reinterpret_cast<uint4*>(h), rows, I / 8, ovf_flag, ovf_mask, h_exp);
  timing_after("h_rescale", s);
  return cudaGetLastError();
}

// one warp per (token, slot) pair: x_perm[r] = x[p / k] (e4m3 bytes), xs_t[g][r] = xs[p / k][g]
__global__ void __launch_bounds__(256) permute_fp8_kernel(const uint4* __restrict__ x, const float* __restrict__ xs,
                                                          const int32_t* __restrict__ inv_pos, int Pn, int k, int H,
                                                          uint4* __restrict__ x_perm, float* __restrict__ xs_t,
                                                          int P) {
  grid_dependency_sync();  // see common.cuh
  const int p = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (p >= Pn) return;
  const int r = inv_pos[p];
  if (r < 0) return;
  const int t = p / k;
  const uint4* src = x + (size_t)t * (H / 16);
  uint4* dst = x_perm + (size_t)r * (H / 16);
  for (int c = lane; c < H / 16; c += 32) dst[c] = __ldg(src + c);
  for (int g = lane; g < H / 128; g += 32) xs_t[(size_t)g * P + r] = __ldg(xs + (size_t)t * (H / 128) + g);
}

cudaError_t launch_permute_fp8(const uint8_t* x, const float* xs, const int32_t* inv_pos, int T, int k, int H,
                               uint8_t* x_perm, float* xs_t, int P, cudaStream_t s) {
  const int Pn = T * k;
  timing_before("permute_fp8", s);
  (void)launch_kernel(permute_fp8_kernel, dim3(ceil_div(Pn, 8)), dim3(256), 0, s, reinterpret_cast<const uint4*>(x), xs, inv_pos, Pn, k, H,
                                                    reinterpret_cast<uint4*>(x_perm), xs_t, P);
  timing_after("permute_fp8", s);
  return cudaGetLastError();
}

// W4A8 input rows: bf16 x -> e4m3 codes with one E8M0 scale per 32 along K (the smallest power
// of two 2^X with amax <= 448 * 2^X; codes e4m3(x * 2^-X), nearest-even, exact scaling), written
// to each of the token's k expert-sorted rows.  One warp per (token, 128-K block), four elements
// per lane, a 32-group = 8 lanes; the block's four scale codes leave as one 32-bit word.
__global__ void __launch_bounds__(256) permute_mx_kernel(const uint2* __restrict__ x,
                                                         const int32_t* __restrict__ inv_pos, int T, int k, int H,
                                                         uint32_t* __restrict__ x_perm, uint32_t* __restrict__ x_sf,
                                                         int P) {
  grid_dependency_sync();  // see common.cuh
  const int gw = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  const int nb = H / 128;
  if (gw >= T * nb) return;
  const int t = gw / nb, b = gw - t * nb;
  const uint2 v = __ldg(x + ((size_t)t * H + b * 128) / 4 + lane);
  const float f0 = __uint_as_float(v.x << 16), f1 = __uint_as_float(v.x & 0xFFFF0000u);
  const float f2 = __uint_as_float(v.y << 16), f3 = __uint_as_float(v.y & 0xFFFF0000u);
  float a = fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3)));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
  if (!(a <= 3.402823466e38f) && (lane & 7) == 0) set_status(MOE_ERR_DEVICE_CHECK);  // an inf or NaN input
  const int X = mx_exponent(__float_as_uint(a));
  const float inv = exp2_neg(X);
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(f0 * inv, f1 * inv), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(f2 * inv, f3 * inv), __NV_SATFINITE, __NV_E4M3);
  const uint32_t codes = lo | (hi << 16);
  const uint32_t sb = (uint32_t)(X + 127);
  const uint32_t word = __shfl_sync(0xffffffffu, sb, 0) | (__shfl_sync(0xffffffffu, sb, 8) << 8) |
                        (__shfl_sync(0xffffffffu, sb, 16) << 16) | (__shfl_sync(0xffffffffu, sb, 24) << 24);
  for (int s = 0; s < k; ++s) {
    const int r = __ldg(inv_pos + (size_t)t * k + s);
    if (r < 0) continue;  // the same for the whole warp
    x_perm[((size_t)r * H + b * 128) / 4 + lane] = codes;
    if (lane == 0) x_sf[(size_t)b * P + r] = word;
  }
}

cudaError_t launch_permute_mx(const uint16_t* x, const int32_t* inv_pos, int T, int k, int H, uint8_t* x_perm,
                              uint32_t* x_sf, int P, cudaStream_t s) {
  const int warps = T * (H / 128);
  timing_before("permute_mx", s);
  (void)launch_kernel(permute_mx_kernel, dim3(ceil_div(warps, 8)), dim3(256), 0, s,
                      reinterpret_cast<const uint2*>(x), inv_pos, T, k, H, reinterpret_cast<uint32_t*>(x_perm), x_sf,
                      P);
  timing_after("permute_mx", s);
  return cudaGetLastError();
}

// 16-bit fixed-point planes of activation rows.  16 threads per (row, 128-K block), 8 K
// elements each: s = max(amax, 1e-30) / kFixMax, X = rint(x / s) = 256*hi + lo with hi =
// floor((X + 128) / 256) in [-64, 64] and lo in [-128, 127]; hi goes to plane row 2r, lo to
// 2r+1, bytes in the order (0,2,4,6,1,3,5,7) of each 8-group (the order in which a packed INT4
// word unpacks); the sum of X over every 32-K group (for the MMA's offset correction) and the
// block scales go to the row's meta words.  Called by whole warps (two units of 16 lanes); a
// lane with r < 0 takes part in the shuffles and writes nothing.
// One 128-K block of a source row, the caller's 8 elements: packed hi and lo bytes, the 32-K
// group sum of X (valid on every lane) and the block scale.
struct PlaneBits {
  uint32_t hb[2], lb[2];
  int sum;
  float sc;
};

__device__ __forceinline__ PlaneBits planes_compute(const uint4* __restrict__ a, int a_is_bf16, bool live, int src,
                                                    int blk, int i, int K) {
  float x[8];
  float amax = 0.f;
  if (live) {
    const uint4 v = __ldg(a + ((size_t)src * K + blk * 128 + 8 * i) / 8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (a_is_bf16) {
        x[2 * j] = __uint_as_float(w[j] << 16);
        x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      } else {
        const __half2 h = *reinterpret_cast<const __half2*>(&w[j]);
        x[2 * j] = __low2float(h);
        x[2 * j + 1] = __high2float(h);
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(x[j]));
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = 0.f;
  }
#pragma unroll
  for (int off = 8; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));  // 16 lanes
  if (!(amax <= 3.402823466e38f) && i == 0) set_status(MOE_ERR_DEVICE_CHECK);  // an inf or NaN input
  PlaneBits pb;
  pb.sc = fmaxf(amax, 1e-30f) * (1.0f / kFixMax);
  int X[8], sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    X[j] = __float2int_rn(__fdiv_rn(x[j], pb.sc));
    sum += X[j];
  }
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);  // 4 threads = one 32-K group
  pb.sum = sum;
  constexpr int ord[8] = {0, 2, 4, 6, 1, 3, 5, 7};
  pb.hb[0] = pb.hb[1] = pb.lb[0] = pb.lb[1] = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int v = X[ord[q]];
    const int h8 = (v + 128) >> 8;
    const int l8 = v - 256 * h8;
    pb.hb[q >> 2] |= (uint32_t)(h8 & 0xFF) << (8 * (q & 3));
    pb.lb[q >> 2] |= (uint32_t)(l8 & 0xFF) << (8 * (q & 3));
  }
  return pb;
}

__device__ __forceinline__ void planes_write(const PlaneBits& pb, int r, int blk, int i, int K,
                                             uint2* __restrict__ planes, int32_t* __restrict__ meta) {
  const size_t o = ((size_t)(2 * r) * K + blk * 128 + 8 * i) / 8;
  planes[o] = make_uint2(pb.hb[0], pb.hb[1]);
  planes[o + K / 8] = make_uint2(pb.lb[0], pb.lb[1]);
  int32_t* m = meta + (size_t)r * meta_words_per_row(K) + (blk >> 1) * kMetaWords;
  if ((i & 3) == 0) m[(blk & 1) * 4 + (i >> 2)] = kFixBias - 8 * pb.sum;
  if (i == 0) m[8 + (blk & 1)] = __float_as_int(pb.sc);
}

__device__ __forceinline__ void planes_unit(const uint4* __restrict__ a, int a_is_bf16, int r, int src, int blk,
                                            int i, int K, uint2* __restrict__ planes, int32_t* __restrict__ meta) {
  const PlaneBits pb = planes_compute(a, a_is_bf16, r >= 0, src, blk, i, K);
  if (r >= 0) planes_write(pb, r, blk, i, K, planes, meta);
}

// ------------------------------------------------------------------ alignment + planes, one launch
// For small batches (P = T*k <= kFusedMaxPairs pairs, E <= kFusedMaxExperts): every CTA computes the
// whole stable alignment in shared memory (a few microseconds for a decode batch), so no CTA waits
// for another; each CTA writes its slice of inv_pos / sorted_ids (CTA 0 also the counts, offsets
// and the int8 GEMM's tile schedule) and the fixed-point planes of its (token, 128-K block) units,
// computed once per token and written to each of the token's k rows.  The same results as
// moe_align (align = 1) followed by the planes kernel.
constexpr int kFusedThreads = 512;
constexpr int kFusedWarps = kFusedThreads / 32;
constexpr int kFusedMaxPairs = 4096;
constexpr int kFusedMaxExperts = kFusedThreads;  // one expert per thread in the block scans

__global__ void __launch_bounds__(kFusedThreads) align_planes_kernel(
    const int32_t* __restrict__ ids, int T, int k, int E, const uint4* __restrict__ x, int K,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ sorted_ids,
    int32_t* __restrict__ inv_pos, int32_t* __restrict__ tile_prefix, int32_t* __restrict__ chunk, int nmax,
    uint2* __restrict__ planes, int32_t* __restrict__ meta) {
  grid_dependency_sync();  // see common.cuh
  extern __shared__ int fsm[];
  int* wcnt = fsm;                          // [kFusedWarps][E]: a warp's count, then its base
  int* offs = wcnt + kFusedWarps * E;       // [E] first row of each expert
  int* inv_s = offs + E;                    // [P] row of each pair (-1: out-of-range id)
  __shared__ int warp_tot[32];
  __shared__ int total;
  const int P = T * k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kFusedWarps * E; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();
  // each warp takes a contiguous run of pairs, 32 at a time in order, so that ranks within an
  // expert follow the pair order (a stable sort)
  const int run = (P + kFusedWarps - 1) / kFusedWarps;
  const int q0 = warp * run, q1 = min(P, q0 + run);
  int* my = wcnt + warp * E;
  for (int b = q0; b < q1; b += 32) {
    const int p = b + lane;
    const int e = p < q1 ? ids[p] : -1;
    const bool valid = e >= 0 && e < E;
    if (p < q1 && !valid && blockIdx.x == 0) set_status(MOE_ERR_DEVICE_CHECK);
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -(lane + 2));
    if (valid && lane == __ffs(peers) - 1) my[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per expert: bases of the warps' runs, the count, then offsets and tiles by block scans
  const int e = threadIdx.x;
  int c = 0;
  if (e < E)
    for (int w = 0; w < kFusedWarps; ++w) {
      const int v = wcnt[w * E + e];
      wcnt[w * E + e] = c;
      c += v;
    }
  const int off = block_exclusive_scan(e < E ? c : 0, warp_tot, &total);
  const int n_rows = total;  // read by every thread before the next scan writes it
  int nt = 0, ch = 16;
  if (e < E) {
    offs[e] = off;
    expert_tiles(c, nmax, &nt, &ch);
  }
  const int tp = block_exclusive_scan(nt, warp_tot, &total);
  if (blockIdx.x == 0) {
    if (e < E) {
      counts[e] = c;
      offsets[e] = off;
      tile_prefix[e] = tp;
      chunk[e] = ch;
    }
    if (e == 0) {
      offsets[E] = n_rows;
      tile_prefix[E] = total;
    }
  }
  __syncthreads();
  // scatter: the same walk, now placing each pair
  for (int b = q0; b < q1; b += 32) {
    const int p = b + lane;
    const int ee = p < q1 ? ids[p] : -1;
    const bool valid = ee >= 0 && ee < E;
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? ee : -(lane + 2));
    int pos = -1;
    if (valid) pos = offs[ee] + my[ee] + __popc(peers & ((1u << lane) - 1u));
    __syncwarp();
    if (valid && lane == __ffs(peers) - 1) my[ee] += __popc(peers);
    if (p < q1) inv_s[p] = pos;
    __syncwarp();
  }
  __syncthreads();
  // this CTA's slice of the pair arrays
  const int slice = (P + gridDim.x - 1) / gridDim.x;
  for (int p = blockIdx.x * slice + threadIdx.x; p < min(P, (int)(blockIdx.x + 1) * slice); p += blockDim.x) {
    const int r = inv_s[p];
    inv_pos[p] = r;
    if (r >= 0) sorted_ids[r] = p;
  }
  // planes: units (token, 128-K block), 16 lanes each, this CTA's share of them
  const int nblk = K / 128;
  const int units = T * nblk;
  const int per = (units + gridDim.x - 1) / gridDim.x;
  const int u0 = blockIdx.x * per, u1 = min(units, u0 + per);
  const int i = threadIdx.x & 15;
  for (int ub = u0; ub < u1; ub += kFusedThreads / 16) {
    const int u = ub + (threadIdx.x >> 4);
    const bool live = u < u1;
    const int t = live ? u / nblk : 0, blk = live ? u % nblk : 0;
    const PlaneBits pb = planes_compute(x, 1, live, t, blk, i, K);
    if (live)
      for (int s = 0; s < k; ++s) {
        const int r = inv_s[t * k + s];
        if (r >= 0) planes_write(pb, r, blk, i, K, planes, meta);
      }
  }
}

bool fused_align_planes_ok(int T, int k, int E) { return (long long)T * k <= kFusedMaxPairs && E <= kFusedMaxExperts; }

cudaError_t launch_align_planes(const int32_t* ids, int T, int k, int E, const uint16_t* x_bf16, int K,
                                int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* inv_pos,
                                int32_t* tile_prefix, int32_t* chunk, int nmax, int8_t* planes, int32_t* meta,
                                cudaStream_t s) {
  const int P = T * k;
  const size_t smem = (size_t)(kFusedWarps * E + E + P) * sizeof(int);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(align_planes_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int units = T * (K / 128);
  const int grid = std::max(1, std::min(sm_count(), ceil_div(units, kFusedThreads / 16)));
  timing_before("align_planes", s);
  (void)launch_kernel(align_planes_kernel, dim3(grid), dim3(kFusedThreads), smem, s, ids, T, k, E, reinterpret_cast<const uint4*>(x_bf16), K,
                                                         counts, offsets, sorted_ids, inv_pos, tile_prefix, chunk,
                                                         nmax, reinterpret_cast<uint2*>(planes), meta);
  timing_after("align_planes", s);
  return cudaGetLastError();
}

// every pair p: plane row inv_pos[p] from source row p / k (or, without inv_pos, row p from row p)
__global__ void __launch_bounds__(256) planes_kernel(const uint4* __restrict__ a, int a_is_bf16,
                                                     const int32_t* __restrict__ inv_pos, int n_pairs, int k, int K,
                                                     uint2* __restrict__ planes, int32_t* __restrict__ meta) {
  grid_dependency_sync();  // see common.cuh
  const int nblk = K / 128;
  const size_t unit = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 4;  // (pair, block)
  const int i = threadIdx.x & 15;                                             // 8-group within the block
  const bool live = unit < (size_t)n_pairs * nblk;
  const int p = live ? (int)(unit / nblk) : 0;
  const int blk = live ? (int)(unit % nblk) : 0;
  const int r = live ? (inv_pos ? inv_pos[p] : p) : -1;
  planes_unit(a, a_is_bf16, r, p / k, blk, i, K, planes, meta);
}

cudaError_t launch_planes(const uint16_t* a, int a_is_bf16, const int32_t* inv_pos, int n_pairs, int k, int K,
                          int8_t* planes, int32_t* meta, cudaStream_t s) {
  const size_t threads = (size_t)n_pairs * (K / 128) * 16;
  timing_before("planes", s);
  (void)launch_kernel(planes_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, s, reinterpret_cast<const uint4*>(a), a_is_bf16,
                                                                  inv_pos, n_pairs, k, K,
                                                                  reinterpret_cast<uint2*>(planes), meta);
  timing_after("planes", s);
  return cudaGetLastError();
}

// The single grouped GEMM's int8 path: its tile schedule (block 0, a thread per expert) and the
// activation planes of its M rows (the other blocks, 16 threads per (row, 128-K block)) in one
// launch - the two are independent, and a launch saved is most of a small GEMM's time.
__global__ void __launch_bounds__(1024) sched_planes_kernel(const int32_t* __restrict__ offsets, int E, int nmax,
                                                            int32_t* __restrict__ row_count,
                                                            int32_t* __restrict__ tile_prefix,
                                                            int32_t* __restrict__ chunk, const uint4* __restrict__ a,
                                                            int a_is_bf16, int M, int K, uint2* __restrict__ planes,
                                                            int32_t* __restrict__ meta) {
  grid_dependency_sync();  // see common.cuh
  if (blockIdx.x == 0) {
    sched_from_offsets_block(offsets, E, M, nmax, row_count, tile_prefix, chunk);
    return;
  }
  const int nblk = K / 128;
  const size_t unit = ((blockIdx.x - 1) * (size_t)blockDim.x + threadIdx.x) >> 4;  // (row, block)
  const int i = threadIdx.x & 15;
  const bool live = unit < (size_t)M * nblk;
  const int p = live ? (int)(unit / nblk) : 0;
  const int blk = live ? (int)(unit % nblk) : 0;
  planes_unit(a, a_is_bf16, live ? p : -1, p, blk, i, K, planes, meta);
}

cudaError_t launch_sched_planes(const int32_t* offsets, int E, int nmax, int32_t* row_count, int32_t* tile_prefix,
                                int32_t* chunk, const uint16_t* a, int a_is_bf16, int M, int K, int8_t* planes,
                                int32_t* meta, cudaStream_t s) {
  const size_t threads = (size_t)M * (K / 128) * 16;
  timing_before("sched_planes", s);
  (void)launch_kernel(sched_planes_kernel, dim3(1 + (unsigned)((threads + 1023) / 1024)), dim3(1024), 0, s, offsets,
                      E, nmax, row_count, tile_prefix, chunk, reinterpret_cast<const uint4*>(a), a_is_bf16, M, K,
                      reinterpret_cast<uint2*>(planes), meta);
  timing_after("sched_planes", s);
  return cudaGetLastError();
}

// the rows of a list of expert runs: list row j < row_prefix[E] is row j - row_prefix[e] of
// expert e (row_prefix[e] <= j < row_prefix[e+1]), i.e. sorted row offsets[e] + j - row_prefix[e],
// whose pair is sorted_ids of that row; the grid covers an upper bound of the list length
__global__ void __launch_bounds__(256) planes_list_kernel(const uint4* __restrict__ a,
                                                          const int32_t* __restrict__ row_prefix,
                                                          const int32_t* __restrict__ offsets,
                                                          const int32_t* __restrict__ sorted_ids, int E, int k, int K,
                                                          uint2* __restrict__ planes, int32_t* __restrict__ meta) {
  grid_dependency_sync();  // see common.cuh
  const int nblk = K / 128;
  const size_t unit = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 4;  // (list row, block)
  const int i = threadIdx.x & 15;
  const int total = __ldg(row_prefix + E);
  const int j = (int)(unit / nblk);
  const int blk = (int)(unit % nblk);
  if (__all_sync(0xffffffffu, j >= total)) return;
  int r = -1, src = 0;
  if (j < total) {
    int lo = 0, hi = E;  // row_prefix[lo] <= j < row_prefix[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(row_prefix + mid) <= j)
        lo = mid;
      else
        hi = mid;
    }
    r = __ldg(offsets + lo) + j - __ldg(row_prefix + lo);
    src = __ldg(sorted_ids + r) / k;
  }
  planes_unit(a, 1, r, src, blk, i, K, planes, meta);
}

cudaError_t launch_planes_list(const uint16_t* x_bf16, const int32_t* row_prefix, const int32_t* offsets,
                               const int32_t* sorted_ids, int E, int k, int max_rows, int K, int8_t* planes,
                               int32_t* meta, cudaStream_t s) {
  const size_t threads = (size_t)max_rows * (K / 128) * 16;
  timing_before("planes", s);
  (void)launch_kernel(planes_list_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, s, 
      reinterpret_cast<const uint4*>(x_bf16), row_prefix, offsets, sorted_ids, E, k, K,
      reinterpret_cast<uint2*>(planes), meta);
  timing_after("planes", s);
  return cudaGetLastError();
}

// Split-K reduction: out[r][n] = sum_s part[s][r][n] in split order (deterministic).  Block row
// blockIdx.y = expert e reduces the rows [row_start[e], row_start[e] + row_count[e]); the
// scheduler sets row_count to 0 for an expert whose offsets failed its check, and the GEMM then
// wrote no partial sums for it, so such rows are left untouched (never filled from unwritten
// workspace).  One thread per 4 outputs, grid-stride over the expert's rows.
__global__ void __launch_bounds__(256) reduce_splits_kernel(const float4* __restrict__ part, int splits, int rows,
                                                            int N, const int32_t* __restrict__ row_start,
                                                            const int32_t* __restrict__ row_count,
                                                            void* __restrict__ out, int out_fp32) {
  grid_dependency_sync();  // see common.cuh
  const int e = blockIdx.y;
  const int cnt = __ldg(row_count + e);
  if (cnt <= 0) return;
  const size_t n4 = (size_t)N / 4, plane = (size_t)rows * n4;
  const size_t i0 = (size_t)__ldg(row_start + e) * n4, i1 = i0 + (size_t)cnt * n4;
  for (size_t i = i0 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < i1; i += (size_t)gridDim.x * blockDim.x) {
    float4 acc = __ldg(part + i);
    for (int sp = 1; sp < splits; ++sp) {
      const float4 v = __ldg(part + (size_t)sp * plane + i);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if (out_fp32) {
      reinterpret_cast<float4*>(out)[i] = acc;
    } else {
      __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(out) + 2 * i;
      o[0] = __floats2bfloat162_rn(acc.x, acc.y);
      o[1] = __floats2bfloat162_rn(acc.z, acc.w);
    }
  }
}

cudaError_t launch_reduce_splits(const float* part, int splits, int rows, int N, const int32_t* row_start,
                                 const int32_t* row_count, int E, void* out, int out_fp32, cudaStream_t s) {
  // about 8 blocks of 256 threads per SM in total, at least one per expert
  const size_t want = ((size_t)rows * (N / 4) + 255) / 256;
  const size_t cap = (size_t)sm_count() * 8;
  const unsigned bx = (unsigned)std::max<size_t>(1, std::min(want, cap) / (size_t)E);
  timing_before("reduce_splits", s);
  (void)launch_kernel(reduce_splits_kernel, dim3(dim3(bx, (unsigned)E)), dim3(256), 0, s, reinterpret_cast<const float4*>(part), splits, rows, N,
                                                              row_start, row_count, out, out_fp32);
  timing_after("reduce_splits", s);
  return cudaGetLastError();
}

// One warp per row of the single grouped GEMM's activations: interleaved fp16 rows
// out[r] = fp16(a[r] * 2^-x_exp[r]), x_exp[r] the smallest exponent >= 0 that fits the row into
// fp16 (always 0 for fp16 input); a non-finite input is recorded as MOE_ERR_DEVICE_CHECK.
__global__ void __launch_bounds__(256) convert_rows_kernel(const uint4* __restrict__ a, int a_is_bf16, int M, int K8,
                                                           uint4* __restrict__ out, int32_t* __restrict__ x_exp) {
  grid_dependency_sync();  // see common.cuh
  const int lane = threadIdx.x & 31;
  for (int r = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5); r < M;
       r += (int)(((size_t)gridDim.x * blockDim.x) >> 5)) {
    const uint4* src = a + (size_t)r * K8;
    uint4* dst = out + (size_t)r * K8;
    uint32_t m = 0;
    for (int c = lane; c < K8; c += 32) m = max(m, mag16x8_max(__ldg(src + c)));
    m = warp_max_u32(m);
    const bool finite = a_is_bf16 ? m < 0x7F80u : m < 0x7C00u;
    if (lane == 0 && !finite) set_status(MOE_ERR_DEVICE_CHECK);
    const int e = a_is_bf16 ? fit_exp(__uint_as_float(m << 16)) : 0;
    const float sc = exp2i(-e);
    for (int c = lane; c < K8; c += 32) {
      const uint4 v = __ldg(src + c);
      dst[c] = a_is_bf16 ? bf16x8_scaled_to_f16x8_interleaved(v, sc) : f16x8_interleave(v);
    }
    if (lane == 0) x_exp[r] = e;
  }
}

cudaError_t launch_convert_rows(const uint16_t* a, int a_is_bf16, int M, int K, __half* out, int32_t* x_exp,
                                cudaStream_t s) {
  const int blocks = (int)std::min<size_t>(((size_t)M + 7) / 8, (size_t)sm_count() * 16);
  timing_before("convert", s);
  (void)launch_kernel(convert_rows_kernel, dim3(blocks), dim3(256), 0, s, reinterpret_cast<const uint4*>(a), a_is_bf16, M, K / 8,
                                             reinterpret_cast<uint4*>(out), x_exp);
  timing_after("convert", s);
  return cudaGetLastError();
}

// out[t][c..c+3] = sum_s w[t][s] * y_perm[inv_pos[t*k+s]][c..c+3], fp32, slot order
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y, const int32_t* __restrict__ inv_pos,
                                                      const float* __restrict__ w, int T, int k, int H4,
                                                      void* __restrict__ out, int out_fp32) {
  grid_dependency_sync();  // see common.cuh
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i >= (size_t)T * H4) return;
  const int t = (int)(i / H4), c = (int)(i % H4);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < k; ++s) {
    const int r = __ldg(inv_pos + (size_t)t * k + s);
    if (r < 0) continue;
    const float ws = __ldg(w + (size_t)t * k + s);
    const float4 v = __ldg(y + (size_t)r * H4 + c);
    acc.x = fmaf(ws, v.x, acc.x);
    acc.y = fmaf(ws, v.y, acc.y);
    acc.z = fmaf(ws, v.z, acc.z);
    acc.w = fmaf(ws, v.w, acc.w);
  }
  if (out_fp32) {
    reinterpret_cast<float4*>(out)[i] = acc;
  } else {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&lo);
    u.y = *reinterpret_cast<const uint32_t*>(&hi);
    reinterpret_cast<uint2*>(out)[i] = u;
  }
}

cudaError_t launch_combine(const float* y_perm, const int32_t* inv_pos, const float* topk_w, int T, int k, int H,
                           void* out, int out_fp32, cudaStream_t s) {
  const size_t n = (size_t)T * (H / 4);
  timing_before("combine", s);
  (void)launch_kernel(combine_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, reinterpret_cast<const float4*>(y_perm), inv_pos, topk_w,
                                                              T, k, H / 4, out, out_fp32);
  timing_after("combine", s);
  return cudaGetLastError();
}

}  // namespace moe
