// a4 permute (x rows -> expert-sorted fp16 rows) and a8 combine (weighted sum of each token's
// k expert outputs, in slot order, fp32).
//
// Activation rows that feed the W4A16 tensor-core GEMMs are stored in fp16 with the K index
// interleaved inside every group of 8: position (0..7) holds K offset (0,4,1,5,2,6,3,7).
// That is the order in which one packed INT4 word dequantizes with two-nibbles-per-lane
// bit tricks, so the GEMM never has to shuffle weights; applying the same permutation to
// both operands of a dot product leaves it unchanged.
#include "common.cuh"
#include "internal.h"

namespace moe {

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// 8 bf16 (k0..k7 in order) -> 8 fp16 in the interleaved order (k0,k4,k1,k5,k2,k6,k3,k7)
__device__ __forceinline__ uint4 bf16x8_to_f16x8_interleaved(uint4 v) {
  const float f0 = bf16lo(v.x), f1 = bf16hi(v.x), f2 = bf16lo(v.y), f3 = bf16hi(v.y);
  const float f4 = bf16lo(v.z), f5 = bf16hi(v.z), f6 = bf16lo(v.w), f7 = bf16hi(v.w);
  return make_uint4(pack_h2(f0, f4), pack_h2(f1, f5), pack_h2(f2, f6), pack_h2(f3, f7));
}
__device__ __forceinline__ uint4 f16x8_interleave(uint4 v) {
  // halves: v.x=(k0,k1) v.y=(k2,k3) v.z=(k4,k5) v.w=(k6,k7)
  const uint32_t a = __byte_perm(v.x, v.z, 0x5410);  // (k0,k4)
  const uint32_t b = __byte_perm(v.x, v.z, 0x7632);  // (k1,k5)
  const uint32_t c = __byte_perm(v.y, v.w, 0x5410);  // (k2,k6)
  const uint32_t d = __byte_perm(v.y, v.w, 0x7632);  // (k3,k7)
  return make_uint4(a, b, c, d);
}

// True when one of the 8 bf16 values is outside the finite fp16 range: |x| >= 65536 (the
// smallest bf16 magnitude above 65504 the cast would turn into infinity), infinite or NaN.
__device__ __forceinline__ bool bf16x8_beyond_f16(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  bool bad = false;
#pragma unroll
  for (int j = 0; j < 4; ++j) bad |= (w[j] & 0x7FFFu) >= 0x4780u || ((w[j] >> 16) & 0x7FFFu) >= 0x4780u;
  return bad;
}
// True when one of the 8 fp16 values is infinite or NaN.
__device__ __forceinline__ bool f16x8_nonfinite(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  bool bad = false;
#pragma unroll
  for (int j = 0; j < 4; ++j) bad |= (w[j] & 0x7C00u) == 0x7C00u || (w[j] & 0x7C000000u) == 0x7C000000u;
  return bad;
}

// one warp per (token, slot) pair: x_perm[inv_pos[p]] = interleave(fp16(x[p / k])).  A row with
// a value the fp16 operand cannot hold is still converted (to +-inf) and recorded as
// MOE_ERR_DEVICE_CHECK.
__global__ void __launch_bounds__(256) permute_w4_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ inv_pos,
                                                         const int32_t* __restrict__ ids,
                                                         const int32_t* __restrict__ cls_rows, int P, int k, int H8,
                                                         uint4* __restrict__ x_perm) {
  const int p = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (p >= P) return;
  const int r = inv_pos[p];
  if (r < 0) return;  // an out-of-range id (inv_pos -1): then ids[p] is not read
  if (cls_rows && __ldg(cls_rows + __ldg(ids + p)) == 0) return;  // the expert runs on the other GEMM
  const uint4* src = x + (size_t)(p / k) * H8;
  uint4* dst = x_perm + (size_t)r * H8;
  bool bad = false;
  for (int c = lane; c < H8; c += 32) {
    const uint4 v = __ldg(src + c);
    bad |= bf16x8_beyond_f16(v);
    dst[c] = bf16x8_to_f16x8_interleaved(v);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(MOE_ERR_DEVICE_CHECK);
}

cudaError_t launch_permute_w4(const uint16_t* x_bf16, const int32_t* inv_pos, const int32_t* ids,
                              const int32_t* cls_rows, int T, int k, int H, __half* x_perm, cudaStream_t s) {
  const int P = T * k;
  timing_before("permute", s);
  permute_w4_kernel<<<ceil_div(P, 8), 256, 0, s>>>(reinterpret_cast<const uint4*>(x_bf16), inv_pos, ids, cls_rows, P,
                                                  k, H / 8, reinterpret_cast<uint4*>(x_perm));
  timing_after("permute", s);
  return cudaGetLastError();
}

// one warp per (token, slot) pair: x_perm[r] = x[p / k] (e4m3 bytes), xs_t[g][r] = xs[p / k][g]
__global__ void __launch_bounds__(256) permute_fp8_kernel(const uint4* __restrict__ x, const float* __restrict__ xs,
                                                          const int32_t* __restrict__ inv_pos, int Pn, int k, int H,
                                                          uint4* __restrict__ x_perm, float* __restrict__ xs_t,
                                                          int P) {
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
  permute_fp8_kernel<<<ceil_div(Pn, 8), 256, 0, s>>>(reinterpret_cast<const uint4*>(x), xs, inv_pos, Pn, k, H,
                                                    reinterpret_cast<uint4*>(x_perm), xs_t, P);
  timing_after("permute_fp8", s);
  return cudaGetLastError();
}

// 16-bit fixed-point planes of activation rows.  16 threads per (row, 128-K block), 8 K
// elements each: s = max(amax, 1e-30) / kFixMax, X = rint(x / s) = 256*hi + lo with hi =
// floor((X + 128) / 256) in [-64, 64] and lo in [-128, 127]; hi goes to plane row 2r, lo to
// 2r+1, bytes in the order (0,2,4,6,1,3,5,7) of each 8-group (the order in which a packed INT4
// word unpacks); the sum of X over every 32-K group (for the MMA's offset correction) and the
// block scales go to the row's meta words.
__global__ void __launch_bounds__(256) planes_kernel(const uint4* __restrict__ a, int a_is_bf16,
                                                     const int32_t* __restrict__ inv_pos,
                                                     const int32_t* __restrict__ ids,
                                                     const int32_t* __restrict__ cls_rows, int n_pairs, int k, int K,
                                                     uint2* __restrict__ planes, int32_t* __restrict__ meta) {
  const int nblk = K / 128;
  const size_t unit = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 4;  // (pair, block)
  const int i = threadIdx.x & 15;                                             // 8-group within the block
  const bool live = unit < (size_t)n_pairs * nblk;
  const int p = live ? (int)(unit / nblk) : 0;
  const int blk = live ? (int)(unit % nblk) : 0;
  int r = live ? (inv_pos ? inv_pos[p] : p) : -1;
  // a pair whose expert runs on the other GEMM (ids[p] is read only for a pair inv_pos placed)
  if (r >= 0 && cls_rows && __ldg(cls_rows + __ldg(ids + p)) == 0) r = -1;
  // a warp's two units are (pair, block) neighbours, nearly always of one pair: a warp with
  // nothing to write leaves before any load or arithmetic
  if (__all_sync(0xffffffffu, r < 0)) return;
  const int src = p / k;
  float x[8];
  float amax = 0.f;
  if (live && r >= 0) {
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
  const float sc = fmaxf(amax, 1e-30f) * (1.0f / kFixMax);
  int X[8], sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    X[j] = __float2int_rn(__fdiv_rn(x[j], sc));
    sum += X[j];
  }
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);  // 4 threads = one 32-K group
  if (!live || r < 0) return;
  constexpr int ord[8] = {0, 2, 4, 6, 1, 3, 5, 7};
  uint32_t hb[2] = {0, 0}, lb[2] = {0, 0};
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int v = X[ord[q]];
    const int h8 = (v + 128) >> 8;
    const int l8 = v - 256 * h8;
    hb[q >> 2] |= (uint32_t)(h8 & 0xFF) << (8 * (q & 3));
    lb[q >> 2] |= (uint32_t)(l8 & 0xFF) << (8 * (q & 3));
  }
  const size_t o = ((size_t)(2 * r) * K + blk * 128 + 8 * i) / 8;
  planes[o] = make_uint2(hb[0], hb[1]);
  planes[o + K / 8] = make_uint2(lb[0], lb[1]);
  int32_t* m = meta + (size_t)r * meta_words_per_row(K) + (blk >> 1) * kMetaWords;
  if ((i & 3) == 0) m[(blk & 1) * 4 + (i >> 2)] = kFixBias - 8 * sum;
  if (i == 0) m[8 + (blk & 1)] = __float_as_int(sc);
}

cudaError_t launch_planes(const uint16_t* a, int a_is_bf16, const int32_t* inv_pos, const int32_t* ids,
                          const int32_t* cls_rows, int n_pairs, int k, int K, int8_t* planes, int32_t* meta,
                          cudaStream_t s) {
  const size_t threads = (size_t)n_pairs * (K / 128) * 16;
  timing_before("planes", s);
  planes_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(reinterpret_cast<const uint4*>(a), a_is_bf16,
                                                                  inv_pos, ids, cls_rows, n_pairs, k, K,
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
  reduce_splits_kernel<<<dim3(bx, (unsigned)E), 256, 0, s>>>(reinterpret_cast<const float4*>(part), splits, rows, N,
                                                              row_start, row_count, out, out_fp32);
  timing_after("reduce_splits", s);
  return cudaGetLastError();
}

// rows of the single grouped GEMM's activations -> interleaved fp16; a value outside the finite
// fp16 range (or a non-finite fp16 input) is recorded as MOE_ERR_DEVICE_CHECK
__global__ void __launch_bounds__(256) convert_rows_kernel(const uint4* __restrict__ a, int a_is_bf16, size_t n8,
                                                           uint4* __restrict__ out) {
  bool bad = false;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(a + i);
    bad |= a_is_bf16 ? bf16x8_beyond_f16(v) : f16x8_nonfinite(v);
    out[i] = a_is_bf16 ? bf16x8_to_f16x8_interleaved(v) : f16x8_interleave(v);
  }
  if (bad) set_status(MOE_ERR_DEVICE_CHECK);
}

cudaError_t launch_convert_rows(const uint16_t* a, int a_is_bf16, int M, int K, __half* out, cudaStream_t s) {
  const size_t n8 = (size_t)M * K / 8;
  const int blocks = (int)std::min<size_t>((n8 + 255) / 256, (size_t)sm_count() * 8);
  timing_before("convert", s);
  convert_rows_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(a), a_is_bf16, n8,
                                             reinterpret_cast<uint4*>(out));
  timing_after("convert", s);
  return cudaGetLastError();
}

// out[t][c..c+3] = sum_s w[t][s] * y_perm[inv_pos[t*k+s]][c..c+3], fp32, slot order
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y, const int32_t* __restrict__ inv_pos,
                                                      const float* __restrict__ w, int T, int k, int H4,
                                                      void* __restrict__ out, int out_fp32) {
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
  combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(reinterpret_cast<const float4*>(y_perm), inv_pos, topk_w,
                                                              T, k, H / 4, out, out_fp32);
  timing_after("combine", s);
  return cudaGetLastError();
}

}  // namespace moe
