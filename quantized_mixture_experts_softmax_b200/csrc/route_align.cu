// a1 router (softmax top-k) and a2/a3 token-to-expert alignment plus the tile scheduler.
//
// Router: one warp per token, the token's E logits spread over the 32 lanes; k rounds of a
// warp-wide arg-max (value descending, expert index ascending) pick the winners; weights are
// exp(l_s - l_max) normalised over the winners (or over all E experts).
//
// Alignment: a stable counting sort of the T*k (token, slot) pairs by expert, done in three
// short kernels so that it is deterministic and needs no host round trip:
//   hist    per 512-pair chunk, a shared-memory histogram over experts;
//   scan    one CTA: per expert, an exclusive scan of the chunk histograms (each chunk's base
//           within the expert), counts, padded offsets, padding sentinels, and the tile
//           scheduler's per-expert token tiles;
//   scatter per chunk, one warp walks its pairs in order; lanes routed to the same expert
//           find each other with __match_any_sync and take consecutive rows.
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kAlignChunk = 512;

// ------------------------------------------------------------------ router
template <int EPL>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                    int renormalize, int32_t* __restrict__ ids,
                                                    float* __restrict__ w) {
  grid_dependency_sync();  // see common.cuh
  const int warp = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  const float* row = logits + (size_t)warp * E;
  float v[EPL];
  uint32_t taken = 0;
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = j * 32 + lane;
    v[j] = e < E ? __ldg(row + e) : -INFINITY;
    if (e >= E) taken |= 1u << j;
  }
  float vmax = 0.f, sum_top = 0.f;
  int32_t* ids_row = ids + (size_t)warp * k;
  float* w_row = w + (size_t)warp * k;
  for (int s = 0; s < k; ++s) {
    float bv = -INFINITY;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      if (!((taken >> j) & 1u) && (bi == 0x7FFFFFFF || v[j] > bv)) {  // ascending index: first max wins
        bv = v[j];
        bi = j * 32 + lane;
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      const bool better = (oi != 0x7FFFFFFF) && (bi == 0x7FFFFFFF || ov > bv || (ov == bv && oi < bi));
      if (better) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (s == 0) vmax = bv;
    const float ex = expf(bv - vmax);
    sum_top += ex;
    if (lane == 0) {
      ids_row[s] = bi;
      w_row[s] = ex;
    }
  }
  float denom = sum_top;
  if (!renormalize) {
    float part = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (j * 32 + lane < E) part += expf(v[j] - vmax);
#pragma unroll
    for (int off = 16; off; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    denom = part;
  }
  __syncwarp();
  const float inv = 1.0f / denom;
  for (int s = lane; s < k; s += 32) w_row[s] = w_row[s] * inv;
}

cudaError_t launch_route(const float* logits, int T, int E, int k, int renormalize, int32_t* ids, float* w,
                         cudaStream_t s) {
  const int blocks = ceil_div(T, 8);
  timing_before("route", s);
  const int epl = ceil_div(E, 32);
  if (epl <= 1)
    (void)launch_kernel(route_kernel<1>, dim3(blocks), dim3(256), 0, s, logits, T, E, k, renormalize, ids, w);
  else if (epl <= 2)
    (void)launch_kernel(route_kernel<2>, dim3(blocks), dim3(256), 0, s, logits, T, E, k, renormalize, ids, w);
  else if (epl <= 4)
    (void)launch_kernel(route_kernel<4>, dim3(blocks), dim3(256), 0, s, logits, T, E, k, renormalize, ids, w);
  else if (epl <= 8)
    (void)launch_kernel(route_kernel<8>, dim3(blocks), dim3(256), 0, s, logits, T, E, k, renormalize, ids, w);
  else if (epl <= 16)
    (void)launch_kernel(route_kernel<16>, dim3(blocks), dim3(256), 0, s, logits, T, E, k, renormalize, ids, w);
  else
    (void)launch_kernel(route_kernel<32>, dim3(blocks), dim3(256), 0, s, logits, T, E, k, renormalize, ids, w);
  timing_after("route", s);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ block-wide exclusive scan (1024 threads)
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  if (lane == 31) warp_tot[wid] = inc;
  __syncthreads();
  if (wid == 0) {
    int t = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
    int ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += o;
    }
    warp_tot[lane] = ti - t;  // exclusive prefix of warp totals
    if (lane == 31) *total = ti;
  }
  __syncthreads();
  const int r = warp_tot[wid] + inc - v;
  __syncthreads();
  return r;
}

// token tiles of an expert with `c` rows, at most `nmax` rows each, balanced, rows a multiple of
// min(nmax, 16)
__device__ __forceinline__ void expert_tiles(int c, int nmax, int* nt, int* ch) {
  if (c <= 0) {
    *nt = 0;
    *ch = 16;
    return;
  }
  const int nt0 = (c + nmax - 1) / nmax;
  const int q = nmax < 16 ? nmax : 16;
  int chunk = (c + nt0 - 1) / nt0;
  chunk = (chunk + q - 1) / q * q;
  *ch = chunk;
  *nt = (c + chunk - 1) / chunk;
}

// ------------------------------------------------------------------ align kernels
__global__ void __launch_bounds__(256) align_hist_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                         int32_t* __restrict__ blockcnt) {
  grid_dependency_sync();  // see common.cuh
  __shared__ int cnt[1024];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int p0 = blockIdx.x * kAlignChunk;
  const int p1 = min(P, p0 + kAlignChunk);
  for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
    const int e = ids[p];
    if (e >= 0 && e < E)
      atomicAdd(&cnt[e], 1);
    else
      set_status(MOE_ERR_DEVICE_CHECK);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) blockcnt[(size_t)blockIdx.x * E + e] = cnt[e];
}

__global__ void __launch_bounds__(1024) align_scan_kernel(int32_t* __restrict__ blockcnt, int nb, int E, int align,
                                                          int P, int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ sorted_ids, SchedOut sch) {
  grid_dependency_sync();  // see common.cuh
  __shared__ int warp_tot[32];
  __shared__ int total;
  const int e = threadIdx.x;
  int c = 0;
  if (e < E) {
    for (int b = 0; b < nb; ++b) {
      const int v = blockcnt[(size_t)b * E + e];
      blockcnt[(size_t)b * E + e] = c;  // base of chunk b within expert e
      c += v;
    }
    counts[e] = c;
  }
  const int padded = e < E ? (c + align - 1) / align * align : 0;
  const int off = block_exclusive_scan(padded, warp_tot, &total);
  if (e < E) offsets[e] = off;
  if (e == 0) offsets[E] = total;
  if (e < E)
    for (int r = off + c; r < off + padded; ++r) sorted_ids[r] = P;
  if (sch.tile_prefix) {
    // per expert, from its actual count: the thin schedule (int8 tensor-core GEMM, small token
    // tiles) when it has at most thin_rows rows, else the main one (fp16 GEMM, wide tiles)
    // (with thin_rows = 0 the thin schedule is still written, empty, so no reader sees stale data)
    const bool two = sch.thin_tile_prefix != nullptr;
    const bool thin = two && c <= sch.thin_rows;
    const int c_main = thin ? 0 : c;
    int nt = 0, ch = 16;
    if (e < E) expert_tiles(c_main, sch.nmax, &nt, &ch);
    const int tp = block_exclusive_scan(nt, warp_tot, &total);
    if (e < E) {
      sch.tile_prefix[e] = tp;
      sch.chunk[e] = ch;
      if (sch.row_count) sch.row_count[e] = c_main;
    }
    if (e == 0) sch.tile_prefix[E] = total;
    if (two) {
      const int c_thin = thin ? c : 0;
      int nt2 = 0, ch2 = 16;
      if (e < E) expert_tiles(c_thin, sch.thin_nmax, &nt2, &ch2);
      const int tp2 = block_exclusive_scan(nt2, warp_tot, &total);
      if (e < E) {
        sch.thin_tile_prefix[e] = tp2;
        sch.thin_chunk[e] = ch2;
        sch.thin_row_count[e] = c_thin;
      }
      if (e == 0) sch.thin_tile_prefix[E] = total;
      if (sch.thin_row_prefix) {
        const int rp = block_exclusive_scan(e < E ? c_thin : 0, warp_tot, &total);
        if (e < E) sch.thin_row_prefix[e] = rp;
        if (e == 0) sch.thin_row_prefix[E] = total;
      }
    }
  }
}

__global__ void __launch_bounds__(32) align_scatter_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                           const int32_t* __restrict__ blockbase,
                                                           const int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ sorted_ids,
                                                           int32_t* __restrict__ inv_pos) {
  grid_dependency_sync();  // see common.cuh
  __shared__ int cur[1024];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) cur[e] = offsets[e] + blockbase[(size_t)blockIdx.x * E + e];
  __syncwarp();
  const int p0 = blockIdx.x * kAlignChunk;
  for (int i = 0; i < kAlignChunk; i += 32) {
    const int p = p0 + i + lane;
    const int e = p < P ? ids[p] : -1;
    const bool valid = e >= 0 && e < E;
    const int key = valid ? e : -(lane + 2);  // invalid lanes never group with anyone
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    int pos = -1;
    if (valid) pos = cur[e] + __popc(peers & ((1u << lane) - 1u));
    __syncwarp();
    if (valid) {
      sorted_ids[pos] = p;
      if (lane == __ffs(peers) - 1) cur[e] += __popc(peers);
    }
    if (p < P) inv_pos[p] = pos;
    __syncwarp();
  }
}

int align_blocks(int T, int k) { return ceil_div(T * k, kAlignChunk); }

cudaError_t launch_align(const int32_t* ids, int T, int k, int E, int align, int32_t* counts, int32_t* offsets,
                         int32_t* sorted_ids, int32_t* inv_pos, int32_t* blockcnt, const SchedOut* sched,
                         cudaStream_t s) {
  const int P = T * k;
  const int nb = align_blocks(T, k);
  timing_before("align_hist", s);
  (void)launch_kernel(align_hist_kernel, dim3(nb), dim3(256), 0, s, ids, P, E, blockcnt);
  timing_after("align_hist", s);
  timing_before("align_scan", s);
  SchedOut none{};
  (void)launch_kernel(align_scan_kernel, dim3(1), dim3(1024), 0, s, blockcnt, nb, E, align, P, counts, offsets, sorted_ids, sched ? *sched : none);
  timing_after("align_scan", s);
  timing_before("align_scatter", s);
  (void)launch_kernel(align_scatter_kernel, dim3(nb), dim3(32), 0, s, ids, P, E, blockcnt, offsets, sorted_ids, inv_pos);
  timing_after("align_scatter", s);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ scheduler from caller offsets
// One block of 1024 threads (one per expert, E <= 1024).
__device__ __forceinline__ void sched_from_offsets_block(const int32_t* __restrict__ offsets, int E, int M, int nmax,
                                                         int32_t* __restrict__ row_count,
                                                         int32_t* __restrict__ tile_prefix,
                                                         int32_t* __restrict__ chunk) {
  __shared__ int warp_tot[32];
  __shared__ int total;
  const int e = threadIdx.x;
  int c = 0;
  if (e < E) {
    const int a = offsets[e], b = offsets[e + 1];
    if (a < 0 || b < a || b > M) {
      set_status(MOE_ERR_DEVICE_CHECK);
    } else {
      c = b - a;
    }
    row_count[e] = c;
  }
  int nt = 0, ch = 16;
  if (e < E) expert_tiles(c, nmax, &nt, &ch);
  const int tp = block_exclusive_scan(nt, warp_tot, &total);
  if (e < E) {
    tile_prefix[e] = tp;
    chunk[e] = ch;
  }
  if (e == 0) tile_prefix[E] = total;
}

__global__ void __launch_bounds__(1024) sched_from_offsets_kernel(const int32_t* __restrict__ offsets, int E, int M,
                                                                  int nmax, int32_t* __restrict__ row_count,
                                                                  int32_t* __restrict__ tile_prefix,
                                                                  int32_t* __restrict__ chunk) {
  grid_dependency_sync();  // see common.cuh
  sched_from_offsets_block(offsets, E, M, nmax, row_count, tile_prefix, chunk);
}

cudaError_t launch_sched_from_offsets(const int32_t* offsets, int E, int M, int nmax, int32_t* row_count,
                                      int32_t* tile_prefix, int32_t* chunk, cudaStream_t s) {
  timing_before("sched", s);
  (void)launch_kernel(sched_from_offsets_kernel, dim3(1), dim3(1024), 0, s, offsets, E, M, nmax, row_count, tile_prefix, chunk);
  timing_after("sched", s);
  return cudaGetLastError();
}

}  // namespace moe
