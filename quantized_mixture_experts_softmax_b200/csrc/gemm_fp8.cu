// a9: block-FP8 grouped expert GEMM (e4m3 x e4m3 on tcgen05 kind::f8f6f4, fp32 promotion).
//
// The format (the Helion article, "Scope: Hopper and quantized formats"): activations carry one
// fp32 scale per 1x128 group of K, weights one fp32 scale per 128x128 block.  A 128-K block of
// the reduction therefore has a single weight scale per 128-row weight tile and one activation
// scale per token, so each block's partial product is computed on the tensor cores in its own
// TMEM tile and promoted on the CUDA cores:
//     acc[row][tok] += P_kb[row][tok] * (w_scale[tile][kb] * x_scale[tok][kb]).
//
// One persistent CTA per SM over the same (expert, 128-row weight tile, token tile) work list as
// the W4A16 GEMM, weights swapped into the MMA's M slot.  Warp roles (352 threads):
//   warp 0      TMA producer: e4m3 weight tiles (128 rows x 128 K, 128-byte swizzle; gate and up
//               tiles for the gate/up GEMM) and the token tile's activations, one stage per
//               128-K block;
//   warp 1      TMEM allocator and single-thread MMA issuer: four K=32 MMAs per matrix per block
//               into one of four partial-product tiles (two where four would pass 512 columns),
//               so the MMAs run up to three blocks ahead of the promotion; it never waits on an
//               mbarrier (see bar_red_and) and is released block by block by
//   warp 2      the MMA scheduler, which waits for the stage's copies and a free partial tile;
//   warps 3-10  promotion and epilogue, two per TMEM lane quarter: each thread owns one weight
//               row and keeps the fp32 accumulators of one half of the tile's tokens (32 of up
//               to 64) in registers.  A block's scale w_scale * x_scale is the same for all 128
//               rows of a token, so each warp forms the 32 products once (a lane per token) and
//               every lane reads them back as float4 broadcasts from shared memory.  The gate/up GEMM ends with h = SiLU(gate) * up,
//               requantized per (token, 128-column group) - the tile's 128 rows are exactly one
//               group - to e4m3 with s = max(amax, 1e-10) / 448; the down GEMM stores fp32.
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace f8 {

constexpr int BM = 128;   // weight rows per tile (MMA M)
constexpr int KB = 128;   // K per stage = one scale block
constexpr int NH = 32;          // tokens per promotion thread (one 32-token part of the tile)
constexpr int kMmaWarp = 1;
constexpr int kSchedWarp = 2;
constexpr int kMmaBarrier = 1;  // named barrier of the MMA and scheduler warps (0 is __syncthreads)
constexpr int kEpiWarp0 = 3;    // warps 3..: promotion; lane quarter warp % 4, token part (warp - 3) / 4

// NMAX = token rows per tile (32 or 64): 4 promotion warps per 32 tokens
// NA_ = 128-row weight tiles per work item: the gate and up tiles (gate/up GEMM), or two
// adjacent output tiles (down GEMM with rows in 256s: twice the MMAs per hand-off and per
// activation tile, half the items), else one.
template <bool GATED, int NMAX, int NA_>
struct Cfg {
  static_assert(NMAX % NH == 0 && NMAX <= 64, "32 or 64 token rows per tile");
  static constexpr int kNumEpi = 4 * (NMAX / NH);
  static constexpr int kThreads = (kEpiWarp0 + kNumEpi) * 32;
  static_assert(!GATED || NA_ == 2, "gate and up tiles");
  static constexpr int NA = NA_;
  static constexpr int W_TILE = BM * KB;    // e4m3 bytes
  static constexpr int B_TILE = NMAX * KB;  // activation bytes
  static constexpr int STAGE = NA * W_TILE + B_TILE;
  static constexpr int ST = NMAX == 32 ? (NA == 2 ? 6 : 10) : (NA == 2 ? 5 : 9);
  static constexpr int P_COLS = NA * NMAX;  // one partial-product tile: [matrix][NMAX] columns
  // partial-product tiles in flight between the MMA and the promotion warps (as many as fit)
  static constexpr int NPB = 4 * P_COLS <= 512 ? 4 : 2;
  static constexpr int TMEM_COLS = NPB * P_COLS <= 32 ? 32 : (NPB * P_COLS <= 64 ? 64 : (NPB * P_COLS <= 128 ? 128 : (NPB * P_COLS <= 256 ? 256 : 512)));
  static_assert(NPB * P_COLS <= TMEM_COLS && TMEM_COLS <= 512, "the partial-product tiles fit the allocation");
  static constexpr int OFF_BAR = ST * STAGE;
  static constexpr int NUM_BARS = 2 * ST + 2 * NPB + 2;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_RED = OFF_MISC + 16;              // [4 lane quarters][NMAX] amax partials
  // [promotion warp][2][NH] block scales of gate and up (gate/up epilogue: h scales and their
  // reciprocals)
  static constexpr int OFF_CS = OFF_RED + 4 * NMAX * 4;
  // gate/up: per promotion warp a [NH tokens][32 rows] byte tile, the e4m3 codes transposed so
  // that each token's 32 bytes leave in two 16-byte stores
  static constexpr int OFF_TR = OFF_CS + kNumEpi * 2 * NH * 4;
  static constexpr int OFF_PREFIX = OFF_TR + (GATED ? kNumEpi * NH * 32 : 0);
  static_assert(OFF_TR % 16 == 0, "the transpose tiles are read as 16-byte vectors");
  static_assert(OFF_CS % 16 == 0, "float4 reads of the block scales");
  static_assert(STAGE % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static constexpr size_t smem_bytes(int E) { return (size_t)OFF_PREFIX + 4 * (size_t)(E + 1) + 1024; }
  static_assert(smem_bytes(1024) <= 232448, "shared memory budget");
};

struct Params {
  int K, E, rows_per_expert, I, m_tiles;
  int row_off2;          // NA = 2: rows of the second tile after the first (I for gate/up, 128 for down)
  const float* w_scale;  // [E, rows_per_expert/128, K/128]
  const float* x_scale;  // transposed activation scales [K/128, act_rows]
  int act_rows;
  TileSched sched;
  void* out;  // GATED: e4m3 h [act_rows, I]; else fp32 y [act_rows, out_ld]
  int out_ld;
  float* h_scale;  // GATED: transposed scales of h [I/128, act_rows]
  uint64_t wait_limit;
};

struct Item {
  int e, m, r0, nvalid, nmma;
};

__device__ __forceinline__ Item decode_item(int it, const int* __restrict__ sprefix, const Params& p) {
  Item I;
  const int tile = it / p.m_tiles;
  int lo = 0, hi = p.E;  // sprefix[lo] <= tile < sprefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (sprefix[mid] <= tile)
      lo = mid;
    else
      hi = mid;
  }
  I.e = lo;
  const int nt = sprefix[lo + 1] - sprefix[lo];
  const int local = it - p.m_tiles * sprefix[lo];
  I.m = local / nt;
  const int t = local - I.m * nt;
  const int ch = __ldg(p.sched.chunk + lo);
  const int cnt = __ldg(p.sched.row_count + lo);
  I.r0 = __ldg(p.sched.row_start + lo) + t * ch;
  I.nvalid = min(ch, cnt - t * ch);
  I.nmma = (I.nvalid + 15) & ~15;
  return I;
}

// Bounded barrier among the 8 epilogue warps (an mbarrier of count 8, alternating phases).
__device__ __forceinline__ bool epi_sync(uint64_t* bar, uint32_t& phase, volatile int* abort, uint64_t lim) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, phase, abort, lim));
  phase ^= 1u;
  return ok;
}

template <bool GATED, int NMAX, int NA_>
__global__ void __launch_bounds__(Cfg<GATED, NMAX, NA_>::kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_b,
                    const Params p) {
  using C = Cfg<GATED, NMAX, NA_>;
  constexpr int NA = C::NA, ST = C::ST, kNumEpi = C::kNumEpi;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + ST;
  uint64_t* p_full = empty + ST;
  uint64_t* p_empty = p_full + C::NPB;
  uint64_t* drain = p_empty + C::NPB;
  uint64_t* epi_bar = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  float* cscale = reinterpret_cast<float*>(smem + C::OFF_CS);
  uint8_t* trbuf = smem + C::OFF_TR;
  int* sprefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < C::NPB; ++i) {
      mbar_init(&p_full[i], 1);
      mbar_init(&p_empty[i], kNumEpi);
    }
    mbar_init(drain, 1);
    mbar_init(epi_bar, kNumEpi);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_b);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  // setup done: wait for the kernels this one depends on (the schedule, the activations),
  // then read the schedule.  The next kernel is not released early: its CTAs would wait through
  // the whole GEMM (measured: the decode layer 35-65 us slower with the release here)
  grid_dependency_wait();
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) sprefix[i] = __ldg(p.sched.tile_prefix + i);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = p.m_tiles * sprefix[p.E];
  const int nkb = p.K / KB;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_b = policy_evict_last();
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
        const Item I = decode_item(it, sprefix, p);
        const int row_g = I.e * p.rows_per_expert + I.m * (GATED ? BM : NA * BM);  // first tile
        const int row_u = row_g + p.row_off2;                                        // second tile
        for (int kb = 0; kb < nkb; ++kb) {
          if (!(ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim))) break;
          uint8_t* st = smem + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], (uint32_t)(NA * C::W_TILE + I.nmma * KB));
          tma_load_2d_hint(st, &tm_w, &full[s], kb * KB, row_g, pol_w);
          if (NA == 2) tma_load_2d_hint(st + C::W_TILE, &tm_w, &full[s], kb * KB, row_u, pol_w);
          for (int r = 0; r < I.nmma; r += 16)
            tma_load_2d_hint(st + NA * C::W_TILE + r * 128, &tm_b, &full[s], kb * KB, I.r0 + r, pol_b);
          ++issued;
          if (++s == ST) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      for (int i = max(0, issued - ST); i < issued; ++i) mbar_wait_plain(&full[i % ST], (i / ST) & 1, lim);
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    // Released block by block by the scheduler warp; identical loop bounds on both sides.
    int s = 0, pb = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      const Item I = decode_item(it, sprefix, p);
      const uint32_t idesc = make_idesc(BM, I.nmma, 0, 0);  // e4m3 x e4m3 -> fp32
      for (int kb = 0; kb < nkb; ++kb) {
        if (!(ok = bar_red_and(kMmaBarrier, 64, true))) break;
        if (lane == 0) {
          tc_fence_after();
          const uint8_t* st = smem + s * C::STAGE;
          const uint64_t a0 = sw128_kmajor_desc(smem_u32(st));
          const uint64_t a1 = sw128_kmajor_desc(smem_u32(st + (NA - 1) * C::W_TILE));
          const uint64_t b = sw128_kmajor_desc(smem_u32(st + NA * C::W_TILE));
          const uint32_t d = tmem_base + (uint32_t)(pb * C::P_COLS);
#pragma unroll
          for (int kk = 0; kk < KB / 32; ++kk) {  // K = 32 e4m3 = 32 bytes per MMA
            umma_f8(d, a0 + 2 * kk, b + 2 * kk, idesc, kk != 0);
            if (NA == 2) umma_f8(d + NMAX, a1 + 2 * kk, b + 2 * kk, idesc, kk != 0);
          }
          umma_commit(&p_full[pb]);
          umma_commit(&empty[s]);
        }
        __syncwarp();
        if (++s == ST) s = 0;
        if (++pb == C::NPB) pb = 0;
      }
    }
    if (lane == 0) {
      umma_commit(drain);
      mbar_wait_plain(drain, 0, lim);
    }
  } else if (warp == kSchedWarp) {
    // ---------------------------------------------------------------- MMA scheduler
    int s = 0, pb = 0;
    uint32_t ph = 0, ph_p = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      for (int kb = 0; kb < nkb; ++kb) {
        const bool ready = __all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag, lim)) &&
                           __all_sync(0xffffffffu, mbar_wait(&p_empty[pb], ph_p ^ 1u, abort_flag, lim));
        if (!(ok = bar_red_and(kMmaBarrier, 64, ready))) break;
        if (++s == ST) {
          s = 0;
          ph ^= 1u;
        }
        if (++pb == C::NPB) {
          pb = 0;
          ph_p ^= 1u;
        }
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- promotion + epilogue
    const int ew = warp & 3;                    // TMEM lanes 32*ew..32*ew+31 (the warp's quarter)
    const int tok0 = ((warp - kEpiWarp0) >> 2) * NH;  // this warp's half of the tile's tokens
    const int mrow = ew * 32 + lane;
    const int GK = p.K / KB;
    // this warp's combined scales of the current block, w_scale * x_scale per token
    float* cs = cscale + (warp - kEpiWarp0) * NA * NH;
    int pb = 0;
    uint32_t ph_p = 0, ph_e = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      const Item I = decode_item(it, sprefix, p);
      const int nv = I.nvalid - tok0;  // tokens of this half (may be <= 0)
      float ag[NH], au[NH];
#pragma unroll
      for (int c = 0; c < NH; ++c) ag[c] = au[c] = 0.f;
      const float* wsg = p.w_scale + ((size_t)I.e * (p.rows_per_expert / BM) + I.m * (GATED ? 1 : NA)) * GK;
      const float* wsu = NA == 2 ? wsg + (size_t)(p.row_off2 / BM) * GK : wsg;
      // per-token activation scales (lane c holds token tok0+c's) and weight-block scales, one
      // block ahead so that their load latency hides behind the current block
      auto xs_at = [&](int kb) {
        return (lane < nv && kb < nkb) ? __ldg(p.x_scale + (size_t)kb * p.act_rows + I.r0 + tok0 + lane) : 0.f;
      };
      float xs_n = xs_at(0), sg_n = __ldg(wsg), su_n = NA == 2 ? __ldg(wsu) : 0.f;
      for (int kb = 0; kb < nkb; ++kb) {
        const float xs_l = xs_n, sg = sg_n, su = su_n;
        xs_n = xs_at(kb + 1);
        if (kb + 1 < nkb) {
          sg_n = __ldg(wsg + kb + 1);
          if (NA == 2) su_n = __ldg(wsu + kb + 1);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&p_full[pb], ph_p, abort_flag, lim));
        if (!ok) break;
        tc_fence_after();
        // the scale of (row block, token) is uniform over the warp's rows: one product per token,
        // read back by every lane as float4 broadcasts
        cs[lane] = sg * xs_l;
        if (NA == 2) cs[NH + lane] = su * xs_l;
        __syncwarp();
        const uint32_t tb = tmem_base + ((uint32_t)(ew * 32) << 16) + (uint32_t)(pb * C::P_COLS + tok0);
        uint32_t pg[16], pu[16];
#pragma unroll
        for (int c0 = 0; c0 < NH; c0 += 16) {
          if (tok0 + c0 < I.nmma) {
            tmem_ld16(tb + c0, pg);
            if (NA == 2) tmem_ld16(tb + NMAX + c0, pu);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
              const float4 g4 = *reinterpret_cast<const float4*>(cs + c0 + i);
              ag[c0 + i + 0] = fmaf(__uint_as_float(pg[i + 0]), g4.x, ag[c0 + i + 0]);
              ag[c0 + i + 1] = fmaf(__uint_as_float(pg[i + 1]), g4.y, ag[c0 + i + 1]);
              ag[c0 + i + 2] = fmaf(__uint_as_float(pg[i + 2]), g4.z, ag[c0 + i + 2]);
              ag[c0 + i + 3] = fmaf(__uint_as_float(pg[i + 3]), g4.w, ag[c0 + i + 3]);
              if (NA == 2) {
                const float4 u4 = *reinterpret_cast<const float4*>(cs + NH + c0 + i);
                au[c0 + i + 0] = fmaf(__uint_as_float(pu[i + 0]), u4.x, au[c0 + i + 0]);
                au[c0 + i + 1] = fmaf(__uint_as_float(pu[i + 1]), u4.y, au[c0 + i + 1]);
                au[c0 + i + 2] = fmaf(__uint_as_float(pu[i + 2]), u4.z, au[c0 + i + 2]);
                au[c0 + i + 3] = fmaf(__uint_as_float(pu[i + 3]), u4.w, au[c0 + i + 3]);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_empty[pb]);
        if (++pb == C::NPB) {
          pb = 0;
          ph_p ^= 1u;
        }
      }
      if (!ok) break;
      if constexpr (GATED) {
        // h = SiLU(gate) * up; requantize each token's 128 values of this tile (one 1x128 group):
        // the token's amax over the tile's rows comes from the four warps of its half.  All
        // arithmetic of the 32 tokens first, then the stores (independent chains overlap).
        // h overwrites the gate accumulators and |h| the up ones
        float* hv = ag;
        float* m = au;
#pragma unroll
        for (int c = 0; c < NH; ++c) {
          hv[c] = __fdividef(ag[c], 1.0f + __expf(-ag[c])) * au[c];
          m[c] = fabsf(hv[c]);
        }
        // the warp's max |h| per token, by recursive halving: after the step that exchanges
        // `half` values, lane l holds maxima of the tokens whose index agrees with l in the bits
        // above; in the end lane l holds token l's max over the warp's 32 rows (31 shuffles)
#pragma unroll
        for (int half = NH / 2; half >= 1; half >>= 1) {
          const bool up = (lane & half) != 0;
#pragma unroll
          for (int i = 0; i < half; ++i) {
            const float give = up ? m[i] : m[half + i];
            const float keep = up ? m[half + i] : m[i];
            m[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, give, half));
          }
        }
        red[ew * NMAX + tok0 + lane] = m[0];
        if (!(ok = epi_sync(epi_bar, ph_e, abort_flag, lim))) break;
        // token tok0 + lane's scale, computed once per lane and read back by every lane
        const int t = tok0 + lane;
        const float a = fmaxf(fmaxf(red[t], red[NMAX + t]), fmaxf(red[2 * NMAX + t], red[3 * NMAX + t]));
        const float sc_l = __fdiv_rn(fmaxf(a, 1e-10f), 448.0f);
        cs[lane] = sc_l;  // the block-scale area is free after the K loop
        cs[NH + lane] = __frcp_rn(sc_l);
        if (ew == 0 && lane < nv) p.h_scale[(size_t)I.m * p.act_rows + I.r0 + t] = sc_l;
        __syncwarp();
        // q = e4m3(h / s), round to nearest even, saturating; h times the correctly rounded
        // reciprocal of s differs from the quotient by at most an ulp of fp32, which moves a
        // code only for a value that close to a rounding boundary of e4m3 (three mantissa bits)
        uint8_t* tr = trbuf + (warp - kEpiWarp0) * (NH * 32);
#pragma unroll
        for (int c = 0; c < NH; ++c) {
          const __nv_fp8_e4m3 e(hv[c] * cs[NH + c]);
          tr[c * 32 + lane] = *reinterpret_cast<const uint8_t*>(&e);
        }
        __syncwarp();
        if (lane < nv) {  // token tok0 + lane: its bytes of this warp's 32 rows
          const uint4* src = reinterpret_cast<const uint4*>(tr + lane * 32);
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.out) +
                                                (size_t)(I.r0 + tok0 + lane) * p.out_ld + I.m * BM + ew * 32);
          dst[0] = src[0];
          dst[1] = src[1];
        }
        // red[], cs and the transpose tile are reused by the next item
        if (!(ok = epi_sync(epi_bar, ph_e, abort_flag, lim))) break;
      } else {
        float* y = reinterpret_cast<float*>(p.out);
#pragma unroll
        for (int mat = 0; mat < NA; ++mat) {
          const int n = I.m * (NA * BM) + mat * BM + mrow;
#pragma unroll
          for (int c = 0; c < NH; ++c)
            if (c < nv) y[(size_t)(I.r0 + tok0 + c) * p.out_ld + n] = mat ? au[c] : ag[c];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <bool GATED, int NMAX, int NA_>
cudaError_t launch_t(const F8GemmProblem& pr, cudaStream_t s) {
  using C = Cfg<GATED, NMAX, NA_>;
  CUtensorMap tm_w, tm_b;
  const uint64_t wrows = (uint64_t)pr.E * pr.rows_per_expert;
  if (encode_tmap_2d(&tm_w, pr.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.K, wrows, (uint64_t)pr.K, KB, BM,
                     CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tmap_2d(&tm_b, pr.act, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.K, (uint64_t)pr.act_rows, (uint64_t)pr.K, KB,
                     16, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  Params p;
  p.K = pr.K;
  p.E = pr.E;
  p.rows_per_expert = pr.rows_per_expert;
  p.I = pr.I;
  p.m_tiles = GATED ? pr.I / BM : pr.rows_per_expert / (NA_ * BM);
  p.row_off2 = GATED ? pr.I : BM;
  p.w_scale = pr.w_scale;
  p.x_scale = pr.x_scale;
  p.act_rows = pr.act_rows;
  p.sched = pr.sched;
  p.out = pr.out;
  p.out_ld = pr.out_ld;
  p.h_scale = pr.h_scale;
  p.wait_limit = wait_limit_ns();
  const size_t smem = C::smem_bytes(pr.E);
  auto kern = fp8_gemm_kernel<GATED, NMAX, NA_>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const char* name = GATED ? "fp8_gemm_gate_up" : "fp8_gemm_down";
  timing_before(name, s);
  (void)launch_kernel(kern, dim3(sm_count()), dim3(C::kThreads), smem, s, tm_w, tm_b, p);
  timing_after(name, s);
  return cudaGetLastError();
}

}  // namespace f8

cudaError_t launch_fp8_gemm(const F8GemmProblem& p, cudaStream_t s) {
  const bool two = p.rows_per_expert % 256 == 0;  // the down GEMM: two output tiles per item
  if (p.nmax == 32)
    return p.gated ? f8::launch_t<true, 32, 2>(p, s)
                   : (two ? f8::launch_t<false, 32, 2>(p, s) : f8::launch_t<false, 32, 1>(p, s));
  if (p.nmax == 64)
    return p.gated ? f8::launch_t<true, 64, 2>(p, s)
                   : (two ? f8::launch_t<false, 64, 2>(p, s) : f8::launch_t<false, 64, 1>(p, s));
  return cudaErrorInvalidValue;
}

}  // namespace moe
