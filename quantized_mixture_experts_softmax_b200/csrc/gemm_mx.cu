// W4A8 grouped expert GEMM: MXFP4 weights x FP8 activations on tcgen05 kind::mxf8f6f4 with
// block scaling.
//
// The format (the Humming issue "[Performance] W4A8 MoE GEMM significantly slower than W4A16 on
// H200", opening report): weights MXFP4 - E2M1 codes sharing one E8M0 power-of-two scale per 32
// along K - and FP8 activations quantized in groups of 32 along K, here with E8M0 scales as
// well.  Both scales are what the block-scaled MMA consumes: each K = 32 step multiplies a weight
// row's and a token's E2M1 x E4M3 products by the row's and the token's scales of those 32 K,
// so the whole reduction accumulates in one TMEM tile, with no promotion on the CUDA cores
// (the block-FP8 GEMM's bottleneck).
//
// Operands in shared memory (128-byte swizzle, K-major, one stage per 128 K):
//   weights  the TMA unpacks a row's 128 packed E2M1 codes (64 bytes in HBM) into a 128-byte
//            row, 16 codes in the first 8 bytes of every 16-byte chunk: the layout the MMA
//            reads for a 4-bit operand of kind::mxf8f6f4;
//   tokens   e4m3 rows.
// Scales in tensor memory: row m's four E8M0 codes of a stage (one per K = 32 step) are the four
// bytes of the 32-bit cell at lane m % 32 and column m / 32 of the stage's scale block, repeated
// in all four lane quarters (each quarter's datapath reads its own copy); the MMA's scale-factor
// id picks the step's byte.  Weight scales arrive with the stage by bulk copy (their HBM layout
// [E, K/128, rows, 4] makes a 128-row tile's stage 512 contiguous bytes); token scales are
// read from the activation producer's [K/128, rows] words.
//
// One persistent CTA per SM over the (expert, weight tile(s), token tile) work list of the other
// grouped GEMMs, weights in the MMA's M slot (128 rows), tokens in N.  Warp roles (384 threads):
//   warp 0      TMA producer: NA weight tiles (gate and up, or two adjacent down tiles), the
//               token tile and the weight scales, one stage per 128 K;
//   warps 1, 3  MMA issuers (warp 1 also allocates TMEM): four K = 32 block-scaled MMAs per
//               matrix and stage into one of two accumulator tiles; with token tiles of up to 64
//               rows one warp per weight matrix (the MMAs' fixed cost per instruction bounds the
//               decode GEMMs: 6% faster than one issuer), else warp 1 alone; they never wait on
//               an mbarrier (a thread with MMAs in flight would stall there until they drain)
//               and are released stage by stage by
//   warp 2      the MMA scheduler, which waits for the stage's copies and scales (and, at an
//               item's first stage, for a free accumulator tile);
//   warps 4-7   scale warps, one per lane quarter: per stage, the weight scales from shared
//               memory and the token scales from global memory into the stage's TMEM block;
//   warps 8-11  epilogue, one per lane quarter, a thread per weight row: the gate/up GEMM ends
//               with h = SiLU(gate) * up quantized to e4m3 per (token, 32 columns) - a warp's
//               32 rows are exactly one group, so the group max is one warp reduction - and
//               the down GEMM stores fp32.
#include <cuda_fp8.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace mx {

constexpr int BM = 128;  // weight rows per tile (MMA M)
constexpr int KB = 128;  // K per stage
constexpr int kMmaWarp = 1;
constexpr int kSchedWarp = 2;
constexpr int kMmaWarp2 = 3;    // the second matrix's MMA issuer (NA = 2)
constexpr int kMmaBarrier = 1;  // named barrier of the MMA and scheduler warps (0 is __syncthreads)
constexpr int kScaleWarp0 = 4;
constexpr int kEpiWarp0 = 8;
constexpr int kThreads = 12 * 32;
constexpr uint32_t kScaleOne = 0x7F7F7F7Fu;  // four E8M0 codes of 1.0

template <bool GATED, int NMAX, int NA_>
struct Cfg {
  static_assert(NMAX % 16 == 0 && NMAX <= 128, "token tile");
  static_assert(!GATED || NA_ == 2, "gate and up tiles");
  static constexpr int NA = NA_;
  static constexpr int NI = NA == 2 && NMAX <= 64 ? 2 : 1;  // MMA issuer warps
  static constexpr int W_TILE = BM * KB;   // unpacked E2M1 bytes in shared memory
  static constexpr int W_TX = BM * KB / 2;  // bytes the TMA reads (packed) and counts
  static constexpr int B_TILE = NMAX * KB;
  static constexpr int SFA_OFF = NA * W_TILE + B_TILE;
  static constexpr int STAGE = (SFA_OFF + NA * BM * 4 + 1023) / 1024 * 1024;
  static constexpr int ST = (232448 - 1024 - 4 * 1025 - 512) / STAGE;
  static_assert(ST >= 3, "pipeline depth");
  static constexpr int P_COLS = NA * NMAX;       // one accumulator tile: [matrix][NMAX] columns
  static constexpr int SF_COLS = NA * 4 + 4;     // TMEM columns of one stage's scales
  // accumulator tiles: two (the epilogue of one item overlaps the next item's MMAs) where they
  // fit next to the scale blocks
  static constexpr int NPB = 2 * P_COLS + ST * SF_COLS <= 512 ? 2 : 1;
  static constexpr int SF_BASE = NPB * P_COLS;
  static constexpr int USED = SF_BASE + ST * SF_COLS;
  static constexpr int TMEM_COLS = USED <= 32 ? 32 : USED <= 64 ? 64 : USED <= 128 ? 128 : USED <= 256 ? 256 : 512;
  static_assert(USED <= 512, "tensor memory");
  static constexpr int OFF_BAR = ST * STAGE;
  static constexpr int NUM_BARS = 3 * ST + 2 * NPB + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_PREFIX = OFF_MISC + 16;
  static_assert(SFA_OFF % 16 == 0, "bulk copies land on 16-byte boundaries");
  static_assert(STAGE % 1024 == 0 && (NA * W_TILE) % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static constexpr size_t smem_bytes(int E) { return (size_t)OFF_PREFIX + 4 * (size_t)(E + 1) + 1024; }
  static_assert(smem_bytes(1024) <= 232448, "shared memory budget");
};

struct Params {
  int K, E, rows_per_expert, I, m_tiles;
  int row_off2;              // NA = 2: rows of the second tile after the first (I for gate/up, 128 for down)
  const uint8_t* w_sf;       // [E, K/128, rows_per_expert, 4]
  const uint32_t* x_sf;      // [K/128, act_rows]: four E8M0 codes per token and 128 K
  int act_rows;
  TileSched sched;
  void* out;                 // GATED: e4m3 h [act_rows, I]; else fp32 y [act_rows, out_ld]
  int out_ld;
  uint8_t* h_sf;             // GATED: [I/128, act_rows, 4]
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

template <bool GATED, int NMAX, int NA_>
__global__ void __launch_bounds__(kThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_b,
                   const Params p) {
  using C = Cfg<GATED, NMAX, NA_>;
  constexpr int NA = C::NA, ST = C::ST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + ST;
  uint64_t* sf_full = empty + ST;
  uint64_t* d_full = sf_full + ST;
  uint64_t* d_empty = d_full + C::NPB;
  uint64_t* drain = d_empty + C::NPB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* sprefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::NI);  // one commit per MMA issuer
      mbar_init(&sf_full[i], 4);
    }
    for (int i = 0; i < C::NPB; ++i) {
      mbar_init(&d_full[i], C::NI);
      mbar_init(&d_empty[i], 4);
    }
    mbar_init(drain, C::NI);
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
  grid_dependency_wait();  // the schedule and the activations come from the preceding kernels
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) sprefix[i] = __ldg(p.sched.tile_prefix + i);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = p.m_tiles * sprefix[p.E];
  const int nkb = p.K / KB;
  constexpr int kMmaThreads = 32 * (1 + C::NI);  // the scheduler and the MMA issuers

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
        const int rin_g = I.m * (GATED ? BM : NA * BM);  // first tile's first row within the expert
        const int rin_u = rin_g + p.row_off2;
        const int row_g = I.e * p.rows_per_expert + rin_g;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!(ok = mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim))) break;
          uint8_t* st = smem + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], (uint32_t)(NA * C::W_TX + I.nmma * KB + NA * BM * 4));
          tma_load_2d_hint(st, &tm_w, &full[s], kb * KB, row_g, pol_w);
          if (NA == 2) tma_load_2d_hint(st + C::W_TILE, &tm_w, &full[s], kb * KB, row_g + p.row_off2, pol_w);
          for (int r = 0; r < I.nmma; r += 16)
            tma_load_2d_hint(st + NA * C::W_TILE + r * KB, &tm_b, &full[s], kb * KB, I.r0 + r, pol_b);
          const uint8_t* sf = p.w_sf + ((size_t)I.e * nkb + kb) * p.rows_per_expert * 4;
          bulk_load(st + C::SFA_OFF, sf + (size_t)rin_g * 4, BM * 4, &full[s]);
          if (NA == 2) bulk_load(st + C::SFA_OFF + BM * 4, sf + (size_t)rin_u * 4, BM * 4, &full[s]);
          ++issued;
          if (++s == ST) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      for (int i = max(0, issued - ST); i < issued; ++i) mbar_wait_plain(&full[i % ST], (i / ST) & 1, lim);
    }
  } else if (warp == kMmaWarp || (C::NI == 2 && warp == kMmaWarp2)) {
    // ---------------------------------------------------------------- MMA issuers
    // Released stage by stage by the scheduler warp; identical loop bounds on all sides.  With
    // one issuer, warp 1 issues matrix 0 and then matrix 1 per K step; with two, its own only.
    const int mat = warp == kMmaWarp ? 0 : 1;
    int s = 0, pb = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      const Item I = decode_item(it, sprefix, p);
      const uint32_t d = tmem_base + (uint32_t)(pb * C::P_COLS + mat * NMAX);  // this warp's first matrix
      for (int kb = 0; kb < nkb; ++kb) {
        if (!(ok = bar_red_and(kMmaBarrier, kMmaThreads, true))) break;
        if (lane == 0) {
          tc_fence_after();
          const uint8_t* st = smem + s * C::STAGE;
          const uint64_t a = sw128_kmajor_desc(smem_u32(st + mat * C::W_TILE));
          const uint64_t a2 = sw128_kmajor_desc(smem_u32(st + (NA - 1) * C::W_TILE));
          const uint64_t b = sw128_kmajor_desc(smem_u32(st + NA * C::W_TILE));
          const uint32_t sfb = tmem_base + (uint32_t)(C::SF_BASE + s * C::SF_COLS + NA * 4);
          const uint32_t sfa = tmem_base + (uint32_t)(C::SF_BASE + s * C::SF_COLS + 4 * mat);
#pragma unroll
          for (int kk = 0; kk < KB / 32; ++kk) {  // K = 32 codes = 32 bytes of a swizzled row per MMA
            const uint32_t idesc = make_idesc_mx(BM, I.nmma, (uint32_t)kk);
            const uint32_t id = (uint32_t)kk << 30;
            const uint32_t acc = (kb | kk) != 0;
            umma_mx(d, a + 2 * kk, b + 2 * kk, idesc, acc, sfa | id, sfb | id);
            if (C::NI == 1 && NA == 2)
              umma_mx(d + NMAX, a2 + 2 * kk, b + 2 * kk, idesc, acc, (sfa + 4) | id, sfb | id);
          }
          umma_commit(&empty[s]);
          if (kb == nkb - 1) umma_commit(&d_full[pb]);
        }
        __syncwarp();
        if (++s == ST) s = 0;
      }
      if (++pb == C::NPB) pb = 0;
    }
    if (lane == 0) {
      umma_commit(drain);
      mbar_wait_plain(drain, 0, lim);
    }
  } else if (warp == kSchedWarp) {
    // ---------------------------------------------------------------- MMA scheduler
    int s = 0, pb = 0;
    uint32_t ph = 0, ph_d = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      for (int kb = 0; kb < nkb; ++kb) {
        bool ready = kb != 0 || __all_sync(0xffffffffu, mbar_wait(&d_empty[pb], ph_d ^ 1u, abort_flag, lim));
        ready = ready && __all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag, lim)) &&
                __all_sync(0xffffffffu, mbar_wait(&sf_full[s], ph, abort_flag, lim));
        if (!(ok = bar_red_and(kMmaBarrier, kMmaThreads, ready))) break;
        if (++s == ST) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (++pb == C::NPB) {
        pb = 0;
        ph_d ^= 1u;
      }
    }
  } else if (warp >= kScaleWarp0 && warp < kEpiWarp0) {
    // ---------------------------------------------------------------- scale warps
    const int q = warp & 3;  // TMEM lanes 32q..32q+31
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      const Item I = decode_item(it, sprefix, p);
      // token scales of tokens lane + 32j, one stage ahead of the copies they wait for
      auto tok_sf = [&](int kb, int j) {
        const int t = lane + 32 * j;
        return (t < I.nvalid && kb < nkb) ? __ldg(p.x_sf + (size_t)kb * p.act_rows + I.r0 + t) : kScaleOne;
      };
      uint32_t xn[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) xn[j] = 32 * j < NMAX ? tok_sf(0, j) : kScaleOne;
      for (int kb = 0; kb < nkb; ++kb) {
        uint32_t xb[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          xb[j] = xn[j];
          xn[j] = 32 * j < NMAX ? tok_sf(kb + 1, j) : kScaleOne;
        }
        // the stage's weight scales have landed; the MMAs of this slot's previous use are
        // complete (the producer refilled the stage after them)
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag, lim)))) break;
        tc_fence_after();
        const uint32_t* sfa = reinterpret_cast<const uint32_t*>(smem + s * C::STAGE + C::SFA_OFF);
        const uint32_t col = tmem_base + lane_base + (uint32_t)(C::SF_BASE + s * C::SF_COLS);
#pragma unroll
        for (int mat = 0; mat < NA; ++mat) {
          uint32_t v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) v[j] = sfa[mat * BM + 32 * j + lane];
          tmem_st4(col + 4 * mat, v);
        }
        tmem_st4(col + 4 * NA, xb);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full[s]);
        if (++s == ST) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int mrow = q * 32 + lane;
    int pb = 0;
    uint32_t ph_d = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      const Item I = decode_item(it, sprefix, p);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&d_full[pb], ph_d, abort_flag, lim)))) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(pb * C::P_COLS);
      for (int c0 = 0; c0 < I.nmma; c0 += 16) {
        uint32_t ra[16], rb[16];
        tmem_ld16(tb + c0, ra);
        if (NA == 2) tmem_ld16(tb + NMAX + c0, rb);
        tmem_ld_wait();
        if constexpr (GATED) {
          // h = SiLU(gate) * up; per token, this warp's 32 rows are one 32-column group of h
          uint8_t* hq = reinterpret_cast<uint8_t*>(p.out);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float g = __uint_as_float(ra[c]), u = __uint_as_float(rb[c]);
            const float h = __fdividef(g, 1.0f + __expf(-g)) * u;
            const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(h) & 0x7FFFFFFFu);
            const int X = mx_exponent(amax);
            const __nv_fp8_e4m3 code(h * exp2_neg(X));
            const int t = c0 + c;
            if (t < I.nvalid) {
              if (amax >= 0x7F800000u && lane == 0) set_status(MOE_ERR_DEVICE_CHECK);  // inf or NaN
              const size_t row = (size_t)(I.r0 + t);
              hq[row * p.out_ld + I.m * BM + mrow] = *reinterpret_cast<const uint8_t*>(&code);
              if (lane == 0) p.h_sf[((size_t)I.m * p.act_rows + row) * 4 + q] = (uint8_t)(X + 127);
            }
          }
        } else {
          float* y = reinterpret_cast<float*>(p.out);
#pragma unroll
          for (int mat = 0; mat < NA; ++mat) {
            const int n = I.m * (NA * BM) + mat * BM + mrow;
#pragma unroll
            for (int c = 0; c < 16; ++c)
              if (c0 + c < I.nvalid) y[(size_t)(I.r0 + c0 + c) * p.out_ld + n] = __uint_as_float(mat ? rb[c] : ra[c]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[pb]);
      if (++pb == C::NPB) {
        pb = 0;
        ph_d ^= 1u;
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
cudaError_t launch_t(const MxGemmProblem& pr, cudaStream_t s) {
  using C = Cfg<GATED, NMAX, NA_>;
  CUtensorMap tm_w, tm_b;
  const uint64_t wrows = (uint64_t)pr.E * pr.rows_per_expert;
  // 4-bit codes, unpacked into 16-byte chunks in shared memory; the inner extent counts codes
  if (encode_tmap_2d(&tm_w, pr.w, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, pr.K, wrows, (uint64_t)pr.K / 2, KB, BM,
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
  p.w_sf = pr.w_sf;
  p.x_sf = pr.x_sf;
  p.act_rows = pr.act_rows;
  p.sched = pr.sched;
  p.out = pr.out;
  p.out_ld = pr.out_ld;
  p.h_sf = pr.h_sf;
  p.wait_limit = wait_limit_ns();
  const size_t smem = C::smem_bytes(pr.E);
  auto kern = mx_gemm_kernel<GATED, NMAX, NA_>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const char* name = GATED ? "w4a8_gemm_gate_up" : "w4a8_gemm_down";
  timing_before(name, s);
  (void)launch_kernel(kern, dim3(sm_count()), dim3(kThreads), smem, s, tm_w, tm_b, p);
  timing_after(name, s);
  return cudaGetLastError();
}

}  // namespace mx

template <bool GATED, int NA>
static cudaError_t launch_nmax(const MxGemmProblem& p, cudaStream_t s) {
  switch (p.nmax) {
    case 32: return mx::launch_t<GATED, 32, NA>(p, s);
    case 112: return mx::launch_t<GATED, 112, NA>(p, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_mx_gemm(const MxGemmProblem& p, cudaStream_t s) {
  if (p.gated) return launch_nmax<true, 2>(p, s);
  if (p.rows_per_expert % 256 == 0) return launch_nmax<false, 2>(p, s);
  return launch_nmax<false, 1>(p, s);
}

}  // namespace moe
