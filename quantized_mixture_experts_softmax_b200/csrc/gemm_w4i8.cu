// a5-a7 for decode-sized experts: W4A16 grouped GEMM on the int8 tensor cores.
//
// With few tokens per expert the tensor core's cost is set by how many weights one MMA covers
// (a 128-row MMA with N <= 64 takes the same time whatever N is).  An fp16 weight operand
// covers 128x16 weights per instruction; here the INT4 weights go to the tensor core as
// exact unsigned 8-bit integers n = q + 8 (one AND/XOR per four weights, no floating-point
// dequantization), so one kind::i8 MMA covers 128x32 weights - exactly one scale group of
// the format (the Chord article, second paragraph: one BF16 scale per 32 weights).
//
// The 16-bit activations enter as 16-bit fixed point: per (token, 128-K block) a scale
// s = amax / 16383 and integers X = rint(x / s) split into two signed 8-bit planes
// X = 256*hi + lo, interleaved along N (tile row 2c = hi of token c, 2c+1 = its lo; 8 tokens
// give N = 16, the smallest N of a 128-row MMA).  For one
// token t and one weight row r, one MMA per 32-K group g gives D_hi and D_lo exactly in int32:
//     sum_{k in g} q[r][k] * X[t][k] = 256*D_hi + D_lo - 8*C[t][g],   C[t][g] = sum_{k in g} X[t][k],
// (|sum| < 2^22, so adding it to the bits of 1.5 * 2^23 converts it to fp32 exactly), which the
// promotion warps scale by the group's weight scale and the block's activation scale and
// accumulate in fp32.  They read from tensor memory only the columns of the tile's live
// tokens (2, 4, 8 or 16 columns of each MMA's 16), batched under one wait; the tokens' group
// sums and block scales arrive with the stage (one TMA box of the meta words), as do the weight
// scales.  The gate/up kernel ends with h = SiLU(gate) * up written straight back in the same
// fixed-point planes (one scale per token per 128-row tile) for the down kernel.
//
// The MMA-issuing thread never waits on an mbarrier: a wait (or any shared-memory access) by
// the thread that has MMAs in flight stalls until they drain, idling the tensor core for
// hundreds of cycles per wait.  A scheduler warp does the waits and releases an MMA warp
// through a named barrier with an AND reduction (which also carries a timeout or abort).  Even
// that hand-off waits for the releasing warp's own MMAs to drain, so two MMA warps take the D
// slots in turn: while one is held at its barrier, the other's MMAs keep the tensor core busy.
//
// Work list, swap (weights in the MMA's M slot) and persistence as in the fp16 GEMM.  Warps
// (512 threads): 0 producer (TMA of the INT4 words, weight scales, activation planes and meta
// words of the token tile per 256-K stage; cp.async for scale rows not 16-byte aligned),
// 1 TMEM allocator + MMA issuer of even D slots, 3 MMA issuer of odd D slots, 2 MMA scheduler,
// 4-7 promotion and epilogue, 8-15 unpacking INT4 words into u8 rows of tensor memory (the
// MMA's A operand).
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace w4i8 {

constexpr int BM = 128;          // weight rows per tile
constexpr int KB = 256;          // K per stage
constexpr int G = 32;            // K per scale group = K per MMA
constexpr int NG = KB / G;       // groups per stage
constexpr int NT = kI8TileRows;  // token rows per tile (each gives a hi and a lo plane row)
constexpr int DC = 2 * NT;       // D columns of one MMA (N)
constexpr int kThreads = 512;
constexpr int kMmaWarp = 1;     // even D slots (and the TMEM allocator)
constexpr int kMmaWarpOdd = 3;  // odd D slots
constexpr int kSchedWarp = 2;
constexpr int kMmaBarrier = 1;  // named barriers 1 (even slots) and 2 (odd slots) of an MMA warp
                                // and the scheduler warp (0 is __syncthreads)
constexpr int kEpiWarp0 = 4;
constexpr int kUnpackWarp0 = 8;
constexpr int kNumUnpack = 8;
static_assert(NT == 8, "the promotion code handles up to 8 tokens per tile");
// The producer decodes each work item (a binary search of the tile prefix plus three global
// loads, ~1300 cycles with shared memory busy) and publishes it in a ring that the promotion
// warps read once the item's first stage has landed, so the decode never holds the D slots.
constexpr int kItemRing = 16;

// A work item covers NA weight tiles of 128 rows: the gate and up tiles of the same 128
// columns of h (gate/up GEMM), or two adjacent 128-row tiles of the output (down GEMM, when the
// output rows come in 256s; one tile otherwise).  A stage (256 K of an item) holds the NA INT4
// weight tiles, then the token tile's activation atoms, its meta words and the NA tiles' weight
// scales.  Per stage the pipeline pays a fixed cost (copies, hand-offs, TMEM slot cycles) besides
// the bytes; two tiles per stage halve that cost per weight byte (measured on the down GEMM of
// the decode layer: 16 KB stages ran at 0.55 of HBM bandwidth, 32 KB stages of gate/up at 0.88).
template <bool GATED, int NA_>
struct Cfg {
  static_assert(NA_ == 1 || NA_ == 2, "one or two weight tiles per item");
  static_assert(!GATED || NA_ == 2, "gate and up tiles");
  static constexpr int NA = NA_;
  static constexpr int SG = NA == 2 ? 4 : 8;  // groups per D slot (SG * NA MMAs per handoff)
  static constexpr int W_TILE = BM * KB / 2;   // INT4 bytes
  static constexpr int STAGE_B = NA * W_TILE;
  static constexpr int B_ATOM = 2 * NT * 128;  // one 128-K atom of the 2*NT plane rows
  static constexpr int META = STAGE_B + (KB / 128) * B_ATOM;  // [NT tokens][kMetaWords] int32
  static constexpr int META_BYTES = NT * kMetaWords * 4;
  static constexpr int SCL = META + 1024;            // [NA][BM rows][NG] bf16 weight scales
  static constexpr int S_TILE = BM * NG * 2;
  static constexpr int STAGE = SCL + NA * S_TILE;
  static_assert(META_BYTES <= 1024, "meta box fits its slot");
  static constexpr int ST = NA == 2 ? 5 : 9;
  // TMEM: D ring of SG-group slots [group][matrix][DC int32 columns], A ring of whole-stage
  // slots [matrix][group][8 columns] (a 32-K row of u8 = 8 columns)
  static constexpr int D_SLOT = SG * NA * DC;
  static constexpr int DSLOTS = 256 / D_SLOT;
  static constexpr int A_SLOT = NA * NG * 8;
  static constexpr int ASLOTS = NA == 2 ? 2 : 4;
  static constexpr int A_COL0 = DSLOTS * D_SLOT;
  static_assert(A_COL0 + ASLOTS * A_SLOT <= 512, "TMEM has 512 columns");
  static constexpr int OFF_BAR = ST * STAGE;
  static constexpr int NUM_BARS = 2 * ST + 2 * ASLOTS + 2 * DSLOTS + 2;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_RED = OFF_MISC + 16;  // [2 items][4 warps][NT] amax partials
  static constexpr int OFF_ITEMS = OFF_RED + 2 * 4 * NT * 4;  // [kItemRing] decoded items
  static constexpr int OFF_PREFIX = OFF_ITEMS + kItemRing * 16;
  // the producer runs at most ST stages (so at most ST items) ahead of the promotion warps
  static_assert(kItemRing > ST + 1, "item ring deeper than the stage ring");
  static_assert(STAGE % 1024 == 0 && STAGE_B % 1024 == 0, "swizzled tiles need 1024-byte alignment");
  static constexpr size_t smem_bytes(int E) { return (size_t)OFF_PREFIX + 4 * (size_t)(E + 1) + 1024; }
  static_assert(smem_bytes(1024) <= 232448, "shared memory budget");
};

struct Params {
  int K, E, rows_per_expert, I, m_tiles;
  int row_off2;          // NA = 2: rows of the second tile after the first (I for gate/up, 128 for down)
  const uint16_t* w_s;   // bf16 [E*rows_per_expert, K/32]
  int scales_tma;        // 1: weight scales by TMA (K % 256 == 0), else by cp.async
  TileSched sched;
  int out_kind;          // OUT_PLANES (gated), OUT_F32, OUT_BF16
  void* out;             // planes int8 [2*rows, out_ld]; else fp32/bf16 [rows, out_ld]
  int32_t* out_meta;     // planes: meta words of h
  int out_ld;
  int splits;            // K splits per (expert, weight tile, token tile); > 1 only for plain outputs
  float* part;           // splits > 1: fp32 partial sums [splits, act_rows, out_ld]
  int act_rows;
  uint64_t wait_limit;
};

struct Item {
  int e, m, r0, nvalid;
};
static_assert(sizeof(Item) == 16, "ring entry");

__device__ __forceinline__ Item decode_item(int it_, const int* __restrict__ sprefix, const Params& p) {
  Item I;
  const int it = p.splits == 1 ? it_ : it_ / p.splits;  // the (expert, weight tile, token tile)
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
  return I;
}

// D[tmem] = A[tmem] * B[smem]^T, u8 x s8 -> s32, D overwritten (no accumulation)
__device__ __forceinline__ void umma_i8_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(0u)
      : "memory");
}

// 32 lanes x NC consecutive 32-bit columns of tensor memory (NC = 2, 4, 8, 16)
template <int NC>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, uint32_t (&r)[NC]);
template <>
__device__ __forceinline__ void tmem_ldn<2>(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ldn<4>(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_ldn<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_ldn<16>(uint32_t taddr, uint32_t (&r)[16]) {
  tmem_ld16(taddr, r);
}
// Bounded barrier among the 4 epilogue warps (an mbarrier of count 4, alternating phases).
__device__ __forceinline__ bool epi_sync(uint64_t* bar, uint32_t& phase, volatile int* abort, uint64_t lim) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, phase, abort, lim));
  phase ^= 1u;
  return ok;
}

// position of K offset j inside its group of 8 in the plane layout: (0,2,4,6,1,3,5,7)
__device__ __forceinline__ int plane_pos(int j) {
  const int r = j & 7;
  return (j & ~7) | ((r & 1) ? 4 + (r >> 1) : (r >> 1));
}

// fp32 accumulators of one epilogue thread's gate (or only) and up rows, per live token
template <int NP>
struct Promo {
  float ag[NP], au[NP];
};

// Tokens [0, NP) of one D slot (groups g0 .. g0+SG-1 x NA matrices, the first `ngs` of them
// present): loads their 2*NP columns of every (group, matrix) in batches of at most 32
// registers, one wait per batch.  swg/swu: weight scales of this thread's rows per group;
// meta: the stage's meta words per token.  (Handing the slot back right after the last batch
// is in registers, before the arithmetic, measured 4-5% slower on the decode gate/up GEMM.)
template <int NA, int SG, int NP>
__device__ __forceinline__ void promote_slot(uint32_t slot_addr, const int* meta, int g0, int ngs,
                                             const float (&swg)[SG], const float (&swu)[SG], Promo<NP>& P) {
  constexpr int NC = 2 * NP, U = SG * NA;
  constexpr int PER = (32 / NC) < U ? (32 / NC) : U;
#pragma unroll
  for (int b0 = 0; b0 < U; b0 += PER) {
    uint32_t d[PER][NC];
#pragma unroll
    for (int u = 0; u < PER; ++u) tmem_ldn<NC>(slot_addr + (uint32_t)((b0 + u) * DC), d[u]);
    tmem_ld_wait();
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int unit = b0 + u, gg = unit / NA, mat = unit % NA;
      if (SG > 4 && gg >= ngs) continue;  // group beyond K (a half stage; 4 divides every stage)
      const float sw = mat ? swu[gg] : swg[gg];
      // all NP columns are promoted: those of tokens >= nv hold finite values of other rows and
      // are never stored
#pragma unroll
      for (int c = 0; c < NP; ++c) {
        const int bias = meta[c * kMetaWords + g0 + gg];  // kFixBias - 8 * C[c][g]
        const float xsc = __int_as_float(meta[c * kMetaWords + 8 + ((g0 + gg) >> 2)]);
        const int t = (int)d[u][2 * c] * 256 + (int)d[u][2 * c + 1] + bias;
        const float v = __int_as_float(t) - kFixBiasF;  // sum_k q*X, exactly
        if (mat)
          P.au[c] = fmaf(v, sw * xsc, P.au[c]);
        else
          P.ag[c] = fmaf(v, sw * xsc, P.ag[c]);
      }
    }
  }
}

// bf16 number g (0..7) of eight packed in a uint4, as fp32
__device__ __forceinline__ float bf16_at(const uint4& v, int g) {
  const uint32_t word = (g >> 1) == 0 ? v.x : (g >> 1) == 1 ? v.y : (g >> 1) == 2 ? v.z : v.w;
  return __uint_as_float((g & 1) ? (word & 0xFFFF0000u) : (word << 16));
}

// The K loop of one work item for the promotion warps, specialised on the live-token bound NP.
template <bool GATED, int NA_, int NP>
__device__ __forceinline__ bool promote_item(const Params& p, const Item& I, int mrow, int lane, uint32_t lane_base,
                                             const uint8_t* smem, int& s, uint32_t& ph, uint64_t* full,
                                             uint64_t* empty, int& ds, uint32_t& ph_d, uint64_t* d_full,
                                             uint64_t* d_empty, volatile int* abort_flag, int kb0, int kb1,
                                             Promo<NP>& P) {
  using C = Cfg<GATED, NA_>;
  constexpr int NA = C::NA, DSL = C::DSLOTS, ST = C::ST, SG = C::SG;
  const int K = p.K;
  const uint64_t lim = p.wait_limit;
  for (int kb = kb0; kb < kb1; ++kb) {
    const int ng = min(KB, K - kb * KB) / G;
    // the stage's meta words and weight scales (their copies completed long before; this wait
    // also orders the reads after them)
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag, lim))) return false;
    const uint8_t* st = smem + s * C::STAGE;
    const int* meta = reinterpret_cast<const int*>(st + C::META);
    const uint4 sgv = *reinterpret_cast<const uint4*>(st + C::SCL + mrow * 16);
    const uint4 suv = NA == 2 ? *reinterpret_cast<const uint4*>(st + C::SCL + C::S_TILE + mrow * 16) : sgv;
#pragma unroll
    for (int g0 = 0; g0 < NG; g0 += SG) {  // unrolled: scale registers are indexed statically
      if (g0 >= ng) break;
      if (!__all_sync(0xffffffffu, mbar_wait(&d_full[ds], ph_d, abort_flag, lim))) return false;
      tc_fence_after();
      float swg[SG], swu[SG];
#pragma unroll
      for (int gg = 0; gg < SG; ++gg) {
        swg[gg] = bf16_at(sgv, g0 + gg);
        swu[gg] = bf16_at(suv, g0 + gg);
      }
      promote_slot<NA, SG, NP>(lane_base + (uint32_t)(ds * C::D_SLOT), meta, g0, min(SG, ng - g0), swg, swu, P);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[ds]);
      if (++ds == DSL) {
        ds = 0;
        ph_d ^= 1u;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // meta words and scales read, the stage's MMAs done
    if (++s == ST) {
      s = 0;
      ph ^= 1u;
    }
  }
  return true;
}

// One work item of the promotion warps: the K loop, then the epilogue (GATED: h = SiLU(gate)
// * up as fixed-point planes with one scale per (token, tile); else fp32 or bf16 rows of the
// item's NA tiles).
template <bool GATED, int NA_, int NP>
__device__ __forceinline__ bool epi_item(const Params& p, const Item& I, int it, int ew, int lane, uint32_t lane_base,
                                         const uint8_t* smem, int& s, uint32_t& ph, uint64_t* full, uint64_t* empty,
                                         int& ds, uint32_t& ph_d, uint64_t* d_full, uint64_t* d_empty,
                                         float* red, uint64_t* epi_bar, uint32_t& ph_e, volatile int* abort_flag) {
  const int mrow = ew * 32 + lane, nv = I.nvalid;
  Promo<NP> P;
#pragma unroll
  for (int c = 0; c < NP; ++c) P.ag[c] = P.au[c] = 0.f;
  int kb0, kb1;
  split_range(it, ceil_div(p.K, KB), p.splits, kb0, kb1);
  if (!promote_item<GATED, NA_, NP>(p, I, mrow, lane, lane_base, smem, s, ph, full, empty, ds, ph_d, d_full,
                                    d_empty, abort_flag, kb0, kb1, P))
    return false;
  if constexpr (GATED) {
#pragma unroll
    for (int c = 0; c < NP; ++c) {
      const float h = __fdividef(P.ag[c], 1.0f + __expf(-P.ag[c])) * P.au[c];
      P.ag[c] = h;
      // the bit patterns of non-negative floats order like the values: one warp reduction (a NaN
      // counts as 0, as fmaxf would skip it)
      const float ah = fabsf(h);
      const uint32_t m = __reduce_max_sync(0xffffffffu, ah == ah ? __float_as_uint(ah) : 0u);
      if (lane == 0) red[ew * NT + c] = __uint_as_float(m);
    }
    if (!epi_sync(epi_bar, ph_e, abort_flag, p.wait_limit)) return false;
    const int j = I.m * BM + mrow;
    const int pos = plane_pos(j);
    const int mw_h = meta_words_per_row(p.I);
    int8_t* planes = reinterpret_cast<int8_t*>(p.out);
#pragma unroll
    for (int c = 0; c < NP; ++c) {
      if (c < nv) {
        const float a = fmaxf(fmaxf(red[c], red[NT + c]), fmaxf(red[2 * NT + c], red[3 * NT + c]));
        const float af = fmaxf(a, 1e-30f);
        const float sc = af * (1.0f / kFixMax);
        // |h| <= a and inv is within 2 ulps of kFixMax / a, so |X| <= kFixMax; the fast divide
        // holds for divisors below 2^126
        const float inv = af < 8.5e37f ? __fdividef((float)kFixMax, af) : (float)kFixMax / af;
        const int X = __float2int_rn(P.ag[c] * inv);
        const int h8 = (X + 128) >> 8;
        const size_t o = (size_t)(2 * (I.r0 + c)) * p.out_ld + pos;
        planes[o] = (int8_t)h8;
        planes[o + p.out_ld] = (int8_t)(X - 256 * h8);
        const int sum = __reduce_add_sync(0xffffffffu, X);  // the warp's 32 rows: one 32-group of h's K
        // h's meta: stage I.m / 2, group (I.m & 1) * 4 + ew, block scale 8 + (I.m & 1)
        int32_t* m = p.out_meta + (size_t)(I.r0 + c) * mw_h + (I.m >> 1) * kMetaWords;
        if (lane == 0) m[(I.m & 1) * 4 + ew] = kFixBias - 8 * sum;
        if (mrow == 0) m[8 + (I.m & 1)] = __float_as_int(sc);
      }
    }
    // no second barrier: red[] alternates between two buffers by item, and a warp can write this
    // buffer again (two items on) only after every warp has passed the next item's barrier,
    // that is, after every warp finished the reads above
    return true;
  } else {
#pragma unroll
    for (int mat = 0; mat < NA_; ++mat) {
      const int n = I.m * (NA_ * BM) + mat * BM + mrow;
      if (p.splits > 1) {  // this split's partial sum, reduced in split order by another kernel
        float* y = p.part + (size_t)(it % p.splits) * p.act_rows * p.out_ld;
#pragma unroll
        for (int c = 0; c < NP; ++c)
          if (c < nv) y[(size_t)(I.r0 + c) * p.out_ld + n] = mat ? P.au[c] : P.ag[c];
      } else if (p.out_kind == OUT_F32) {
        float* y = reinterpret_cast<float*>(p.out);
#pragma unroll
        for (int c = 0; c < NP; ++c)
          if (c < nv) y[(size_t)(I.r0 + c) * p.out_ld + n] = mat ? P.au[c] : P.ag[c];
      } else {
        __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(p.out);
#pragma unroll
        for (int c = 0; c < NP; ++c)
          if (c < nv) y[(size_t)(I.r0 + c) * p.out_ld + n] = __float2bfloat16_rn(mat ? P.au[c] : P.ag[c]);
      }
    }
    return true;
  }
}

template <bool GATED, int NA_>
__global__ void __launch_bounds__(kThreads, 1)
    w4i8_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_m, const __grid_constant__ CUtensorMap tm_s,
                     const Params p) {
  using C = Cfg<GATED, NA_>;
  constexpr int NA = C::NA, ST = C::ST, ASL = C::ASLOTS, DSL = C::DSLOTS, SG = C::SG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + ST;
  uint64_t* a_full = empty + ST;
  uint64_t* a_empty = a_full + ASL;
  uint64_t* d_full = a_empty + ASL;
  uint64_t* d_empty = d_full + DSL;
  uint64_t* drain = d_empty + DSL;
  uint64_t* epi_bar = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  Item* items = reinterpret_cast<Item*>(smem + C::OFF_ITEMS);
  int* sprefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&full[i], p.scales_tma ? 1 : 1 + 32);
      // unpack warps (words) and epilogue warps (meta, scales; they finish a stage only after
      // its last MMA completed, so the planes are free too)
      mbar_init(&empty[i], kNumUnpack + 4);
    }
    for (int i = 0; i < ASL; ++i) {
      mbar_init(&a_full[i], kNumUnpack);
      mbar_init(&a_empty[i], 2);  // a commit from each MMA warp
    }
    for (int i = 0; i < DSL; ++i) {
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], 4);
    }
    mbar_init(drain, 2);
    mbar_init(epi_bar, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_m);
    if (p.scales_tma) prefetch_tmap(&tm_s);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
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
  const int total = p.m_tiles * sprefix[p.E] * p.splits;
  const int K = p.K;
  const int nkb = ceil_div(K, KB);

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_b = policy_evict_last();
    const int kg = K / G;
    int s = 0, issued = 0, local = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x, ++local) {
      const Item I = decode_item(it, sprefix, p);
      const int row_g = I.e * p.rows_per_expert + I.m * (GATED ? BM : NA * BM);  // first tile
      const int row_u = row_g + p.row_off2;                                      // second tile
      int kb0, kb1;
      split_range(it, nkb, p.splits, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, abort_flag, lim)))) break;
        uint8_t* st = smem + s * C::STAGE;
        const int natom = min(KB, K - kb * KB) / 128;  // 2, or 1 for a half stage
        if (lane == 0) {
          // the item's entry, released to the promotion warps by this stage's full barrier (its
          // slot was last read for item local - kItemRing, whose stages are all done: the empty
          // wait above)
          if (kb == kb0) items[local & (kItemRing - 1)] = I;
          uint32_t bytes = NA * C::W_TILE + natom * C::B_ATOM + C::META_BYTES;
          if (p.scales_tma) bytes += NA * C::S_TILE;
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d_hint(st, &tm_w, &full[s], kb * (KB / 8), row_g, pol_w);
          if (NA == 2) tma_load_2d_hint(st + C::W_TILE, &tm_w, &full[s], kb * (KB / 8), row_u, pol_w);
          for (int a = 0; a < natom; ++a)
            tma_load_2d_hint(st + C::STAGE_B + a * C::B_ATOM, &tm_x, &full[s], kb * KB + a * 128, 2 * I.r0, pol_b);
          tma_load_2d_hint(st + C::META, &tm_m, &full[s], kb * kMetaWords, I.r0, pol_b);
          if (p.scales_tma) {
            tma_load_2d_hint(st + C::SCL, &tm_s, &full[s], kb * NG, row_g, pol_w);
            if (NA == 2) tma_load_2d_hint(st + C::SCL + C::S_TILE, &tm_s, &full[s], kb * NG, row_u, pol_w);
          }
        }
        if (!p.scales_tma) {  // scale rows 8-byte aligned: 8 or 4 bf16 per row by cp.async
#pragma unroll
          for (int mat = 0; mat < NA; ++mat) {
            const int row0 = mat ? row_u : row_g;
            for (int rr = lane; rr < BM; rr += 32) {
              const uint16_t* src = p.w_s + (size_t)(row0 + rr) * kg + kb * NG;
              uint8_t* dst = st + C::SCL + mat * C::S_TILE + rr * 16;
              cp_async_8(dst, src);
              if (natom == 2) cp_async_8(dst + 8, src + 4);
            }
          }
          cp_async_arrive_noinc(&full[s]);
        }
        ++issued;
        if (++s == ST) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (lane == 0)
      for (int i = max(0, issued - ST); i < issued; ++i) mbar_wait_plain(&full[i % ST], (i / ST) & 1, lim);
  } else if (warp == kMmaWarp || warp == kMmaWarpOdd) {
    // ---------------------------------------------------------------- MMA issuers
    // Warp 1 takes the even D slots, warp 3 the odd ones (a running slot count q), each released
    // by the scheduler warp on its own named barrier; every loop bound is the scheduler's, so
    // both sides take the same barrier steps.
    // u8 A x s8 B -> s32, M = 128, N = DC (NT tokens x (hi, lo))
    const uint32_t idesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(DC >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);
    const int mine = warp == kMmaWarpOdd ? 1 : 0;
    int s = 0, as = 0, ds = 0, q = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      int kb0, kb1;
      split_range(it, nkb, p.splits, kb0, kb1);
      for (int kb = kb0; kb < kb1 && ok; ++kb) {
        const int ng = min(KB, K - kb * KB) / G;
        // descriptors and addresses from per-stage bases plus constants, so that the issue loop
        // between MMAs is a few instructions
        const uint64_t b_base = sw128_kmajor_desc(smem_u32(smem + s * C::STAGE + C::STAGE_B));
        const uint32_t a_slot = tmem_base + (uint32_t)(C::A_COL0 + as * C::A_SLOT);
#pragma unroll
        for (int g0 = 0; g0 < NG; g0 += SG) {
          if (g0 >= ng) break;
          if ((q & 1) == mine) {
            if (!(ok = bar_red_and(kMmaBarrier + mine, 64, true))) break;
            if (lane == 0) {
              tc_fence_after();
              const uint32_t d_slot = tmem_base + (uint32_t)(ds * C::D_SLOT);
#pragma unroll
              for (int gg = 0; gg < SG; ++gg) {
                const int g = g0 + gg;
                if (SG > 4 && g >= ng) break;  // a half stage (4 divides every stage)
                // B atom g/4 (B_ATOM bytes = B_ATOM/16 descriptor units), 32-byte K step within it
                const uint64_t b = b_base + (uint64_t)((g >> 2) * (C::B_ATOM >> 4) + 2 * (g & 3));
#pragma unroll
                for (int mat = 0; mat < NA; ++mat)
                  umma_i8_ts(d_slot + (uint32_t)((gg * NA + mat) * DC), a_slot + (uint32_t)(mat * NG * 8 + g * 8),
                             b, idesc);
              }
              umma_commit(&d_full[ds]);
            }
            __syncwarp();
          }
          ++q;
          if (++ds == DSL) ds = 0;
        }
        if (!ok) break;
        // each MMA warp's commit: the A slot is free once both warps' MMAs of the stage are done
        if (lane == 0) umma_commit(&a_empty[as]);
        __syncwarp();
        if (++as == ASL) as = 0;
        if (++s == ST) s = 0;
      }
    }
    if (lane == 0) {
      umma_commit(drain);
      mbar_wait_plain(drain, 0, lim);
    }
  } else if (warp == kSchedWarp) {
    // ---------------------------------------------------------------- MMA scheduler
    // For each D slot: the stage's copies landed, its A slot is unpacked and the D slot is
    // free; then one named-barrier step releases the slot's MMA warp (false on timeout or
    // abort, after which the other MMA warp, held for the next slot, is released with false).
    int s = 0, as = 0, ds = 0, q = 0;
    uint32_t ph = 0, ph_a = 0, ph_d = 0;
    bool ok = true;

    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      int kb0, kb1;
      split_range(it, nkb, p.splits, kb0, kb1);
      for (int kb = kb0; kb < kb1 && ok; ++kb) {
        const int ng = min(KB, K - kb * KB) / G;
        bool ready = __all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag, lim)) &&
                     __all_sync(0xffffffffu, mbar_wait(&a_full[as], ph_a, abort_flag, lim));
        for (int g0 = 0; g0 < ng; g0 += SG) {
          ready = ready && __all_sync(0xffffffffu, mbar_wait(&d_empty[ds], ph_d ^ 1u, abort_flag, lim));
          if (!(ok = bar_red_and(kMmaBarrier + (q & 1), 64, ready))) {
            // the other MMA warp is held for the next slot, if there is one
            if (g0 + SG < ng || kb + 1 < kb1 || it + (int)gridDim.x < total)
              bar_red_and(kMmaBarrier + ((q + 1) & 1), 64, false);
            break;
          }
          ++q;
          if (++ds == DSL) {
            ds = 0;
            ph_d ^= 1u;
          }
        }
        if (!ok) break;
        if (++as == ASL) {
          as = 0;
          ph_a ^= 1u;
        }
        if (++s == ST) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ---------------------------------------------------------------- promotion + epilogue
    const int ew = warp - kEpiWarp0;  // == warp % 4: TMEM lanes 32*ew..
    const uint32_t lane_base = tmem_base + ((uint32_t)(ew * 32) << 16);
    int ds = 0, s = 0;
    uint32_t ph_d = 0, ph_e = 0, ph = 0;
    bool ok = true;
    for (int it = blockIdx.x, local = 0; it < total && ok; it += gridDim.x, ++local) {
      // the item's first stage has landed, so its entry is published (the same wait opens the
      // K loop below)
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag, lim)))) break;
      const Item I = items[local & (kItemRing - 1)];
      const int nv = I.nvalid;
      float* red_it = red + (local & 1) * (4 * NT);
#define MOE_EPI_ITEM(NP_)                                                                                           \
  epi_item<GATED, NA_, NP_>(p, I, it, ew, lane, lane_base, smem, s, ph, full, empty, ds, ph_d, d_full, d_empty,      \
                            red_it, epi_bar, ph_e, abort_flag)
      if (nv <= 1)
        ok = MOE_EPI_ITEM(1);
      else if (nv <= 2)
        ok = MOE_EPI_ITEM(2);
      else if (nv <= 4)
        ok = MOE_EPI_ITEM(4);
      else
        ok = MOE_EPI_ITEM(8);
#undef MOE_EPI_ITEM
    }
  } else if (warp >= kUnpackWarp0) {
    // ---------------------------------------------------------------- INT4 -> u8 rows of TMEM
    // two tiles: warps 8-11 rows of the first (gate) tile, 12-15 of the second (up), a thread =
    // a row, the whole stage; one tile: a thread = a row and one 128-K half of the stage.
    const int uw = warp - kUnpackWarp0;
    const int row = (uw & 3) * 32 + lane;
    const int sw = row & 7;
    const int mat = NA == 2 ? (uw >> 2) : 0;
    const int half = NA == 2 ? 0 : (uw >> 2);
    constexpr int CHK = NA == 2 ? 8 : 4;  // 16-byte chunks (32 K each) this thread unpacks per stage
    const uint32_t lane_base = tmem_base + ((uint32_t)((uw & 3) * 32) << 16);
    int s = 0, as = 0;
    uint32_t ph = 0, ph_a = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      int kb0, kb1;
      split_range(it, nkb, p.splits, kb0, kb1);
      for (int kb = kb0; kb < kb1 && ok; ++kb) {
        const int ng = min(KB, K - kb * KB) / G;
        ok = __all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag, lim));
        if (!ok) break;
        const uint8_t* wrow = smem + s * C::STAGE + mat * C::W_TILE + row * 128;
        uint4 wv[CHK];
#pragma unroll
        for (int c = 0; c < CHK; ++c) {
          const int lc = NA == 2 ? c : 4 * half + c;  // logical 16-byte chunk = 32-K group
          wv[c] = *reinterpret_cast<const uint4*>(wrow + ((lc ^ sw) << 4));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // words are in registers
        if (++s == ST) {
          s = 0;
          ph ^= 1u;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&a_empty[as], ph_a ^ 1u, abort_flag, lim));
        if (!ok) break;
        tc_fence_after();
        // group g's 32 K = 4 words -> 8 columns of 4 bytes; word w gives K offsets
        // (0,2,4,6) then (1,3,5,7) as offset-binary bytes n = q + 8
        uint32_t r[CHK * 8];
#pragma unroll
        for (int c = 0; c < CHK; ++c) {
          const uint32_t w4[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const uint32_t n = w4[w] ^ 0x88888888u;
            r[c * 8 + 2 * w] = n & 0x0F0F0F0Fu;
            r[c * 8 + 2 * w + 1] = (n >> 4) & 0x0F0F0F0Fu;
          }
        }
        const uint32_t col0 = (uint32_t)(C::A_COL0 + as * C::A_SLOT + mat * NG * 8 + (NA == 2 ? 0 : half * 32));
        if constexpr (NA == 2) {
          uint32_t r0[32], r1[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) r0[i] = r[i], r1[i] = r[32 + i];
          tmem_st32(lane_base + col0, r0);
          if (ng > 4) tmem_st32(lane_base + col0 + 32, r1);
        } else {
          uint32_t r0[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) r0[i] = r[i];
          if (ng > 4 * half) tmem_st32(lane_base + col0, r0);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[as]);
        if (++as == ASL) {
          as = 0;
          ph_a ^= 1u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <bool GATED, int NA_>
cudaError_t launch_t(const W4I8Problem& pr, cudaStream_t s) {
  using C = Cfg<GATED, NA_>;
  CUtensorMap tm_w, tm_x, tm_m, tm_s;
  const uint64_t wrows = (uint64_t)pr.E * pr.rows_per_expert;
  if (encode_tmap_2d(&tm_w, pr.w_q, CU_TENSOR_MAP_DATA_TYPE_INT32, pr.K / 8, wrows, (uint64_t)pr.K / 2, KB / 8, BM,
                     CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tmap_2d(&tm_x, pr.act, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.K, 2 * (uint64_t)pr.act_rows, (uint64_t)pr.K,
                     128, 2 * NT, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int mw = meta_words_per_row(pr.K);
  if (encode_tmap_2d(&tm_m, pr.act_meta, CU_TENSOR_MAP_DATA_TYPE_INT32, mw, (uint64_t)pr.act_rows, (uint64_t)mw * 4,
                     kMetaWords, NT, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int scales_tma = (pr.K % KB) == 0;  // scale rows are then a multiple of 16 bytes
  if (scales_tma) {
    if (encode_tmap_2d(&tm_s, pr.w_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.K / G, wrows, (uint64_t)pr.K / 16, NG, BM,
                       CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    tm_s = tm_w;  // unused
  }
  Params p;
  p.K = pr.K;
  p.scales_tma = scales_tma;
  p.E = pr.E;
  p.rows_per_expert = pr.rows_per_expert;
  p.I = pr.I;
  p.m_tiles = GATED ? pr.I / BM : pr.rows_per_expert / (NA_ * BM);
  p.row_off2 = GATED ? pr.I : BM;
  p.w_s = pr.w_s;
  p.sched = pr.sched;
  p.out_kind = pr.out_kind;
  p.out = pr.out;
  p.out_meta = pr.out_meta;
  p.out_ld = pr.out_ld;
  p.splits = pr.splits > 1 && !GATED ? pr.splits : 1;
  p.part = pr.part;
  p.act_rows = pr.act_rows;
  p.wait_limit = wait_limit_ns();
  const size_t smem = C::smem_bytes(pr.E);
  auto kern = w4i8_gemm_kernel<GATED, NA_>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const char* name = GATED ? "w4i8_gemm_gate_up" : "w4i8_gemm_down";
  timing_before(name, s);
  (void)launch_kernel(kern, dim3(sm_count()), dim3(kThreads), smem, s, tm_w, tm_x, tm_m, tm_s, p);
  timing_after(name, s);
  return cudaGetLastError();
}

}  // namespace w4i8

int w4i8_tiles_per_item(bool gated, int rows_per_expert) { return gated || rows_per_expert % 256 == 0 ? 2 : 1; }

cudaError_t launch_w4i8_gemm(const W4I8Problem& p, cudaStream_t s) {
  if (p.gated) return w4i8::launch_t<true, 2>(p, s);
  return w4i8_tiles_per_item(false, p.rows_per_expert) == 2 ? w4i8::launch_t<false, 2>(p, s)
                                                            : w4i8::launch_t<false, 1>(p, s);
}

}  // namespace moe
