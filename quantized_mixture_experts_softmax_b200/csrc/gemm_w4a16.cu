// a5-a7 for experts with many rows: W4A16 grouped expert GEMM on the 5th-generation tensor
// cores (tcgen05 kind::f16, sm_100a).
//
// One persistent CTA per SM walks a static round-robin list of work items.  An item is
// (expert e, weight tile m of 128 output rows, token tile t of up to NMAX = 192 activation
// rows); the item list is ordered expert-major, then weight tile, then token tile, so that CTAs
// running at the same time share weight tiles through L2 when an expert has several token
// tiles.  The MMA runs "swapped": the 128 weight rows are the M operand and the token rows the
// N operand, N = the item's row count rounded up to 16, chosen per item at run time from the
// expert's actual token count (the Chord article's per-expert scheduling and the Swap-AB
// transposition of the AWS and Helion articles, on tcgen05's M=128 instead of Hopper's 64-row
// WGMMA).
//
// The dequantized weights (the MMA's A operand) live in tensor memory, not shared memory: per
// 64-K step a 128-row fp16 tile staged in shared memory would be written once and read once per
// matrix, which next to the activation tile's copy and two reads asks more of shared memory than
// it delivers; from tensor memory the MMA reads A without touching it.  The accumulators and the
// A ring then share the 512 TMEM columns, which sets the token tile to 192 rows.
//
// Warp roles (512 threads, 544 for the gate/up GEMM):
//   warp 0      TMA producer of the packed INT4 weight tiles (NA x 128 rows x 256 K, 128-byte
//               swizzle) and their bf16 scales (TMA; cp.async when a scale row is not 16-byte
//               aligned), WST-deep ring of 256-K stages;
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer (A from tensor memory, B
//               from shared memory) of the gate (or only) matrix, and for the gate/up GEMM
//   warp 16     the issuer of the up matrix's MMAs: a thread with MMAs in flight stalls at its
//               next synchronisation until they drain, so with one issuer the tensor core idles
//               at every step's hand-off; with two, one's MMAs run while the other waits.  The
//               issuers never wait on an mbarrier (see bar_red_and) and are released step by
//               step by
//   warp 2      the MMA scheduler, which waits for the accumulator, the dequantized A tile and
//               the activation tile of each 64-K step;
//   warp 3      TMA producer of the fp16 activation tiles (N rows x 64 K, boxes of 128, 64, 32
//               and 16 rows), BST-deep ring;
//   warps 4-7   epilogue: tcgen05.ld of the fp32 accumulators, times each row's power-of-two
//               exponent, SiLU(gate)*up for the gate/up GEMM (fp16 h) or a plain store (fp32 /
//               bf16) for the down GEMM;
//   warps 8-15  dequantization: each thread copies its weight row's words and scales of a stage
//               into registers (freeing the stage at once), then per 64-K step writes
//               INT4 -> fp16 = q * s exactly (|q| <= 8 has 3 significant bits, a bf16 scale 8,
//               fp16 holds 11) into an A slot of tensor memory (tcgen05.st), ABUF-deep.
// The gate/up GEMM keeps two accumulators (gate rows m*128.., up rows I+m*128..) so each
// epilogue thread holds gate_j and up_j of the same j.
//
// Every wait is bounded: a stuck pipeline records MOE_ERR_TIMEOUT, releases TMEM and exits.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace w4 {

constexpr int BM = 128;             // weight rows per tile (MMA M)
constexpr int KB = 256;             // K per weight stage
constexpr int KS = 64;              // K per MMA step (one 128-byte swizzle atom of fp16)
constexpr int NMAX = kWideTileRows; // token rows per tile
constexpr int kWProdWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kSchedWarp = 2;
constexpr int kActWarp = 3;
constexpr int kEpiWarp0 = 4;  // warps 4-7: epilogue
constexpr int kDqWarp0 = 8;   // warps 8-15: dequantization
constexpr int kNumDq = 8;
constexpr int kMmaWarpUp = kDqWarp0 + kNumDq;  // warp 16: the second tile's issuer (NA = 2)
template <int NA>
constexpr int threads() { return (kDqWarp0 + kNumDq + (NA == 2 ? 1 : 0)) * 32; }
constexpr int kMmaBarrier = 1;  // named barriers 1 (gate/only) and 2 (up) of an MMA warp and the
                                // scheduler warp (0 is __syncthreads)
static_assert(NMAX % 32 == 0 && NMAX <= 256, "token tile");

// NA_ = 128-row weight tiles per work item: gate and up (gate/up GEMM), or two adjacent tiles
// of the output (down GEMM with rows in 256s: twice the MMAs per 64-K hand-off, whose fixed cost
// made the one-tile down GEMM the less efficient of the two), else one.
template <bool GATED, int NA_>
struct Cfg {
  static_assert(NA_ == 1 || NA_ == 2, "one or two weight tiles per item");
  static_assert(!GATED || NA_ == 2, "gate and up tiles");
  static constexpr int NA = NA_;
  static constexpr int NSUB = KB / KS;               // 64-K steps per weight stage
  static constexpr int W_TILE = BM * KB / 2;         // packed INT4 bytes of one 128-row tile
  static constexpr int S_TILE = BM * (KB / 32) * 2;  // its bf16 scales
  static constexpr int W_STAGE = NA * (W_TILE + S_TILE);
  static constexpr int B_ATOM = NMAX * KS * 2;       // activation tile of one 64-K step
  // ring depths: weight stages, activation tiles, A slots in tensor memory
  static constexpr int WST = NA == 2 ? 3 : 2;
  static constexpr int BST = NA == 2 ? 4 : 7;
  static constexpr int ABUF = NA == 2 ? 2 : 4;
  static constexpr int ACC_COLS = NA * NMAX;         // [matrix][NMAX] fp32 columns
  static constexpr int ACC_BUFS = (2 * ACC_COLS + ABUF * NA * (KS / 2) <= 512) ? 2 : 1;
  static constexpr int A_COLS = KS / 2;              // a 64-K fp16 row of one tile = 32 TMEM columns
  static constexpr int A_COL0 = ACC_BUFS * ACC_COLS; // first TMEM column of the A ring
  static constexpr int OFF_W = 0;
  static constexpr int OFF_B = OFF_W + WST * W_STAGE;
  static constexpr int OFF_BAR = OFF_B + BST * B_ATOM;
  static constexpr int NUM_BARS = 2 * WST + 2 * BST + 2 * ABUF + 2 * ACC_BUFS + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  // per epilogue warp a [16 tokens][32 rows] fp16 staging tile of a 16-column chunk of h, so
  // that each token's 32 values (64 bytes) leave in 16-byte stores
  static constexpr int STG_BYTES = 16 * 32 * 2;
  static constexpr int OFF_STG = (OFF_MISC + 16 + 127) / 128 * 128;  // read as 16-byte vectors
  static_assert(OFF_STG % 16 == 0 && STG_BYTES % 16 == 0, "16-byte aligned staging tiles");
  static constexpr int OFF_PREFIX = OFF_STG + 4 * STG_BYTES;
  static_assert(W_STAGE % 1024 == 0 && W_TILE % 1024 == 0 && OFF_B % 1024 == 0 && B_ATOM % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
  static_assert(A_COL0 + ABUF * NA * A_COLS <= 512, "TMEM has 512 columns");
  // then the tile prefix [E+1] and the epilogue warps' row exponents [4][NMAX]
  static constexpr size_t smem_bytes(int E) { return (size_t)OFF_PREFIX + 4 * (size_t)(E + 1 + 4 * NMAX) + 1024; }
  static_assert(smem_bytes(1024) <= 232448, "shared memory budget");
};

// tensor maps of the activation matrix with boxes of 128, 64, 32 and 16 rows (64 K each)
struct BoxMaps {
  CUtensorMap m[4];
  __device__ const CUtensorMap& operator[](int i) const { return m[i]; }
};

struct Params {
  int K, E, rows_per_expert, I, m_tiles;
  int row_off2;    // NA = 2: rows of the second tile after the first (I for gate/up, 128 for down)
  int scales_tma;  // 1: weight scales by TMA (K % 256 == 0), else by cp.async
  const uint16_t* w_s;
  TileSched sched;
  void* out;
  int out_ld;
  int out_kind;
  int splits;   // K splits per (expert, weight tile, token tile); > 1 only for plain outputs
  float* part;  // splits > 1: fp32 partial sums [splits, act_rows, out_ld]
  int act_rows;
  const int32_t* acc_exp;  // null, or per activation row e: its accumulators are multiplied by 2^e
  int32_t* ovf_flag;       // gated: row r set to 1 when one of its h values was stored prescaled
  uint32_t* ovf_mask;      // gated: [act_rows, out_ld/32] bit per stored h position prescaled by 2^-16
  uint64_t wait_limit;
};

// 2^e as a float for an exponent e in [-126, 127]
__device__ __forceinline__ float exp2_int(int e) { return __int_as_float((127 + e) << 23); }

struct Item {
  int e, m, r0, nvalid, nmma;
};

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
  I.nmma = (I.nvalid + 15) & ~15;
  return I;
}

// bf16 scale number g (0..7) of a 16-byte scale row -> (s, s) in fp16 (exact for the range);
// g is a constant after unrolling, so the selects fold away.
__device__ __forceinline__ __half2 scale_h2(const uint4& sc, int g) {
  const int w2 = g >> 1;
  const uint32_t w = w2 == 0 ? sc.x : w2 == 1 ? sc.y : w2 == 2 ? sc.z : sc.w;
  const uint32_t bits = (g & 1) ? (w & 0xFFFF0000u) : (w << 16);
  return __float2half2_rn(__uint_as_float(bits));
}

__device__ __forceinline__ __half2 h2_bits(uint32_t u) { return *reinterpret_cast<const __half2*>(&u); }
__device__ __forceinline__ uint32_t bits_h2(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }

// One packed word (8 signed nibbles, K offsets 0..7) -> 8 fp16 weights q*s in the order
// (k0,k4,k1,k5,k2,k6,k3,k7).  Flipping a nibble's top bit turns its two's-complement value q
// into q+8 in [0,15]; OR-ing that into the mantissa of 1024.0 (fp16 0x6400) gives 1024+q+8
// (1024+16(q+8) for the nibble held 4 bits higher), from which q follows exactly.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, __half2 s) {
  const uint32_t w8 = w >> 8;
  const uint32_t a = (w & 0x000F000Fu) ^ 0x64086408u;   // 1032+q   : k0, k4
  const uint32_t b = (w & 0x00F000F0u) ^ 0x64806480u;   // 1152+16q : k1, k5
  const uint32_t c = (w8 & 0x000F000Fu) ^ 0x64086408u;  //          : k2, k6
  const uint32_t d = (w8 & 0x00F000F0u) ^ 0x64806480u;  //          : k3, k7
  const __half2 k1032 = h2_bits(0x64086408u);           // (1032, 1032)
  const __half2 k16th = h2_bits(0x2C002C00u);           // (1/16, 1/16)
  const __half2 km72 = h2_bits(0xD480D480u);            // (-72, -72)
  const __half2 qa = __hsub2(h2_bits(a), k1032);
  const __half2 qb = __hfma2(h2_bits(b), k16th, km72);
  const __half2 qc = __hsub2(h2_bits(c), k1032);
  const __half2 qd = __hfma2(h2_bits(d), k16th, km72);
  return make_uint4(bits_h2(__hmul2(qa, s)), bits_h2(__hmul2(qb, s)), bits_h2(__hmul2(qc, s)),
                    bits_h2(__hmul2(qd, s)));
}

// position of column j inside its group of 8 in the interleaved activation layout
__device__ __forceinline__ int interleave_pos(int j) {
  const int r = j & 7;
  return (j & ~7) | (r < 4 ? 2 * r : 2 * (r - 4) + 1);
}

template <bool GATED, int NA_>
__global__ void __launch_bounds__(threads<NA_>(), 1)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                      const __grid_constant__ BoxMaps tm_b, const Params p) {
  using C = Cfg<GATED, NA_>;
  constexpr int NA = C::NA, WST = C::WST, BST = C::BST, ABUF = C::ABUF, ACCB = C::ACC_BUFS, NSUB = C::NSUB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_w = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty_w = full_w + WST;
  uint64_t* full_b = empty_w + WST;
  uint64_t* empty_b = full_b + BST;
  uint64_t* a_full = empty_b + BST;
  uint64_t* a_empty = a_full + ABUF;
  uint64_t* acc_full = a_empty + ABUF;
  uint64_t* acc_empty = acc_full + ACCB;
  uint64_t* drain = acc_empty + ACCB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* sprefix = reinterpret_cast<int*>(smem + C::OFF_PREFIX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit;

  if (threadIdx.x == 0) {
    for (int i = 0; i < WST; ++i) {
      mbar_init(&full_w[i], p.scales_tma ? 1 : 1 + 32);
      mbar_init(&empty_w[i], kNumDq);
    }
    for (int i = 0; i < BST; ++i) {
      mbar_init(&full_b[i], 1);
      mbar_init(&empty_b[i], NA);
    }
    // the A slot, the activation tile and the accumulator are released by a commit of each MMA warp
    for (int i = 0; i < ABUF; ++i) {
      mbar_init(&a_full[i], kNumDq);
      mbar_init(&a_empty[i], NA);
    }
    for (int i = 0; i < ACCB; ++i) {
      mbar_init(&acc_full[i], NA);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain, NA);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_w);
    if (p.scales_tma) prefetch_tmap(&tm_s);
    for (int b = 0; b < 4; ++b) prefetch_tmap(&tm_b[b]);
  }
  if (warp == kMmaWarp) {
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

  if (warp == kWProdWarp) {
    // ---------------------------------------------------------------- weight producer
    const uint64_t pol_w = policy_evict_first();
    const int kg = K / 32;
    int ws = 0, issued = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      const Item I = decode_item(it, sprefix, p);
      const int row_g = I.e * p.rows_per_expert + I.m * (GATED ? BM : NA * BM);  // first tile
      const int row_u = row_g + p.row_off2;                                      // second tile
      int kb0, kb1;
      split_range(it, nkb, p.splits, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&empty_w[ws], ph ^ 1u, abort_flag, lim)))) break;
        uint8_t* st = smem + C::OFF_W + ws * C::W_STAGE;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full_w[ws], (uint32_t)(NA * C::W_TILE + (p.scales_tma ? NA * C::S_TILE : 0)));
          tma_load_2d_hint(st, &tm_w, &full_w[ws], kb * (KB / 8), row_g, pol_w);
          if (NA == 2) tma_load_2d_hint(st + C::W_TILE, &tm_w, &full_w[ws], kb * (KB / 8), row_u, pol_w);
          if (p.scales_tma) {
            tma_load_2d_hint(st + NA * C::W_TILE, &tm_s, &full_w[ws], kb * (KB / 32), row_g, pol_w);
            if (NA == 2)
              tma_load_2d_hint(st + NA * C::W_TILE + C::S_TILE, &tm_s, &full_w[ws], kb * (KB / 32), row_u, pol_w);
          }
        }
        if (!p.scales_tma) {  // scale rows 8-byte aligned: 8 or 4 bf16 per row by cp.async
          const int ngrp = min(KB, K - kb * KB) / 32;
#pragma unroll
          for (int mat = 0; mat < NA; ++mat) {
            const int row0 = mat ? row_u : row_g;
            for (int rr = lane; rr < BM; rr += 32) {
              const uint16_t* src = p.w_s + (size_t)(row0 + rr) * kg + kb * (KB / 32);
              uint8_t* dst = st + NA * C::W_TILE + mat * C::S_TILE + rr * 16;
              cp_async_8(dst, src);
              if (ngrp > 4) cp_async_8(dst + 8, src + 4);
            }
          }
          cp_async_arrive_noinc(&full_w[ws]);
        }
        ++issued;
        if (++ws == WST) {
          ws = 0;
          ph ^= 1u;
        }
      }
    }
    if (lane == 0)
      for (int i = max(0, issued - WST); i < issued; ++i) mbar_wait_plain(&full_w[i % WST], (i / WST) & 1, lim);
  } else if (warp == kMmaWarp || (NA == 2 && warp == kMmaWarpUp)) {
    // ---------------------------------------------------------------- MMA issuers
    // One per matrix, each released step by step by the scheduler warp on its own named barrier;
    // identical loop bounds on all three sides.
    const int mat = warp == kMmaWarp ? 0 : 1;
    int ab = 0, bs = 0, acc = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      const Item I = decode_item(it, sprefix, p);
      const uint32_t idesc = make_idesc(BM, I.nmma, 0, 0);
      const uint32_t d = tmem_base + (uint32_t)(acc * C::ACC_COLS + mat * NMAX);  // [matrix][NMAX] columns
      int kb0, kb1;
      split_range(it, nkb, p.splits, kb0, kb1);
      for (int kb = kb0; kb < kb1 && ok; ++kb) {
        const int nsub = min(NSUB, (K - kb * KB) / KS);
        for (int j = 0; j < nsub; ++j) {
          if (!(ok = bar_red_and(kMmaBarrier + mat, 64, true))) break;
          if (lane == 0) {
            tc_fence_after();
            const uint64_t b = sw128_kmajor_desc(smem_u32(smem + C::OFF_B + bs * C::B_ATOM));
            const uint32_t a0 = tmem_base + (uint32_t)(C::A_COL0 + (ab * NA + mat) * C::A_COLS);
#pragma unroll
            for (int kk = 0; kk < KS / 16; ++kk) {
              const uint32_t accum = (kb != kb0) || j != 0 || kk != 0;  // fresh at the split's first K
              // 16 K = 8 TMEM columns of A, 32 bytes of the activation atom
              umma_f16_ts(d, a0 + 8 * kk, b + 2 * kk, idesc, accum);
            }
            umma_commit(&a_empty[ab]);
            umma_commit(&empty_b[bs]);
          }
          __syncwarp();
          if (++ab == ABUF) ab = 0;
          if (++bs == BST) bs = 0;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&acc_full[acc]);
      __syncwarp();
      if (++acc == ACCB) acc = 0;
    }
    if (lane == 0) {
      umma_commit(drain);  // all MMAs issued by this thread have completed once this fires
      mbar_wait_plain(drain, 0, lim);
    }
  } else if (warp == kSchedWarp) {
    // ---------------------------------------------------------------- MMA scheduler
    // Per 64-K step: the item's accumulator is free (first step), the dequantized A tile and
    // the activation tile have landed; then one named-barrier step releases the MMA warp.
    int ab = 0, bs = 0, acc = 0;
    uint32_t ph_a = 0, ph_b = 0, ph_acc = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      bool ready = __all_sync(0xffffffffu, mbar_wait(&acc_empty[acc], ph_acc ^ 1u, abort_flag, lim));
      int kb0, kb1;
      split_range(it, nkb, p.splits, kb0, kb1);
      for (int kb = kb0; kb < kb1 && ok; ++kb) {
        const int nsub = min(NSUB, (K - kb * KB) / KS);
        for (int j = 0; j < nsub; ++j) {
          ready = ready && __all_sync(0xffffffffu, mbar_wait(&a_full[ab], ph_a, abort_flag, lim)) &&
                  __all_sync(0xffffffffu, mbar_wait(&full_b[bs], ph_b, abort_flag, lim));
          ok = bar_red_and(kMmaBarrier, 64, ready);
          if (NA == 2) bar_red_and(kMmaBarrier + 1, 64, ok);  // the second issuer takes the same step
          if (!ok) break;
          if (++ab == ABUF) {
            ab = 0;
            ph_a ^= 1u;
          }
          if (++bs == BST) {
            bs = 0;
            ph_b ^= 1u;
          }
        }
      }
      if (!ok) break;
      if (++acc == ACCB) {
        acc = 0;
        ph_acc ^= 1u;
      }
    }
  } else if (warp == kActWarp) {
    // ---------------------------------------------------------------- activation producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      const int nks = K / KS;
      int bs = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
        const Item I = decode_item(it, sprefix, p);
        int kb0, kb1;
        split_range(it, nkb, p.splits, kb0, kb1);
        const int ks1 = min(nks, kb1 * (KB / KS));
        for (int ks = kb0 * (KB / KS); ks < ks1; ++ks) {
          if (!(ok = mbar_wait(&empty_b[bs], ph ^ 1u, abort_flag, lim))) break;
          mbar_arrive_expect_tx(&full_b[bs], (uint32_t)(I.nmma * KS * 2));
          // boxes of 128, 64, 32 and 16 rows, largest first (at most 4 copies per tile)
          uint8_t* dst = smem + C::OFF_B + bs * C::B_ATOM;
          int r = 0;
          for (int b = 0; b < 4; ++b) {
            const int h = 128 >> b;
            for (; r + h <= I.nmma; r += h) tma_load_2d_hint(dst + r * 128, &tm_b[b], &full_b[bs], ks * KS, I.r0 + r, pol);
          }
          ++issued;
          if (++bs == BST) {
            bs = 0;
            ph ^= 1u;
          }
        }
      }
      for (int i = max(0, issued - BST); i < issued; ++i) mbar_wait_plain(&full_b[i % BST], (i / BST) & 1, lim);
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ---------------------------------------------------------------- epilogue
    // Per chunk of 16 token columns the arithmetic of all 16 values is done first and the stores
    // after it, with the rare h beyond fp16 handled out of line, so that the 16 independent
    // SiLU chains overlap their latencies (one per thread at a time took ~10x longer).
    const int ew = warp - kEpiWarp0;  // == warp % 4: this warp may read TMEM lanes 32*ew..32*ew+31
    const int mrow = ew * 32 + lane;
    int* rexp = sprefix + p.E + 1 + ew * NMAX;  // this warp's copy of the item's row exponents
    uint8_t* stg = smem + C::OFF_STG + ew * C::STG_BYTES;
    int acc = 0;
    uint32_t ph = 0;
    for (int it = blockIdx.x; it < total; it += gridDim.x) {
      const Item I = decode_item(it, sprefix, p);
      // the item's row exponents, loaded while the MMAs run (almost always all 0: then the
      // accumulators need no scaling)
      int nz = 0;
      if (p.acc_exp)
        for (int rr = lane; rr < I.nmma; rr += 32) {
          const int e = rr < I.nvalid ? __ldg(p.acc_exp + I.r0 + rr) : 0;
          rexp[rr] = e;
          nz |= e;
        }
      const bool scale_rows = __any_sync(0xffffffffu, nz != 0);
      __syncwarp();
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[acc], ph, abort_flag, lim))) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(ew * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
      const int col = I.m * BM + mrow;
      for (int c0 = 0; c0 < I.nmma; c0 += 16) {
        uint32_t g[16], u[16];
        tmem_ld16(tb + c0, g);
        if (NA == 2) tmem_ld16(tb + NMAX + c0, u);
        tmem_ld_wait();
        const int nv = min(16, I.nvalid - c0);
        if (scale_rows) {  // rows whose fp16 operand was scaled by 2^-e to fit fp16: undo it
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float sc = exp2_int(rexp[c0 + i]);  // the same word for every lane: a broadcast
            g[i] = __float_as_uint(__uint_as_float(g[i]) * sc);
            if (NA == 2) u[i] = __float_as_uint(__uint_as_float(u[i]) * sc);
          }
        }
        if (GATED) {
          const int pos = interleave_pos(col);
          __half* out = reinterpret_cast<__half*>(p.out) + (size_t)(I.r0 + c0) * p.out_ld + pos;
          float hv[16];
          bool over = false;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float gv = __uint_as_float(g[i]), uv = __uint_as_float(u[i]);
            hv[i] = __fdividef(gv, 1.0f + __expf(-gv)) * uv;  // SiLU(g) * u; fp16 rounding follows
            over |= i < nv && !(fabsf(hv[i]) < 65520.0f);
          }
          if (!__any_sync(0xffffffffu, over)) {
            // the warp's 32 rows are 32 consecutive positions of h: transpose through shared
            // memory, then each token's 64 bytes leave as four 16-byte stores
            __half* sh = reinterpret_cast<__half*>(stg);
#pragma unroll
            for (int i = 0; i < 16; ++i) sh[i * 32 + (pos & 31)] = __float2half_rn(hv[i]);
            __syncwarp();
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int i = (lane >> 2) + 8 * h2, q = lane & 3;
              if (i < nv)
                *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(p.out) + (size_t)(I.r0 + c0 + i) * p.out_ld +
                                          (pos & ~31) + q * 8) = *reinterpret_cast<const uint4*>(sh + i * 32 + q * 8);
            }
            __syncwarp();
          } else {
            bool huge = false;  // an h beyond even the prescaled fp16 range (2^32)
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (i < nv) {
                if (fabsf(hv[i]) < 65520.0f) {
                  out[(size_t)i * p.out_ld] = __float2half_rn(hv[i]);
                } else {  // beyond fp16: stored as h * 2^-16 and marked; h_rescale fixes its row
                  const int r = I.r0 + c0 + i;
                  out[(size_t)i * p.out_ld] = __float2half_rn(hv[i] * (1.0f / 65536.0f));
                  atomicOr(p.ovf_mask + (size_t)r * (p.out_ld / 32) + pos / 32, 1u << (pos & 31));
                  p.ovf_flag[r] = 1;
                  huge |= !(fabsf(hv[i]) < 65520.0f * 65536.0f);
                }
              }
            }
            if (huge) set_status(MOE_ERR_DEVICE_CHECK);
          }
        } else {
          // plain output: the item's NA tiles, output columns m * NA * 128 + mat * 128 + row
#pragma unroll
          for (int mat = 0; mat < NA; ++mat) {
            const uint32_t* v = mat ? u : g;
            const int ncol = I.m * (NA * BM) + mat * BM + mrow;
            if (p.splits > 1) {  // this split's partial sum, reduced in split order by another kernel
              float* out =
                  p.part + (size_t)(it % p.splits) * p.act_rows * p.out_ld + (size_t)(I.r0 + c0) * p.out_ld + ncol;
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (i < nv) out[(size_t)i * p.out_ld] = __uint_as_float(v[i]);
            } else if (p.out_kind == OUT_F32) {
              // a warp's store writes 32 consecutive floats (a whole 128-byte line) per token;
              // staging these through shared memory as for h measured 10% slower
              float* out = reinterpret_cast<float*>(p.out) + (size_t)(I.r0 + c0) * p.out_ld + ncol;
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (i < nv) out[(size_t)i * p.out_ld] = __uint_as_float(v[i]);
            } else {
              __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)(I.r0 + c0) * p.out_ld + ncol;
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (i < nv) out[(size_t)i * p.out_ld] = __float2bfloat16_rn(__uint_as_float(v[i]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == ACCB) {
        acc = 0;
        ph ^= 1u;
      }
    }
  } else if (warp >= kDqWarp0 && warp < kDqWarp0 + kNumDq) {
    // ---------------------------------------------------------------- dequantization -> TMEM
    // GATED: thread = one row of the gate (warps 8-11) or up (warps 12-15) tile, all 64 K of
    // each step (8 words -> 32 TMEM columns); plain: thread = one row and one 32-K half of each
    // step (warps 8-11 the first half, 12-15 the second; 4 words -> 16 columns).  Warp 8 + q
    // and 12 + q write TMEM lanes 32q .. 32q+31, the rows they own.
    const int dw = warp - kDqWarp0;
    const int row = (dw & 3) * 32 + lane;
    const int sw = row & 7;
    const int mat = NA == 2 ? (dw >> 2) : 0;
    const int half = NA == 2 ? 0 : (dw >> 2);
    constexpr int CHK = NA == 2 ? 8 : 4;  // 16-byte chunks of packed words this thread takes per stage
    const uint32_t lane_base = tmem_base + ((uint32_t)((dw & 3) * 32) << 16);
    int ws = 0, ab = 0;
    uint32_t ph_w = 0, ph_a = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      int kb0, kb1;
      split_range(it, nkb, p.splits, kb0, kb1);
      for (int kb = kb0; kb < kb1 && ok; ++kb) {
        ok = __all_sync(0xffffffffu, mbar_wait(&full_w[ws], ph_w, abort_flag, lim));
        if (!ok) break;
        const uint8_t* st = smem + C::OFF_W + ws * C::W_STAGE;
        const uint8_t* wrow = st + mat * C::W_TILE + row * 128;
        const uint4 sc = *reinterpret_cast<const uint4*>(st + NA * C::W_TILE + mat * C::S_TILE + row * 16);
        uint4 wv[CHK];
#pragma unroll
        for (int c = 0; c < CHK; ++c) {
          const int lc = NA == 2 ? c : 2 * c + half;  // logical 16-byte chunk (32 K) of the stage
          wv[c] = *reinterpret_cast<const uint4*>(wrow + ((lc ^ sw) << 4));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_w[ws]);  // words and scales are in registers
        if (++ws == WST) {
          ws = 0;
          ph_w ^= 1u;
        }
        const int nsub = min(NSUB, (K - kb * KB) / KS);
#pragma unroll
        for (int j = 0; j < NSUB; ++j) {
          if (j < nsub) {
            ok = __all_sync(0xffffffffu, mbar_wait(&a_empty[ab], ph_a ^ 1u, abort_flag, lim));
            if (!ok) break;
            tc_fence_after();  // the MMAs that last read this A slot have completed
            const uint32_t col = (uint32_t)(C::A_COL0 + (ab * NA + mat) * C::A_COLS);
            if constexpr (NA == 2) {
              uint32_t r[32];
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const uint4 w = wv[2 * j + q];
                const __half2 s2 = scale_h2(sc, 2 * j + q);
                const uint4 d0 = dequant_word(w.x, s2), d1 = dequant_word(w.y, s2);
                const uint4 d2 = dequant_word(w.z, s2), d3 = dequant_word(w.w, s2);
                const uint32_t v[16] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w,
                                        d2.x, d2.y, d2.z, d2.w, d3.x, d3.y, d3.z, d3.w};
#pragma unroll
                for (int i = 0; i < 16; ++i) r[16 * q + i] = v[i];
              }
              tmem_st32(lane_base + col, r);
            } else {
              const uint4 w = wv[j];
              const __half2 s2 = scale_h2(sc, 2 * j + half);
              const uint4 d0 = dequant_word(w.x, s2), d1 = dequant_word(w.y, s2);
              const uint4 d2 = dequant_word(w.z, s2), d3 = dequant_word(w.w, s2);
              const uint32_t r[16] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w,
                                      d2.x, d2.y, d2.z, d2.w, d3.x, d3.y, d3.z, d3.w};
              tmem_st16(lane_base + col + 16 * half, r);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[ab]);
            if (++ab == ABUF) {
              ab = 0;
              ph_a ^= 1u;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <bool GATED, int NA_>
cudaError_t launch_t(const W4GemmProblem& pr, cudaStream_t s) {
  using C = Cfg<GATED, NA_>;
  CUtensorMap tm_w, tm_s;
  BoxMaps tm_b;
  const uint64_t wrows = (uint64_t)pr.E * pr.rows_per_expert;
  if (encode_tmap_2d(&tm_w, pr.w_q, CU_TENSOR_MAP_DATA_TYPE_INT32, pr.K / 8, wrows, (uint64_t)pr.K / 2, KB / 8, BM,
                     CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int scales_tma = (pr.K % KB) == 0;  // scale rows are then a multiple of 16 bytes
  if (scales_tma) {
    if (encode_tmap_2d(&tm_s, pr.w_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, pr.K / 32, wrows, (uint64_t)pr.K / 16, KB / 32,
                       BM, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    tm_s = tm_w;  // unused
  }
  for (int b = 0; b < 4; ++b)
    if (encode_tmap_2d(&tm_b.m[b], pr.act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, pr.K, (uint64_t)pr.act_rows,
                       (uint64_t)pr.K * 2, KS, 128 >> b, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  Params p;
  p.K = pr.K;
  p.E = pr.E;
  p.rows_per_expert = pr.rows_per_expert;
  p.I = pr.I;
  p.m_tiles = GATED ? pr.I / BM : pr.rows_per_expert / (NA_ * BM);
  p.row_off2 = GATED ? pr.I : BM;
  p.scales_tma = scales_tma;
  p.w_s = pr.w_s;
  p.sched = pr.sched;
  p.out = pr.out;
  p.out_ld = pr.out_ld;
  p.out_kind = pr.out_kind;
  p.splits = pr.splits > 1 && !GATED ? pr.splits : 1;
  p.part = pr.part;
  p.act_rows = pr.act_rows;
  p.acc_exp = pr.acc_exp;
  p.ovf_flag = pr.ovf_flag;
  p.ovf_mask = pr.ovf_mask;
  if (GATED && (!p.ovf_flag || !p.ovf_mask)) return cudaErrorInvalidValue;
  p.wait_limit = wait_limit_ns();
  const size_t smem = C::smem_bytes(pr.E);
  auto kern = w4a16_gemm_kernel<GATED, NA_>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const char* name = GATED ? "w4a16_gemm_gate_up" : "w4a16_gemm_down";
  timing_before(name, s);
  (void)launch_kernel(kern, dim3(sm_count()), dim3(threads<NA_>()), smem, s, tm_w, tm_s, tm_b, p);
  timing_after(name, s);
  return cudaGetLastError();
}

}  // namespace w4

int w4a16_tiles_per_item(int rows) { return rows % 256 == 0 ? 2 : 1; }

cudaError_t launch_w4a16_gemm(const W4GemmProblem& p, cudaStream_t s) {
  if (p.nmax > w4::NMAX) return cudaErrorInvalidValue;
  if (p.gated) return w4::launch_t<true, 2>(p, s);
  return w4a16_tiles_per_item(p.rows_per_expert) == 2 ? w4::launch_t<false, 2>(p, s) : w4::launch_t<false, 1>(p, s);
}

}  // namespace moe
