// a5-a7: W4A16 grouped expert GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// One persistent CTA per SM walks a static round-robin list of work items.  An item is
// (expert e, weight tile m of 128 output rows, token tile t of up to NMAX activation rows);
// the item list is ordered expert-major, then weight tile, then token tile, so that CTAs
// running at the same time share weight tiles through L2 when an expert has several token
// tiles.  The MMA runs "swapped": the 128 weight rows are the M operand and the (thin) token
// rows the N operand, N = the item's row count rounded up to 16, chosen per item at run time
// from the expert's actual token count (the Chord article's per-expert scheduling and the
// Swap-AB transposition of the AWS and Helion articles, on tcgen05's M=128 instead of
// Hopper's 64-row WGMMA).
//
// Warp roles (512 threads):
//   warp 0      TMA producer of the packed INT4 weight tiles (128 rows x 256 K, 128-byte
//               swizzle) plus cp.async of their bf16 group scales, WST-deep ring;
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer;
//   warp 2      TMA producer of the fp16 activation tiles (N rows x 64 K), BST-deep ring;
//   warps 4-7   epilogue: tcgen05.ld of the fp32 accumulators, SiLU(gate)*up for the gate/up
//               GEMM (fp16 h) or a plain store (fp32 / bf16) for the down GEMM;
//   warps 8-15  dequantization: INT4 -> fp16 = q * s exactly (|q| <= 8 has 3 significant
//               bits, a bf16 scale 8, fp16 holds 11), written in the 128-byte swizzled K-major
//               layout the MMA reads, double buffered per 64-K step.
// The gate/up GEMM keeps two accumulators (gate rows m*128.., up rows I+m*128..) so each
// epilogue thread holds gate_j and up_j of the same j.
//
// Every wait is bounded: a stuck pipeline records MOE_ERR_TIMEOUT, releases TMEM and exits.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace w4 {

constexpr int BM = 128;  // weight rows per tile (MMA M)
constexpr int KB = 256;  // K per weight stage
constexpr int KS = 64;   // K per MMA step (one 128-byte swizzle atom of fp16)
constexpr int kEpiWarp0 = 4;  // warps 4-7: epilogue
constexpr int kDqWarp0 = 8;   // warps 8..: dequantization

__host__ __device__ constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

// Two variants by token-tile height:
//  thin (at most kThinN rows, decode-sized experts): the activation tile of each 256-K weight
//    stage travels in that stage, so it is prefetched as deep as the weights;
//  wide (up to 256 rows): activations have their own ring of 64-K tiles (a 256-row tile of
//    256 K would not fit next to the weights).
// Depths: (weight stages, activation stages [wide only], dequantized-A buffers).
#ifndef MOE_W4_THIN_N
#define MOE_W4_THIN_N 16
#endif
#ifndef MOE_W4_GT
#define MOE_W4_GT 5, 0, 3
#endif
#ifndef MOE_W4_PT
#define MOE_W4_PT 8, 0, 6
#endif
#ifndef MOE_W4_GW
#define MOE_W4_GW 2, 2, 2
#endif
#ifndef MOE_W4_PW
#define MOE_W4_PW 4, 3, 2
#endif
constexpr int kThinN = MOE_W4_THIN_N;
struct Depths {
  int wst, bst, abuf;
};
template <bool GATED, bool THIN>
constexpr Depths depths() {
  return GATED ? (THIN ? Depths{MOE_W4_GT} : Depths{MOE_W4_GW}) : (THIN ? Depths{MOE_W4_PT} : Depths{MOE_W4_PW});
}

template <bool GATED, int NMAX>
struct Cfg {
  static constexpr bool THIN = NMAX <= kThinN;
  // thin: the dequantized A operand goes to tensor memory (tcgen05.st by the dequant warps,
  // read by the MMA as its A operand), which leaves room for a deep A ring; wide: the
  // accumulators fill tensor memory, so A is staged in shared memory.
  static constexpr bool A_TMEM = THIN;
  static constexpr int NA = GATED ? 2 : 1;
  // Dependent tcgen05.mma on one accumulator serialise on the MMA latency when N is small;
  // the thin variant spreads each matrix's K steps over CH independent accumulators (summed
  // in the epilogue) so that 4 MMAs are in flight.
  static constexpr int CH = THIN ? 4 / NA : 1;
#ifndef MOE_W4_THIN_DQ
#define MOE_W4_THIN_DQ 8
#endif
  static constexpr int NDQ = THIN ? MOE_W4_THIN_DQ : 8;  // dequantization warps
  // thin: each thread dequantizes one row and 1/PARTS of every 64-K step
  static constexpr int PARTS = THIN ? NDQ / (4 * NA) : 1;
  static_assert(!THIN || (PARTS >= 1 && 8 % PARTS == 0 && NDQ == 4 * NA * PARTS), "thin dequant split");
  static constexpr int THREADS = (kDqWarp0 + NDQ) * 32;
  static constexpr int WST = depths<GATED, THIN>().wst;
  static constexpr int BST = THIN ? 0 : depths<GATED, THIN>().bst;
  static constexpr int ABUF = depths<GATED, THIN>().abuf;
  static constexpr int NSUB = KB / KS;               // 64-K steps per weight stage
  static constexpr int W_TILE = BM * KB / 2;         // packed INT4 bytes
  static constexpr int S_TILE = BM * (KB / 32) * 2;  // bf16 scales
  static constexpr int A_TILE = BM * KS * 2;         // dequantized fp16 operand
  static constexpr int B_ATOM = NMAX * KS * 2;       // activation tile of one 64-K step
  static constexpr int STAGE_W = 0;
  static constexpr int STAGE_S = NA * W_TILE;
  static constexpr int STAGE_B = STAGE_S + NA * S_TILE;
  static constexpr int STAGE = STAGE_B + (THIN ? NSUB * B_ATOM : 0);
  static constexpr int ACC_COLS = NA * CH * NMAX;
  static constexpr int ACC_BUFS = (2 * ACC_COLS <= 512) ? 2 : 1;
  static constexpr int A_COLS = KS / 2;                 // one 64-K fp16 row = 32 TMEM columns
  // thin: an A slot holds SPS consecutive 64-K steps of every matrix, handed over with one
  // barrier round trip and one commit
  static constexpr int SPS = A_TMEM ? 2 : 1;
  static constexpr int SLOT_COLS = NA * SPS * A_COLS;   // [matrix][step][32 columns]
  static constexpr int A_COL0 = ACC_BUFS * ACC_COLS;    // first TMEM column of the A ring
  static constexpr int TMEM_COLS = pow2_at_least(A_COL0 + (A_TMEM ? ABUF * SLOT_COLS : 0));
  static constexpr int OFF_A = WST * STAGE;
  static constexpr int OFF_B = OFF_A + (A_TMEM ? 0 : ABUF * NA * A_TILE);  // wide activation ring
  static constexpr int OFF_BAR = OFF_B + BST * B_ATOM;
  static constexpr int NUM_BARS = 2 * WST + 2 * BST + 2 * ABUF + 2 * ACC_BUFS + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_PREFIX = OFF_MISC + 16;
  static_assert(STAGE % 1024 == 0 && STAGE_B % 1024 == 0 && OFF_A % 1024 == 0 && OFF_B % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
  static_assert(A_COL0 + (A_TMEM ? ABUF * SLOT_COLS : 0) <= 512, "TMEM has 512 columns");
  static_assert(NSUB % SPS == 0, "whole slots per stage");
  static constexpr size_t smem_bytes(int E) { return (size_t)OFF_PREFIX + 4 * (size_t)(E + 1) + 1024; }
  static_assert(smem_bytes(1024) <= 232448, "shared memory budget");
  static_assert(!THIN || A_TMEM, "the thin variant keeps A in tensor memory");
};

struct Params {
  int K, E, rows_per_expert, I, m_tiles;
  int scales_tma;  // 1: scales arrive by TMA (K % 256 == 0), else by cp.async
  const uint16_t* w_s;
  TileSched sched;
  void* out;
  int out_ld;
  int out_kind;
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

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

// position of column j inside its group of 8 in the interleaved activation layout
__device__ __forceinline__ int interleave_pos(int j) {
  const int r = j & 7;
  return (j & ~7) | (r < 4 ? 2 * r : 2 * (r - 4) + 1);
}

template <bool GATED, int NMAX>
__global__ void __launch_bounds__(Cfg<GATED, NMAX>::THREADS, 1)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                      const __grid_constant__ CUtensorMap tm_b, const Params p) {
  using C = Cfg<GATED, NMAX>;
  constexpr bool THIN = C::THIN;
  constexpr int NA = C::NA, WST = C::WST, BST = C::BST, ABUF = C::ABUF, ACCB = C::ACC_BUFS, NSUB = C::NSUB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_w = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty_w = full_w + WST;
  uint64_t* full_b = empty_w + WST;  // wide variant only
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

  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) sprefix[i] = __ldg(p.sched.tile_prefix + i);
  if (threadIdx.x == 0) {
    for (int i = 0; i < WST; ++i) {
      // full: the expect_tx arrival (+ one cp.async arrival per producer lane when scales
      // come by cp.async); empty: the dequant warps (+ the MMA commit when the stage also
      // holds the activation tile)
      mbar_init(&full_w[i], p.scales_tma ? 1 : 1 + 32);
      mbar_init(&empty_w[i], C::NDQ + (THIN ? 1 : 0));
    }
    for (int i = 0; i < BST; ++i) {
      mbar_init(&full_b[i], 1);
      mbar_init(&empty_b[i], 1);
    }
    for (int i = 0; i < ABUF; ++i) {
      mbar_init(&a_full[i], C::NDQ);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < ACCB; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_w);
    if (p.scales_tma) prefetch_tmap(&tm_s);
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = p.m_tiles * sprefix[p.E];
  const int K = p.K;
  const int nkb = ceil_div(K, KB);

  if (warp == 0) {
    // ---------------------------------------------------------------- weight (+ activation) producer
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_b = policy_evict_last();
    const int kg = K / 32;
    int ws = 0, issued = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
      const Item I = decode_item(it, sprefix, p);
      const int row_g = I.e * p.rows_per_expert + I.m * BM;
      const int row_u = row_g + p.I;
      for (int kb = 0; kb < nkb; ++kb) {
        ok = __all_sync(0xffffffffu, mbar_wait(&empty_w[ws], ph ^ 1u, abort_flag, lim));
        if (!ok) break;
        uint8_t* st = smem + ws * C::STAGE;
        const int nsub = min(NSUB, (K - kb * KB) / KS);
        if (lane == 0) {
          uint32_t bytes = NA * C::W_TILE + (p.scales_tma ? NA * C::S_TILE : 0);
          if (THIN) bytes += (uint32_t)(nsub * I.nmma * KS * 2);
          mbar_arrive_expect_tx(&full_w[ws], bytes);
          tma_load_2d_hint(st + C::STAGE_W, &tm_w, &full_w[ws], kb * (KB / 8), row_g, pol_w);
          if (GATED) tma_load_2d_hint(st + C::STAGE_W + C::W_TILE, &tm_w, &full_w[ws], kb * (KB / 8), row_u, pol_w);
          if (p.scales_tma) {
            tma_load_2d_hint(st + C::STAGE_S, &tm_s, &full_w[ws], kb * (KB / 32), row_g, pol_w);
            if (GATED) tma_load_2d_hint(st + C::STAGE_S + C::S_TILE, &tm_s, &full_w[ws], kb * (KB / 32), row_u, pol_w);
          }
          if (THIN) {
            for (int j = 0; j < nsub; ++j)
              for (int r = 0; r < I.nmma; r += 16)
                tma_load_2d_hint(st + C::STAGE_B + j * C::B_ATOM + r * 128, &tm_b, &full_w[ws], kb * KB + j * KS,
                                 I.r0 + r, pol_b);
          }
        }
        if (!p.scales_tma) {
          const int ng = min(8, kg - kb * 8);  // 4 or 8: K is a multiple of 128
#pragma unroll
          for (int mat = 0; mat < NA; ++mat) {
            const int row0 = mat ? row_u : row_g;
#pragma unroll
            for (int rr = lane; rr < BM; rr += 32) {
              const uint16_t* src = p.w_s + (size_t)(row0 + rr) * kg + kb * 8;
              uint8_t* dst = st + C::STAGE_S + mat * C::S_TILE + rr * 16;
              cp_async_8(dst, src);
              if (ng == 8) cp_async_8(dst + 8, src + 4);
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
    // let every copy this warp issued land before the CTA can exit
    for (int i = max(0, issued - WST); i < issued; ++i) mbar_wait_plain(&full_w[i % WST], (i / WST) & 1, lim);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int ab = 0, bs = 0, acc = 0, ws = 0;
      uint32_t ph_a = 0, ph_b = 0, ph_acc = 0, ph_w = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
        const Item I = decode_item(it, sprefix, p);
        const uint32_t idesc = make_idesc(BM, I.nmma, 0, 0);
        if (!(ok = mbar_wait(&acc_empty[acc], ph_acc ^ 1u, abort_flag, lim))) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * C::ACC_COLS);  // [matrix][chain][NMAX] columns
        const uint32_t d1 = d0 + C::CH * NMAX;
        for (int kb = 0; kb < nkb && ok; ++kb) {
          const int nsub = min(NSUB, (K - kb * KB) / KS);
          if (THIN && !(ok = mbar_wait(&full_w[ws], ph_w, abort_flag, lim))) break;
          for (int j = 0; j < nsub; j += C::SPS) {
            if (!(ok = mbar_wait(&a_full[ab], ph_a, abort_flag, lim))) break;
            if (!THIN && !(ok = mbar_wait(&full_b[bs], ph_b, abort_flag, lim))) break;
            tc_fence_after();
            if constexpr (C::A_TMEM) {
              constexpr int CH = C::CH;
              const uint32_t slot = tmem_base + (uint32_t)(C::A_COL0 + ab * C::SLOT_COLS);
#pragma unroll
              for (int s2 = 0; s2 < C::SPS; ++s2) {
                const uint64_t b = sw128_kmajor_desc(smem_u32(smem + ws * C::STAGE + C::STAGE_B + (j + s2) * C::B_ATOM));
#pragma unroll
                for (int kk = 0; kk < KS / 16; ++kk) {
                  const uint32_t accum = (kb | j | s2 | (kk / CH)) != 0;  // each chain starts fresh at K = 0
                  const uint32_t dc = d0 + (uint32_t)((kk % CH) * NMAX);
                  const uint32_t a = slot + (uint32_t)(s2 * C::A_COLS + 8 * kk);  // 16 K = 8 columns
                  umma_f16_ts(dc, a, b + 2 * kk, idesc, accum);
                  if (GATED) umma_f16_ts(dc + CH * NMAX, a + C::SPS * C::A_COLS, b + 2 * kk, idesc, accum);
                }
              }
            } else {
              const uint8_t* bt = THIN ? smem + ws * C::STAGE + C::STAGE_B + j * C::B_ATOM : smem + C::OFF_B + bs * C::B_ATOM;
              const uint64_t b = sw128_kmajor_desc(smem_u32(bt));
              const uint64_t a0 = sw128_kmajor_desc(smem_u32(smem + C::OFF_A + (ab * NA + 0) * C::A_TILE));
              const uint64_t a1 = sw128_kmajor_desc(smem_u32(smem + C::OFF_A + (ab * NA + (NA - 1)) * C::A_TILE));
#pragma unroll
              for (int kk = 0; kk < KS / 16; ++kk) {
                const uint32_t accum = (kb | j | kk) != 0;
                umma_f16(d0, a0 + 2 * kk, b + 2 * kk, idesc, accum);  // +32 bytes along K
                if (GATED) umma_f16(d1, a1 + 2 * kk, b + 2 * kk, idesc, accum);
              }
            }
            umma_commit(&a_empty[ab]);
            if (++ab == ABUF) {
              ab = 0;
              ph_a ^= 1u;
            }
            if (!THIN) {
              umma_commit(&empty_b[bs]);
              if (++bs == BST) {
                bs = 0;
                ph_b ^= 1u;
              }
            }
          }
          if (THIN && ok) {
            umma_commit(&empty_w[ws]);  // the stage's activation tile has been read
            if (++ws == WST) {
              ws = 0;
              ph_w ^= 1u;
            }
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        if (++acc == ACCB) {
          acc = 0;
          ph_acc ^= 1u;
        }
      }
      umma_commit(drain);  // all MMAs issued by this thread have completed once this fires
      mbar_wait_plain(drain, 0, lim);
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------------- activation producer (wide variant)
    if constexpr (!THIN) {
     if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      const int nks = K / KS;
      int bs = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
        const Item I = decode_item(it, sprefix, p);
        for (int ks = 0; ks < nks; ++ks) {
          if (!(ok = mbar_wait(&empty_b[bs], ph ^ 1u, abort_flag, lim))) break;
          mbar_arrive_expect_tx(&full_b[bs], (uint32_t)(I.nmma * KS * 2));
          for (int r = 0; r < I.nmma; r += 16)
            tma_load_2d_hint(smem + C::OFF_B + bs * C::B_ATOM + r * 128, &tm_b, &full_b[bs], ks * KS, I.r0 + r, pol);
          ++issued;
          if (++bs == BST) {
            bs = 0;
            ph ^= 1u;
          }
        }
      }
      for (int i = max(0, issued - BST); i < issued; ++i) mbar_wait_plain(&full_b[i % BST], (i / BST) & 1, lim);
     }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - kEpiWarp0;  // == warp % 4: this warp may read TMEM lanes 32*ew..32*ew+31
    const int mrow = ew * 32 + lane;
    int acc = 0;
    uint32_t ph = 0;
    for (int it = blockIdx.x; it < total; it += gridDim.x) {
      const Item I = decode_item(it, sprefix, p);
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[acc], ph, abort_flag, lim))) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(ew * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
      const int col = I.m * BM + mrow;
      for (int c0 = 0; c0 < I.nmma; c0 += 16) {
        uint32_t g[16], u[16];
        tmem_ld16(tb + c0, g);
        if (GATED) tmem_ld16(tb + C::CH * NMAX + c0, u);
        tmem_ld_wait();
#pragma unroll
        for (int c = 1; c < C::CH; ++c) {  // sum the independent K chains
          uint32_t g2[16], u2[16];
          tmem_ld16(tb + c * NMAX + c0, g2);
          if (GATED) tmem_ld16(tb + (C::CH + c) * NMAX + c0, u2);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            g[i] = __float_as_uint(__uint_as_float(g[i]) + __uint_as_float(g2[i]));
            if (GATED) u[i] = __float_as_uint(__uint_as_float(u[i]) + __uint_as_float(u2[i]));
          }
        }
        const int nv = min(16, I.nvalid - c0);
        if (GATED) {
          __half* out = reinterpret_cast<__half*>(p.out) + (size_t)(I.r0 + c0) * p.out_ld + interleave_pos(col);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (i < nv) {
              const float gv = __uint_as_float(g[i]), uv = __uint_as_float(u[i]);
              out[(size_t)i * p.out_ld] = __float2half_rn(gv / (1.0f + __expf(-gv)) * uv);
            }
          }
        } else if (p.out_kind == OUT_F32) {
          float* out = reinterpret_cast<float*>(p.out) + (size_t)(I.r0 + c0) * p.out_ld + col;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (i < nv) out[(size_t)i * p.out_ld] = __uint_as_float(g[i]);
        } else {
          __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)(I.r0 + c0) * p.out_ld + col;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (i < nv) out[(size_t)i * p.out_ld] = __float2bfloat16_rn(__uint_as_float(g[i]));
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
  } else if (warp >= kDqWarp0) {
    if constexpr (THIN) {
      // ---------------------------------------------------------------- dequantization -> TMEM
      // 16 warps; warp dw writes TMEM lanes 32*(dw%4).. (its rows).  GATED: warps 0-7 gate,
      // 8-15 up, each thread one row and one 32-K half of every 64-K step.  Plain: each thread
      // one row and one 16-K quarter of every step.
      const int dw = warp - kDqWarp0;
      const int row = (dw & 3) * 32 + lane;
      const int sw = row & 7;
      constexpr int PARTS = C::PARTS;
      constexpr int WPS = 8 / PARTS;  // packed words of each 64-K step this thread takes
      const int mat = GATED ? (dw / (4 * PARTS)) : 0;
      const int part = (dw >> 2) % PARTS;  // which 1/PARTS of the step
      const uint32_t lane_base = tmem_base + ((uint32_t)((dw & 3) * 32) << 16);
      int ws = 0, ab = 0;
      uint32_t ph_w = 0, ph_a = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
        for (int kb = 0; kb < nkb && ok; ++kb) {
          ok = __all_sync(0xffffffffu, mbar_wait(&full_w[ws], ph_w, abort_flag, lim));
          if (!ok) break;
          const uint8_t* st = smem + ws * C::STAGE;
          const uint8_t* wrow = st + C::STAGE_W + mat * C::W_TILE + row * 128;
          const uint4 sc = *reinterpret_cast<const uint4*>(st + C::STAGE_S + mat * C::S_TILE + row * 16);
          // this thread's packed words of every step of the stage: step j = bytes 32j..32j+31
          // of the row (before the swizzle), of which this thread takes words
          // part*WPS .. part*WPS+WPS-1
          uint32_t wv[NSUB][WPS];
#pragma unroll
          for (int j = 0; j < NSUB; ++j) {
#pragma unroll
            for (int c = 0; c < WPS; c += 4 > WPS ? WPS : 4) {
              const int w0 = part * WPS + c;              // first word within the step (0..7)
              const int lc = 2 * j + (w0 >> 2);           // logical 16-byte chunk
              const uint8_t* src = wrow + ((lc ^ sw) << 4) + 4 * (w0 & 3);
              if constexpr (WPS >= 4) {
                const uint4 v = *reinterpret_cast<const uint4*>(src);
                wv[j][c] = v.x, wv[j][c + 1] = v.y, wv[j][c + 2] = v.z, wv[j][c + 3] = v.w;
              } else if constexpr (WPS == 2) {
                const uint2 v = *reinterpret_cast<const uint2*>(src);
                wv[j][c] = v.x, wv[j][c + 1] = v.y;
              } else {
                wv[j][c] = *reinterpret_cast<const uint32_t*>(src);
              }
            }
          }
          const int nsub = min(NSUB, (K - kb * KB) / KS);
#pragma unroll
          for (int j0 = 0; j0 < NSUB; j0 += C::SPS) {
            if (j0 < nsub) {
              ok = __all_sync(0xffffffffu, mbar_wait(&a_empty[ab], ph_a ^ 1u, abort_flag, lim));
              if (!ok) break;
              tc_fence_after();  // the MMAs that last read this A slot have completed
              const uint32_t slot = (uint32_t)(C::A_COL0 + ab * C::SLOT_COLS + mat * C::SPS * C::A_COLS);
#pragma unroll
              for (int s2 = 0; s2 < C::SPS; ++s2) {
                const int j = j0 + s2;
                const uint32_t col = slot + (uint32_t)(s2 * C::A_COLS + part * WPS * 4);
                uint32_t r[WPS * 4];
#pragma unroll
                for (int w = 0; w < WPS; ++w) {
                  const __half2 sc2 = scale_h2(sc, 2 * j + ((part * WPS + w) >> 2));  // 32 K per scale
                  const uint4 d = dequant_word(wv[j][w], sc2);
                  r[4 * w + 0] = d.x, r[4 * w + 1] = d.y, r[4 * w + 2] = d.z, r[4 * w + 3] = d.w;
                }
                if constexpr (WPS == 8)
                  tmem_st32(lane_base + col, r);
                else if constexpr (WPS == 4)
                  tmem_st16(lane_base + col, r);
                else
                  tmem_st8(lane_base + col, r);
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
          if (!ok) break;
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty_w[ws]);  // every word read from the stage is consumed
          if (++ws == WST) {
            ws = 0;
            ph_w ^= 1u;
          }
        }
      }
    } else {
      // ---------------------------------------------------------------- dequantization -> SMEM
      // 8 warps.  GATED: thread = one row of the gate (warps 8-11) or up (warps 12-15) tile,
      // all 64 K of each step; plain: thread = one row, half of each 64-K step.
      const int dt = threadIdx.x - kDqWarp0 * 32;  // 0..255
      const int mat = GATED ? (dt >> 7) : 0;
      const int half = GATED ? 0 : (dt >> 7);
      const int row = dt & 127;
      const int sw = row & 7;
      constexpr int CHK = GATED ? 8 : 4;  // 16-byte chunks of packed words this thread takes per stage
      int ws = 0, ab = 0;
      uint32_t ph_w = 0, ph_a = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < total && ok; it += gridDim.x) {
        for (int kb = 0; kb < nkb && ok; ++kb) {
          ok = __all_sync(0xffffffffu, mbar_wait(&full_w[ws], ph_w, abort_flag, lim));
          if (!ok) break;
          const uint8_t* st = smem + ws * C::STAGE;
          const uint8_t* wrow = st + C::STAGE_W + mat * C::W_TILE + row * 128;
          const uint4 sc = *reinterpret_cast<const uint4*>(st + C::STAGE_S + mat * C::S_TILE + row * 16);
          uint4 wv[CHK];
#pragma unroll
          for (int c = 0; c < CHK; ++c) {
            const int lc = GATED ? c : 2 * c + half;  // logical 16-byte chunk (32 K) of the 128-byte row
            wv[c] = *reinterpret_cast<const uint4*>(wrow + ((lc ^ sw) << 4));
          }
          const int nsub = min(NSUB, (K - kb * KB) / KS);
#pragma unroll
          for (int j = 0; j < NSUB; ++j) {
            if (j < nsub) {
              ok = __all_sync(0xffffffffu, mbar_wait(&a_empty[ab], ph_a ^ 1u, abort_flag, lim));
              if (!ok) break;
              uint8_t* arow = smem + C::OFF_A + (ab * NA + mat) * C::A_TILE + row * 128;
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                if (GATED || q == half) {
                  const uint4 w = GATED ? wv[2 * j + q] : wv[j];
                  const __half2 s2 = scale_h2(sc, 2 * j + q);
                  *reinterpret_cast<uint4*>(arow + (((4 * q + 0) ^ sw) << 4)) = dequant_word(w.x, s2);
                  *reinterpret_cast<uint4*>(arow + (((4 * q + 1) ^ sw) << 4)) = dequant_word(w.y, s2);
                  *reinterpret_cast<uint4*>(arow + (((4 * q + 2) ^ sw) << 4)) = dequant_word(w.z, s2);
                  *reinterpret_cast<uint4*>(arow + (((4 * q + 3) ^ sw) << 4)) = dequant_word(w.w, s2);
                }
              }
              fence_proxy_async_smem();  // generic-proxy smem writes -> visible to the tensor core
              __syncwarp();
              if (lane == 0) mbar_arrive(&a_full[ab]);
              if (++ab == ABUF) {
                ab = 0;
                ph_a ^= 1u;
              }
            }
          }
          if (!ok) break;
          // release the stage only after every word loaded from it has been consumed
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty_w[ws]);
          if (++ws == WST) {
            ws = 0;
            ph_w ^= 1u;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <bool GATED, int NMAX>
cudaError_t launch_t(const W4GemmProblem& pr, cudaStream_t s) {
  using C = Cfg<GATED, NMAX>;
  CUtensorMap tm_w, tm_s, tm_b;
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
  if (encode_tmap_2d(&tm_b, pr.act, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, pr.K, (uint64_t)pr.act_rows, (uint64_t)pr.K * 2,
                     KS, 16, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  Params p;
  p.K = pr.K;
  p.E = pr.E;
  p.rows_per_expert = pr.rows_per_expert;
  p.I = pr.I;
  p.m_tiles = GATED ? pr.I / BM : pr.rows_per_expert / BM;
  p.scales_tma = scales_tma;
  p.w_s = pr.w_s;
  p.sched = pr.sched;
  p.out = pr.out;
  p.out_ld = pr.out_ld;
  p.out_kind = pr.out_kind;
  p.wait_limit = wait_limit_ns();
  const size_t smem = C::smem_bytes(pr.E);
  auto kern = w4a16_gemm_kernel<GATED, NMAX>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const char* name = GATED ? "w4a16_gemm_gate_up" : "w4a16_gemm_down";
  timing_before(name, s);
  kern<<<sm_count(), C::THREADS, smem, s>>>(tm_w, tm_s, tm_b, p);
  timing_after(name, s);
  return cudaGetLastError();
}

}  // namespace w4

cudaError_t launch_w4a16_gemm(const W4GemmProblem& p, cudaStream_t s) {
  constexpr int THIN = w4::kThinN;
  if (p.gated) {
    if (p.nmax <= THIN) return w4::launch_t<true, THIN>(p, s);
    return w4::launch_t<true, 256>(p, s);
  }
  if (p.nmax <= THIN) return w4::launch_t<false, THIN>(p, s);
  return w4::launch_t<false, 256>(p, s);
}

}  // namespace moe
