// Tensor-core path (tcgen05 + TMEM + TMA) for many tokens.
//
// Once M is large the product stops being bandwidth-bound and becomes a dense
// contraction; the decode-then-multiply order of the GPTQ-Triton summary ("How
// It Works": quantized weights decoded on the fly before the matmul) is kept,
// but the multiply runs on the 5th-generation tensor cores:
//
//   D[128 weight rows, BN tokens] (fp32, TMEM) += A[128, 64] . B[BN, 64]^T
//
// per 64-column K block, with A = decoded weights (fp16/bf16, written into
// shared memory in the 128-byte-swizzled K-major layout by decode warps) and
// B = a TMA-loaded tile of x.  Warp roles:
//   warp 0      TMA producers: lane 0 code tiles (4 KB per K block, 8 row
//               blocks) with their group scales / zero-points, lane 1 x tiles
//   warp 1      TMEM owner and MMA issuer (one elected thread)
//   next kDecWarps warps   decode, one row block each: codes and scales (smem)
//                          -> (q - z) s, T[q] s -> A tile
//   last 4 warps           epilogue: TMEM -> registers -> y (or split-K partials)
// Work is split stream-K over (tile, unit) pairs, a unit being one or two K
// blocks (one round of the rings), across a grid of one CTA per SM, like the
// decode path; partial tiles are reduced deterministically by the last CTA
// that finishes them.  A CTA's last segment is finished after the role loops
// by the decode and epilogue warps together (warp 1 staging the other
// contributors' partial sums).  Every mbarrier wait is bounded: a wait that
// runs out sets the device error word (qmm_check_error) and the CTA drains and
// exits instead of hanging.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace qk {

__device__ unsigned g_tc_error = 0;

namespace {

constexpr int kDecWarps = 8;                        // decode warps (one of the 8 row blocks each)
constexpr int kRbPerDec = 8 / kDecWarps;            // row blocks per decode warp
constexpr int kTcThreads = 32 * (2 + kDecWarps + 4);
constexpr int kEpi0 = 32 * (2 + kDecWarps);          // first epilogue thread
constexpr int kKB = 64;             // K columns per k block (one 128-byte swizzle row of fp16)
constexpr int kRowsTile = 128;      // weight rows per tile (UMMA M)
constexpr int kCodeBytes = 8 * 512; // a k block's codes: 8 row blocks x one 512-byte chunk
constexpr int kATileBytes = kRowsTile * kKB * 2;   // 16 KB
// Per code stage, the unit's group scales (and ASYM zero-points) of the
// tile's 8 row blocks, loaded by TMA with the codes: [8][sx] fp16, sx = 16
// slots x the groups in the unit's columns, 1 KB per 64 columns.
constexpr int kMetaTile = 1024;
// Bound of the waits a CTA makes for its own copies and MMAs while draining
// (they always complete): ~2 s at 1.9 GHz.
constexpr long long kDrainCycles = 4000000000ll;
// Final reduction of a CTA's last partial tile: the other contributors'
// partial sums are brought into the (then idle) A / B ring by bulk copies,
// 32 columns x 128 rows of fp32 (16 KB) per copy; one arrival barrier per
// 32-column chunk (at most 8) and one release barrier per buffer set.
constexpr int kRedChunk = 32 * kRowsTile * 4;
constexpr int kRedSets = 9;   // >= the 8 chunks of a 256-token tile

// SPLIT: bf16 activations whose A operand is not an exact small integer
// (group scales, or a table): each decoded weight w, exact in fp32, becomes
// two bf16 operands hi = bf16(w) and lo = bf16(w - hi) (|w - hi - lo| <=
// 2^-18 |w|), two A tiles per stage and two MMAs per k step into the same
// accumulator.  A single bf16 rounding of w (2^-9) together with the bf16
// output would use most of the error budget.
//
// KU: 64-column k blocks per unit of work (1 or 2).  A unit is one round of the
// rings and barriers (one code tile, one x tile, one A tile per k block, one
// commit); two k blocks per unit halve those rounds per column where the
// doubled stages still fit: 64 tokens in every format but a table with split
// operands; 128 tokens without a table or a split; 256 tokens without them or
// zero-points (two A / B stages and three code stages).
template <int BN, bool SPLIT = false, bool TABLE = false, int KU = 1>
struct TcCfg {
  static_assert(KU == 1 || (KU == 2 && !(SPLIT && TABLE) && (BN == 64 || (!SPLIT && !TABLE))),
                "two k blocks per unit");
  // A / B ring depth within 227 KB (the table takes 32 KB)
  static constexpr int STAGES =
      KU == 2 ? (BN == 64 ? (SPLIT ? 2 : 3) : 2)
              : (SPLIT ? (BN == 64 ? (TABLE ? 3 : 4) : (BN == 128 ? 3 : 2)) : (BN == 256 ? 3 : 4));
  static constexpr int B_BYTES = KU * BN * kKB * 2;
  static constexpr int A_BYTES = KU * (SPLIT ? 2 : 1) * kATileBytes;   // one stage's A tile(s)
  static constexpr int CODE_STAGES = (KU == 2 && BN == 256) ? 3 : 8 / KU;
  static constexpr int CODE_BYTES = KU * kCodeBytes;
  static constexpr int META_TILE = KU * kMetaTile;
  template <int MODE>
  static constexpr int META_BYTES = MODE == kASYM ? 2 * META_TILE : META_TILE;
  static constexpr int TMEM_COLS = 2 * BN;     // two accumulator buffers
  static constexpr int RED_BUFS = std::min(STAGES * (A_BYTES + B_BYTES) / kRedChunk, kRedSets);
  static_assert(RED_BUFS >= 6, "staging buffers of the final reduction (two slot chunks per group)");
};

// ------------------------------------------------------------------ PTX helpers

// Bounded wait for phase `parity` of `bar`.  Returns false (and raises the
// CTA's abort flag and the device error word) if `limit` clock cycles pass,
// or at once if another thread of the CTA has already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          long long limit) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > limit) {
      *abort = 1;
      atomicOr(&g_tc_error, 1u);
      return false;
    }
  }
}

// Wait for a copy or MMA the CTA issued itself, before it frees what they
// use: ignores the abort flag, bounded by kDrainCycles.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return;
  const long long t0 = clock64();
  while (!mbar_try(bar, parity))
    if (clock64() - t0 > kDrainCycles) return;
}

// The shared memory of all but the most recent committed bulk store has been read.
__device__ __forceinline__ void bulk_wait_read_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

// Named barrier whose result is the AND of every participating thread's
// predicate: a decision the warps of a role take together.
__device__ __forceinline__ bool named_bar_and(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (tile bases are 1024-byte aligned).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;              // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;    // stride byte offset
  d |= (uint64_t)1 << 46;              // descriptor version
  d |= (uint64_t)2 << 61;              // 128-byte swizzle
  return d;
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void named_bar(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ------------------------------------------------------------------ kernel

struct TcArgs {
  const uint16_t* scales;
  const uint16_t* zl;
  uint16_t* y;
  int M, N, K, L, G, nrb, nkb;
  int sx;                   // scale (zero) elements per row block in a k block's meta tile
  int lg;                   // log2 of the group length; 30 for one group per row
  int gated;                // 1: alternating 16-row gate / up blocks, y[M, N/2] = silu(gate) up
  int tiles_n, tiles_m, tiles;
  long long units;          // tiles * nkb
  int ctas;
  long long wait_limit;     // clock cycles a barrier wait may take before the call gives up
  float* slots;             // [2 * ctas][BN][128]: a CTA's first / last partial tile,
                            // column-major so that a warp's 32 rows are 128 contiguous bytes
  unsigned* counters;       // [tiles]
};

__device__ __forceinline__ int owner_of_tc(long long u, long long U, int C) {
  return (int)(((u + 1) * (long long)C - 1) / U);
}

__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Scaled decoded pair (row of the pair, two k) -> packed fp16 / bf16.
template <bool BF16>
__device__ __forceinline__ uint32_t scale_pair(uint32_t v, float s) {
  if constexpr (BF16) {
    const float lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xFFFF0000u);
    return pack2<true>(lo * s, hi * s);
  } else {
    const __half2 sh = __float2half2_rn(s);
    const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&v), sh);
    return *reinterpret_cast<const uint32_t*>(&r);
  }
}

// fp16 table pair -> A operand pair: T s rounded once (fp16: one HMUL2; bf16:
// product in fp32, then rounded); with per-row scales (group -1) the scale is
// applied in the epilogue and T alone is converted.
template <bool BF16, bool GM1>
__device__ __forceinline__ uint32_t lut_pair(uint32_t t16, float s) {
  if constexpr (!BF16) {
    return GM1 ? t16 : scale_pair<false>(t16, s);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&t16));
    return GM1 ? pack2<true>(f.x, f.y) : pack2<true>(f.x * s, f.y * s);
  }
}

template <int MODE, bool BF16, int BN, bool GM1, int KU>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
              const __grid_constant__ CUtensorMap map_s, const __grid_constant__ CUtensorMap map_z,
              const __grid_constant__ CUtensorMap map_y, const TcArgs a) {
  constexpr bool SPLIT = BF16 && (!GM1 || MODE == kLUT);
  using Cfg = TcCfg<BN, SPLIT, MODE == kLUT, KU>;
  constexpr int S = Cfg::STAGES;
  constexpr int kCodeStages = Cfg::CODE_STAGES;
  constexpr int kStageCode = Cfg::CODE_BYTES;
  constexpr int kStageMeta = Cfg::template META_BYTES<MODE>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // carve: A stages | B stages | code stages | meta stages | LUT table | barriers.
  // The 1024-byte aligned start is an offset from the shared array itself, so
  // the compiler keeps every access below in the shared address space (a
  // pointer rebuilt from an integer would turn them into generic accesses).
  unsigned char* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* sA = base;
  unsigned char* sB = sA + S * Cfg::A_BYTES;
  unsigned char* sC = sB + S * Cfg::B_BYTES;
  unsigned char* sM = sC + kCodeStages * kStageCode;
  unsigned char* sT = sM + kCodeStages * kStageMeta;
  // group scales and zero-points come with the codes (per-row scales of
  // group -1 are applied in the epilogue instead)
  constexpr bool kScales = !GM1;
  constexpr bool kZeros = MODE == kASYM;
  constexpr int TAB = MODE == kLUT ? 256 * 32 * 4 : 0;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sT + TAB);
  uint64_t* code_full = bars;
  uint64_t* code_empty = code_full + kCodeStages;
  uint64_t* b_full = code_empty + kCodeStages;
  uint64_t* a_full = b_full + S;
  uint64_t* ab_empty = a_full + S;
  uint64_t* acc_full = ab_empty + S;      // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2]
  uint64_t* mma_drain = acc_empty + 2;    // the MMA thread's last commit
  uint64_t* red_full = mma_drain + 1;     // [kRedSets]: a chunk's staged partial sums landed
  uint64_t* red_empty = red_full + kRedSets;   // [kRedSets]: a set read by its group
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_empty + kRedSets);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* last_flag = const_cast<int*>(abort_flag) + 1;
  int* meta = last_flag + 1;   // [3]: first contributor, contributors, first's slot parity
  int* fin = meta + 3;         // [2]: the CTA's last segment is pending (1), its index
  long long* fin_u = reinterpret_cast<long long*>(fin + 2);   // its first unit

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const long long u_begin = (long long)b * a.units / a.ctas;
  const long long u_end = (long long)(b + 1) * a.units / a.ctas;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kCodeStages; ++i) {
      mbar_init(&code_full[i], 1);
      mbar_init(&code_empty[i], kDecWarps);
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&a_full[i], kDecWarps);
      mbar_init(&ab_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(mma_drain, 1);
    for (int i = 0; i < kRedSets; ++i) {
      mbar_init(&red_full[i], 1);
      mbar_init(&red_empty[i], 4);
    }
    *abort_flag = 0;
    fin[0] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_w)) : "memory");
    if constexpr (kScales)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_s)) : "memory");
    if constexpr (kZeros)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_z)) : "memory");
  }
  pdl_wait();                 // inputs may come from the previous grid; TMEM taken after this
  pdl_launch_dependents();

  if constexpr (MODE == kLUT) {
    // 4-bit pair table replicated per bank (see the decode path): fp16
    // entries; with bf16 activations the scaled product is rounded per weight.
    uint32_t* tab = reinterpret_cast<uint32_t*>(sT);
    for (int i = threadIdx.x; i < 256 * 32; i += kTcThreads) {
      const int e = i >> 5;
      tab[i] = (uint32_t)a.zl[e & 15] | ((uint32_t)a.zl[e >> 4] << 16);
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(Cfg::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // y for tokens c0 .. c0 + 31 of `tile` at TMEM lane row_l (weight row
  // tn 128 + row_l), per-row scale of group -1 applied here.  Gated layout: the
  // quadrant's 32 rows are one gate block (lanes 0-15) and its up block (lanes
  // 16-31).  Called by whole warps.
  auto store_y32 = [&](const float (&vals)[32], int tile, int row_l, int c0) {
    const int tn = tile % a.tiles_n, tm = tile / a.tiles_n;
    const int row = tn * kRowsTile + row_l;
    float s_row = 1.0f;
    if constexpr (GM1) {
      if (row < a.N)
        s_row = __half2float(__ushort_as_half(a.scales[(size_t)(row >> 4) * 16 + scale_slot(row & 15)]));
    }
    if (!a.gated) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int m = tm * BN + c0 + i;
        if (row < a.N && m < a.M) {
          const float o = vals[i] * s_row;
          a.y[(size_t)m * a.N + row] = BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(o))
                                            : __half_as_ushort(__float2half_rn(o));
        }
      }
    } else {
      const int ny = a.N >> 1;
      const int col = (row >> 5) * 16 + (row & 15);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float o = vals[i] * s_row;
        const float up = __shfl_down_sync(0xffffffffu, o, 16);
        const int m = tm * BN + c0 + i;
        if ((row_l & 31) < 16 && row < a.N && m < a.M) {
          const float gv = silu(o) * up;
          a.y[(size_t)m * ny + col] = BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(gv))
                                           : __half_as_ushort(__float2half_rn(gv));
        }
      }
    }
  };

  // Segments of this CTA: [u, u + len) within one tile.
  auto seg_of = [&](long long u, int& tile, int& kb0, int& kb1) {
    tile = (int)(u / a.nkb);
    kb0 = (int)(u % a.nkb);
    kb1 = (int)std::min<long long>(a.nkb, kb0 + (u_end - u));
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producers
    // Two independent single-thread loops: lane 0 streams the code tiles from
    // HBM as far ahead as the code ring allows (its latency is the long one),
    // lane 1 the x tiles (L2-resident) as the A/B ring frees its stages.
    if (lane == 0) {
      int kc = 0;             // running k-block counter of the code ring
      for (long long u = u_begin; u < u_end && !*abort_flag;) {
        int tile, kb0, kb1;
        seg_of(u, tile, kb0, kb1);
        const int tn = tile % a.tiles_n;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb, ++kc) {
          const int c = kc % kCodeStages;
          if (!mbar_wait(&code_empty[c], ((kc / kCodeStages) & 1) ^ 1, abort_flag, a.wait_limit)) {
            ok = false;
            break;
          }
          constexpr int kMetaCopies = (kScales ? 1 : 0) + (kZeros ? 1 : 0);
          mbar_expect_tx(&code_full[c], kStageCode + kMetaCopies * 8 * a.sx * 2);
          // the unit's KU chunks of each of the 8 row blocks (columns past K
          // read as zero codes; their x columns are zero too)
          tma_load_2d(sC + c * kStageCode, &map_w, &code_full[c], kb * 128 * KU, tn * 8);
          // the unit's first group, 16 slots per group (the x coordinate is
          // a multiple of 16 elements: 32-byte aligned)
          const int gx = ((kb * KU * kKB) >> a.lg) * 16;
          if constexpr (kScales)
            tma_load_2d(sM + c * kStageMeta, &map_s, &code_full[c], gx, tn * 8);
          if constexpr (kZeros)
            tma_load_2d(sM + c * kStageMeta + Cfg::META_TILE, &map_z, &code_full[c], gx, tn * 8);
        }
        if (!ok) break;
        u += kb1 - kb0;
      }
      // nothing may land after the CTA exits: the last fill of every slot
      // (consumed already, unless the CTA is giving up)
      for (int j = kc > kCodeStages ? kc - kCodeStages : 0; j < kc; ++j)
        drain_wait(&code_full[j % kCodeStages], (j / kCodeStages) & 1);
    } else if (lane == 1) {
      int ks = 0;             // running k-block counter of the A/B ring
      for (long long u = u_begin; u < u_end && !*abort_flag;) {
        int tile, kb0, kb1;
        seg_of(u, tile, kb0, kb1);
        const int tm = tile / a.tiles_n;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb, ++ks) {
          const int s = ks % S;
          if (!mbar_wait(&ab_empty[s], ((ks / S) & 1) ^ 1, abort_flag, a.wait_limit)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&b_full[s], Cfg::B_BYTES);
#pragma unroll
          for (int kb2 = 0; kb2 < KU; ++kb2)
            tma_load_2d(sB + s * Cfg::B_BYTES + kb2 * (BN * kKB * 2), &map_x, &b_full[s],
                        (kb * KU + kb2) * kKB, tm * BN);
        }
        if (!ok) break;
        u += kb1 - kb0;
      }
      for (int j = ks > S ? ks - S : 0; j < ks; ++j) drain_wait(&b_full[j % S], (j / S) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = (1u << 4) | (BF16 ? (1u << 7) | (1u << 10) : 0u) |
                                 ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(kRowsTile >> 4) << 24);
      int ks = 0, seg = 0;
      for (long long u = u_begin; u < u_end && !*abort_flag; ++seg) {
        int tile, kb0, kb1;
        seg_of(u, tile, kb0, kb1);
        const int buf = seg & 1;
        if (!mbar_wait(&acc_empty[buf], ((seg >> 1) & 1) ^ 1, abort_flag, a.wait_limit)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * BN);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb, ++ks) {
          const int s = ks % S;
          const uint32_t ph = (ks / S) & 1;
          if (!mbar_wait(&a_full[s], ph, abort_flag, a.wait_limit) || !mbar_wait(&b_full[s], ph, abort_flag, a.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kb2 = 0; kb2 < KU; ++kb2) {
            const uint32_t sa = smem_u32(sA + s * Cfg::A_BYTES + kb2 * (SPLIT ? 2 : 1) * kATileBytes);
            const uint32_t sb = smem_u32(sB + s * Cfg::B_BYTES + kb2 * (BN * kKB * 2));
#pragma unroll
            for (int k = 0; k < kKB / 16; ++k) {
              umma_f16(d, sw128_desc(sa + 32 * k), sw128_desc(sb + 32 * k), idesc,
                       (kb > kb0 || kb2 > 0 || k > 0) ? 1u : 0u);
              if constexpr (SPLIT)   // the low parts of the weights, same accumulator
                umma_f16(d, sw128_desc(sa + kATileBytes + 32 * k), sw128_desc(sb + 32 * k), idesc, 1u);
            }
          }
          umma_commit(&ab_empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
        u += kb1 - kb0;
      }
      // every MMA issued has finished before TMEM (and the A / B tiles) can
      // be released: one more commit, which arrives once they all have
      umma_commit(mma_drain);
      drain_wait(mma_drain, 0);
    }
  } else if (warp < 2 + kDecWarps) {
    // ------------------------------------------------------------ decode warps
    const int dw = warp - 2;                 // row blocks kRbPerDec dw + rr of the tile
    const int g = lane >> 2, t = lane & 3;
    const unsigned char* tabp = sT;
    int kc = 0, ks = 0;
    for (long long u = u_begin; u < u_end; ++u, ++kc, ++ks) {
      const int c = kc % kCodeStages, s = ks % S;
      // the warp stops as one (it ends each stage with a warp-wide sync)
      const bool ok = mbar_wait(&code_full[c], (kc / kCodeStages) & 1, abort_flag, a.wait_limit) &&
                      mbar_wait(&ab_empty[s], ((ks / S) & 1) ^ 1, abort_flag, a.wait_limit);
      if (!__all_sync(0xffffffffu, ok)) break;
#pragma unroll
      for (int kb2 = 0; kb2 < KU; ++kb2) {   // the unit's k blocks, one A tile each
      unsigned char* At = sA + s * Cfg::A_BYTES + kb2 * (SPLIT ? 2 : 1) * kATileBytes;
      // group scales (and zero-points) of the lane's rows g and g + 8, one word
      // per 16-column slice j, from the unit's meta tile (landed with the codes)
      uint32_t sw[kRbPerDec][4], zw[kRbPerDec][4];
      if constexpr (kScales || kZeros) {
        const unsigned char* mt = sM + c * kStageMeta;
#pragma unroll
        for (int rr = 0; rr < kRbPerDec; ++rr)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int e = (kRbPerDec * dw + rr) * a.sx + ((16 * j + kKB * kb2) >> a.lg) * 16 + 2 * g;
            if constexpr (kScales) sw[rr][j] = *reinterpret_cast<const uint32_t*>(mt + 2 * e);
            if constexpr (kZeros) zw[rr][j] = *reinterpret_cast<const uint32_t*>(mt + Cfg::META_TILE + 2 * e);
          }
      }
#pragma unroll
      for (int rr = 0; rr < kRbPerDec; ++rr) {
        const int rbl = kRbPerDec * dw + rr;               // row block in the tile
        const uint4 wv = *reinterpret_cast<const uint4*>(sC + c * kStageCode + rbl * (KU * 512) +
                                                         kb2 * 512 + lane * 16);
        const int R0 = rbl * 16 + g, R1 = R0 + 8;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t w = (&wv.x)[j];
          uint32_t af[4];
          if constexpr (MODE == kSYM) {
            decode_int4<BF16, 8>(w, af);
          } else if constexpr (MODE == kASYM) {
            decode_int4<BF16, 0>(w, af);
            uint32_t z = zw[rr][j];
            if constexpr (BF16) {
              const float2 zf = __half22float2(*reinterpret_cast<const __half2*>(&z));
              z = pack2<true>(zf.x, zf.y);
            }
            sub_zero<BF16>(__byte_perm(z, 0, 0x1010), __byte_perm(z, 0, 0x3232), af);
          } else {
            const uint32_t l4 = (uint32_t)lane << 2;
            af[0] = *reinterpret_cast<const uint32_t*>(tabp + lop3_and_or(w << 7, 0x7F80u, l4));
            af[1] = *reinterpret_cast<const uint32_t*>(tabp + lop3_and_or(w >> 1, 0x7F80u, l4));
            af[2] = *reinterpret_cast<const uint32_t*>(tabp + lop3_and_or(w >> 9, 0x7F80u, l4));
            af[3] = *reinterpret_cast<const uint32_t*>(tabp + lop3_and_or(w >> 17, 0x7F80u, l4));
          }
          uint32_t alo[4];   // SPLIT: the low bf16 parts
          if constexpr (SPLIT) {
            // w exact in fp32 ((q - z) s, or T s, or T alone with per-row
            // scales), then hi = bf16(w), lo = bf16(w - hi)
            float2 sc = make_float2(1.f, 1.f);
            if constexpr (kScales) sc = __half22float2(*reinterpret_cast<const __half2*>(&sw[rr][j]));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float2 v;
              if constexpr (MODE == kLUT) {
                v = __half22float2(*reinterpret_cast<const __half2*>(&af[i]));
              } else {
                v = make_float2(__uint_as_float(af[i] << 16), __uint_as_float(af[i] & 0xFFFF0000u));
              }
              const float si = (i & 1) ? sc.y : sc.x;   // registers 0, 2: row g; 1, 3: row g + 8
              v.x *= si;
              v.y *= si;
              const uint32_t hi = pack2<true>(v.x, v.y);
              alo[i] = pack2<true>(v.x - __uint_as_float(hi << 16), v.y - __uint_as_float(hi & 0xFFFF0000u));
              af[i] = hi;
            }
          } else if constexpr (kScales && !BF16 && MODE != kLUT) {
            // (s_g, s_g) and (s_g8, s_g8) as fp16 pairs: one HMUL2 per register
            const uint32_t sg = __byte_perm(sw[rr][j], 0, 0x1010);
            const uint32_t sg8 = __byte_perm(sw[rr][j], 0, 0x3232);
            af[0] = hmul2_u(af[0], sg);
            af[2] = hmul2_u(af[2], sg);
            af[1] = hmul2_u(af[1], sg8);
            af[3] = hmul2_u(af[3], sg8);
          } else if constexpr (kScales || MODE == kLUT) {
            float2 sc = make_float2(1.f, 1.f);
            if constexpr (kScales) sc = __half22float2(*reinterpret_cast<const __half2*>(&sw[rr][j]));
            if constexpr (MODE == kLUT) {
              af[0] = lut_pair<BF16, GM1>(af[0], sc.x);
              af[2] = lut_pair<BF16, GM1>(af[2], sc.x);
              af[1] = lut_pair<BF16, GM1>(af[1], sc.y);
              af[3] = lut_pair<BF16, GM1>(af[3], sc.y);
            } else {
              af[0] = scale_pair<BF16>(af[0], sc.x);
              af[2] = scale_pair<BF16>(af[2], sc.x);
              af[1] = scale_pair<BF16>(af[1], sc.y);
              af[3] = scale_pair<BF16>(af[3], sc.y);
            }
          }
          // k_local = 16 j + 4 t: 16-byte chunk 2j + t/2, offset 8 (t & 1)
          const int ch = 2 * j + (t >> 1);
          const int off = 8 * (t & 1);
          *reinterpret_cast<uint2*>(At + R0 * 128 + ((ch ^ (R0 & 7)) << 4) + off) =
              make_uint2(af[0], af[2]);
          *reinterpret_cast<uint2*>(At + R1 * 128 + ((ch ^ (R1 & 7)) << 4) + off) =
              make_uint2(af[1], af[3]);
          if constexpr (SPLIT) {
            *reinterpret_cast<uint2*>(At + kATileBytes + R0 * 128 + ((ch ^ (R0 & 7)) << 4) + off) =
                make_uint2(alo[0], alo[2]);
            *reinterpret_cast<uint2*>(At + kATileBytes + R1 * 128 + ((ch ^ (R1 & 7)) << 4) + off) =
                make_uint2(alo[1], alo[3]);
          }
        }
      }
      }   // k blocks of the unit
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&code_empty[c]);
        mbar_arrive(&a_full[s]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int row_l = q * 32 + lane;         // weight row within the tile
    int seg = 0;
    for (long long u = u_begin; u < u_end; ++seg) {
      int tile, kb0, kb1;
      seg_of(u, tile, kb0, kb1);
      const int buf = seg & 1;
      // the four epilogue warps stop together (they share named barriers)
      const bool ok = mbar_wait(&acc_full[buf], (seg >> 1) & 1, abort_flag, a.wait_limit);
      if (!named_bar_and(1, 128, ok)) break;
      tc_fence_after();
      if (u + (kb1 - kb0) == u_end) {
        // the CTA's last segment: its epilogue is shared by the decode and
        // epilogue warps once every role has finished (after the role loops)
        if (threadIdx.x == kEpi0) {
          fin[0] = 1;
          fin[1] = seg;
          *fin_u = u;
        }
        break;
      }
      const long long t_first = (long long)tile * a.nkb;
      const bool whole = (u == t_first) && (kb1 == a.nkb);
      // partial tiles: slot 2 b + e holds this CTA's [BN][128 rows] fp32 sums
      // (e = 1 when the tile is not the CTA's first); contributors are CTAs
      // first .. first + nb - 1, of which only `first` can have e = 1
      float* slot = nullptr;
      if (!whole) {
        const int e = (tile == (int)(u_begin / a.nkb)) ? 0 : 1;
        slot = a.slots + (size_t)(2 * b + e) * (size_t)(BN * kRowsTile) + row_l;
        if (threadIdx.x == kEpi0) {     // 64-bit stream-K bookkeeping, once
          const int first = owner_of_tc(t_first, a.units, a.ctas);
          meta[0] = first;
          meta[1] = owner_of_tc(t_first + a.nkb - 1, a.units, a.ctas) - first + 1;
          meta[2] = ((long long)first * a.units / a.ctas < t_first) ? 1 : 0;
        }
      }
      auto store32 = [&](const float (&vals)[32], int c0) { store_y32(vals, tile, row_l, c0); };
      // A partial tile whose other contributors have all arrived already:
      // this CTA is certainly the last one, so it adds the others' slots to its
      // own sums straight from TMEM, without writing its own slot.
      // Contributors are added in order, as in the general path.
      if (!whole) {
        named_bar(1, 128);   // meta written
        if (threadIdx.x == kEpi0) {
          unsigned cur;
          asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(cur) : "l"(&a.counters[tile]) : "memory");
          *last_flag = cur == (unsigned)(meta[1] - 1) ? 2 : 0;
        }
        named_bar(1, 128);
      }
      if (!whole && *last_flag == 2) {
        const int first = meta[0], nb = meta[1], first_e = meta[2];
        const int own = b - first;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          float accv[32];
          tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + c0), accv);
          if (own != 0) {
#pragma unroll
            for (int i = 0; i < 32; ++i) accv[i] = 0.0f;
          }
          for (int k = 0; k < nb; ++k) {
            float va[32];
            if (k == own) {
              if (k == 0) continue;   // own sums already in accv
              tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + c0), va);
            } else {
              const float* pa = a.slots +
                                (size_t)(2 * (first + k) + (k == 0 ? first_e : 0)) * (BN * kRowsTile) +
                                (size_t)c0 * kRowsTile + row_l;
#pragma unroll
              for (int i = 0; i < 32; ++i) va[i] = __ldcg(pa + (size_t)i * kRowsTile);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) accv[i] += va[i];
          }
          store32(accv, c0);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);     // the accumulator may be reused
        if (threadIdx.x == kEpi0) a.counters[tile] = 0u;   // ready for the next call
        named_bar(1, 128);   // last_flag / meta are reused by the next segment
        u += kb1 - kb0;
        continue;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float v[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + c0), v);
        if (whole) {
          store32(v, c0);
        } else {
          // column c of the slot: the warp's 32 rows are one 128-byte line
#pragma unroll
          for (int i = 0; i < 32; ++i) __stcg(slot + (size_t)(c0 + i) * kRowsTile, v[i]);
        }
      }
      // the tile's last contributor may read the slot with bulk copies (async proxy)
      if (!whole) fence_proxy_async_global();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);     // the accumulator may be reused
      if (!whole) {
        // every epilogue thread's slot stores, then one release increment
        named_bar(1, 128);
        if (threadIdx.x == kEpi0) {
          unsigned prev;
          asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;"
                       : "=r"(prev)
                       : "l"(&a.counters[tile])
                       : "memory");
          *last_flag = prev == (unsigned)(meta[1] - 1);
        }
        named_bar(1, 128);
        if (*last_flag) {
          const int first = meta[0], nb = meta[1], first_e = meta[2];
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 32) {
            float accv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) accv[i] = 0.0f;
            for (int k = 0; k < nb; ++k) {      // one contributor's 32 loads in flight
              const float* pa = a.slots +
                                (size_t)(2 * (first + k) + (k == 0 ? first_e : 0)) * (BN * kRowsTile) +
                                (size_t)c0 * kRowsTile + row_l;
              float va[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) va[i] = __ldcg(pa + (size_t)i * kRowsTile);
#pragma unroll
              for (int i = 0; i < 32; ++i) accv[i] += va[i];
            }
            store32(accv, c0);
          }
          if (threadIdx.x == kEpi0) a.counters[tile] = 0u;   // ready for the next call
        }
        named_bar(1, 128);   // last_flag / meta are reused by the next segment
      }
      u += kb1 - kb0;
    }
  }

  // ---------------------------------------------------------- last segment
  // Every role has finished: all MMAs are complete (the MMA thread waited for
  // them) and no copy is in flight, so TMEM holds the last segment's sums and
  // the rings are free.  The decode and epilogue warps share the segment's
  // epilogue, which a CTA's range always ends with and which no later MMA work
  // hides: y for a whole tile; for a partial one, the slot and, if this CTA is
  // the tile's last contributor, the sum of all contributors in order (the
  // others' slots staged into the A / B ring by bulk copies when they fit).
  // The twelve warps form three groups of four (one per TMEM lane quadrant);
  // group g takes the 32-column chunks g, g + 3, ...  A group writes each
  // chunk's y tile (32 tokens x 128 rows) or slot chunk into shared memory,
  // and one of its threads stores it with one bulk copy.
  tc_fence_before();
  __syncthreads();
  const bool fin_go = __syncthreads_and(fin[0] != 0 && *abort_flag == 0);
  if (fin_go && warp >= 1) {
    tc_fence_after();
    constexpr int kFinThreads = kTcThreads - 32;         // warps 1 .. 13
    constexpr int kGroups = (kTcThreads - 64) / 128;     // groups of warps 2 .. 13
    constexpr int kChunks = BN / 32;
    static_assert(kChunks <= kRedSets, "one arrival barrier per chunk");
    constexpr int kFin0 = 64;                            // bookkeeping thread
    const bool worker = warp >= 2;                       // warp 1 only stages slots
    const bool copier = threadIdx.x == 32;
    const int q = warp & 3, row_l = q * 32 + lane;
    const int grp = worker ? (warp - 2) >> 2 : 0;
    const bool gissuer = worker && threadIdx.x == 64 + 128 * grp;   // the group's bulk-store thread
    const long long u = *fin_u;
    int tile, kb0, kb1;
    seg_of(u, tile, kb0, kb1);
    const int tn = tile % a.tiles_n, tm = tile / a.tiles_n;
    const int buf = fin[1] & 1;
    const uint32_t tq = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN);
    const long long t_first = (long long)tile * a.nkb;
    const bool whole = (u == t_first) && (kb1 == a.nkb);
    const int row = tn * kRowsTile + row_l;
    float s_row = 1.0f;
    if constexpr (GM1) {
      if (worker && row < a.N)
        s_row = __half2float(__ushort_as_half(a.scales[(size_t)(row >> 4) * 16 + scale_slot(row & 15)]));
    }
    // staging: y tiles in the code ring (one per group), slot chunks at the
    // start of the A / B ring (two per group, so a store and the next chunk's
    // writes overlap)
    uint16_t* ybuf = reinterpret_cast<uint16_t*>(sC + grp * (32 * kRowsTile * 2));
    int yput = 0;
    auto put_y = [&](const float (&vals)[32], int c) {
      if (yput++ > 0) {   // the previous store of the group's y buffer has read it
        if (gissuer) bulk_wait_read_all();
        named_bar(3 + grp, 128);
      }
      if (!a.gated) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float o = vals[i] * s_row;
          ybuf[i * kRowsTile + row_l] = BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(o))
                                             : __half_as_ushort(__float2half_rn(o));
        }
      } else {
        // gate rows (lanes 0-15) and up rows (lanes 16-31) of the quadrant
        // give its 16 outputs, columns q 16 .. q 16 + 15 of the tile's 64
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float o = vals[i] * s_row;
          const float up = __shfl_down_sync(0xffffffffu, o, 16);
          if (lane < 16) {
            const float gv = silu(o) * up;
            ybuf[i * (kRowsTile / 2) + q * 16 + lane] =
                BF16 ? __bfloat16_as_ushort(__float2bfloat16_rn(gv)) : __half_as_ushort(__float2half_rn(gv));
          }
        }
      }
      fence_proxy_async();
      named_bar(3 + grp, 128);
      if (gissuer) {
        tma_store_2d(&map_y, ybuf, a.gated ? tn * (kRowsTile / 2) : tn * kRowsTile, tm * BN + c * 32);
        bulk_commit();
      }
    };
    if (whole) {
      if (worker) {
#pragma unroll 1
        for (int c = grp; c < kChunks; c += kGroups) {
          float v[32];
          tmem_ld32(tq + (uint32_t)(c * 32), v);
          put_y(v, c);
        }
      }
    } else {
      const int first = owner_of_tc(t_first, a.units, a.ctas);
      const int nb = owner_of_tc(t_first + a.nkb - 1, a.units, a.ctas) - first + 1;
      const int first_e = ((long long)first * a.units / a.ctas < t_first) ? 1 : 0;
      const int own = b - first;
      if (threadIdx.x == kFin0) {   // have all other contributors arrived?
        unsigned cur;
        asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(cur) : "l"(&a.counters[tile]) : "memory");
        *last_flag = cur == (unsigned)(nb - 1) ? 1 : 0;
      }
      named_bar(2, kFinThreads);
      bool last = *last_flag != 0;
      named_bar(2, kFinThreads);   // last_flag is written again below
      if (!last) {
        if (worker) {
          const int e = (tile == (int)(u_begin / a.nkb)) ? 0 : 1;
          float* slot = a.slots + (size_t)(2 * b + e) * (size_t)(BN * kRowsTile);
          int sput = 0;
#pragma unroll 1
          for (int c = grp; c < kChunks; c += kGroups, ++sput) {
            float v[32];
            tmem_ld32(tq + (uint32_t)(c * 32), v);
            float* sbuf = reinterpret_cast<float*>(sA + (2 * grp + (sput & 1)) * kRedChunk);
            if (sput >= 2) {   // the store of two chunks ago has read this buffer
              if (gissuer) bulk_wait_read_one();
              named_bar(3 + grp, 128);
            }
            // column-major chunk: column i's 128 rows are 512 contiguous bytes
#pragma unroll
            for (int i = 0; i < 32; ++i) sbuf[i * kRowsTile + row_l] = v[i];
            fence_proxy_async();
            named_bar(3 + grp, 128);
            if (gissuer) {
              bulk_store(slot + (size_t)c * 32 * kRowsTile, sbuf, kRedChunk);
              bulk_commit();
            }
          }
          // the slot is written before the release increment (the last
          // contributor reads it with generic loads or bulk copies)
          if (gissuer) {
            bulk_wait_all();
            fence_proxy_async_global();
          }
        }
        named_bar(2, kFinThreads);
        if (threadIdx.x == kFin0) {
          unsigned prev;
          asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(prev) : "l"(&a.counters[tile]) : "memory");
          *last_flag = prev == (unsigned)(nb - 1) ? 1 : 0;
        }
        named_bar(2, kFinThreads);
        last = *last_flag != 0;
      }
      if (last) {
        // own sums from TMEM, the others' from their slots, added in order.
        // Warp 1 stages the others' chunks into the A / B ring (free again:
        // the slot stores above completed) with bulk copies, kSets chunks at
        // a time: chunk c goes to buffer set c mod kSets once the chunk that
        // used the set before has been read by its group.  Each chunk has its
        // own arrival barrier (used once): different groups read different
        // uses of a set, and none of them has seen the set's earlier uses, so
        // a phase parity on a shared barrier could not tell them apart.
        const int P = nb - 1;
        const bool staged = P <= Cfg::RED_BUFS;
        const int kSets = staged ? Cfg::RED_BUFS / P : 1;
        if (staged && copier) {
          unsigned cur;   // the slots' release, observed by this thread too
          asm volatile("ld.acquire.gpu.u32 %0, [%1];" : "=r"(cur) : "l"(&a.counters[tile]) : "memory");
          (void)cur;
          fence_proxy_async_global();
          int issued = 0;
          for (int c = 0; c < kChunks; ++c) {
            const int set = c % kSets;
            if (c >= kSets && !mbar_wait(&red_empty[set], ((c / kSets) - 1) & 1, abort_flag, a.wait_limit))
              break;
            mbar_expect_tx(&red_full[c], (uint32_t)(P * kRedChunk));
            for (int k = 0, j = 0; k < nb; ++k) {
              if (k == own) continue;
              const float* src = a.slots +
                                 (size_t)(2 * (first + k) + (k == 0 ? first_e : 0)) * (BN * kRowsTile) +
                                 (size_t)c * 32 * kRowsTile;
              bulk_load(sA + (size_t)(set * P + j) * kRedChunk, src, kRedChunk, &red_full[c]);
              ++j;
            }
            issued = c + 1;
          }
          // every fill lands before the CTA can exit
          for (int c = 0; c < issued; ++c) drain_wait(&red_full[c], 0);
        }
        if (worker) {
#pragma unroll 1
          for (int c = grp; c < kChunks; c += kGroups) {
            const int set = c % kSets;
            float tv[32], accv[32];
            tmem_ld32(tq + (uint32_t)(c * 32), tv);
#pragma unroll
            for (int i = 0; i < 32; ++i) accv[i] = own == 0 ? tv[i] : 0.0f;
            // a failed wait (the call is giving up) leaves garbage in y, which
            // the error status covers
            if (staged) mbar_wait(&red_full[c], 0, abort_flag, a.wait_limit);
            for (int k = 0, j = 0; k < nb; ++k) {
              if (k == own) {
                if (k != 0) {
#pragma unroll
                  for (int i = 0; i < 32; ++i) accv[i] += tv[i];
                }
                continue;
              }
              float va[32];
              if (staged) {
                const float* pj = reinterpret_cast<const float*>(sA + (size_t)(set * P + j) * kRedChunk) + row_l;
#pragma unroll
                for (int i = 0; i < 32; ++i) va[i] = pj[i * kRowsTile];
              } else {
                const float* pa = a.slots +
                                  (size_t)(2 * (first + k) + (k == 0 ? first_e : 0)) * (BN * kRowsTile) +
                                  (size_t)c * 32 * kRowsTile + row_l;
#pragma unroll
                for (int i = 0; i < 32; ++i) va[i] = __ldcg(pa + (size_t)i * kRowsTile);
              }
#pragma unroll
              for (int i = 0; i < 32; ++i) accv[i] += va[i];
              ++j;
            }
            if (staged) {   // the group is done with the set
              __syncwarp();
              if (lane == 0) mbar_arrive(&red_empty[set]);
            }
            put_y(accv, c);
          }
          if (threadIdx.x == kFin0) a.counters[tile] = 0u;   // ready for the next call
        }
      }
    }
    if (gissuer) bulk_wait_read_all();   // the staging buffers outlive no bulk store
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(Cfg::TMEM_COLS)
                 : "memory");
  }
}

}  // namespace
}  // namespace qk

namespace qk {
namespace {

template <int MODE, int BN, bool SPLIT, int KU>
constexpr size_t tc_smem_bytes() {
  using Cfg = TcCfg<BN, SPLIT, MODE == kLUT, KU>;
  return 1024 + (size_t)Cfg::STAGES * (Cfg::A_BYTES + Cfg::B_BYTES) +
         (size_t)Cfg::CODE_STAGES * (Cfg::CODE_BYTES + Cfg::template META_BYTES<MODE>) +
         (MODE == kLUT ? 256 * 32 * 4 : 0) +
         (2 * Cfg::CODE_STAGES + 3 * Cfg::STAGES + 5 + 2 * kRedSets) * 8 + 64;
}

template <int MODE, bool BF16, int BN, bool GM1, int KU>
cudaError_t launch_tc_t(const CUtensorMap& mx, const CUtensorMap& mw, const CUtensorMap& ms,
                        const CUtensorMap& mz, const CUtensorMap& my, const TcArgs& args, cudaStream_t stream) {
  auto k = tc_kernel<MODE, BF16, BN, GM1, KU>;
  constexpr size_t smem = tc_smem_bytes<MODE, BN, BF16 && (!GM1 || MODE == kLUT), KU>();
  static_assert(smem <= 227 * 1024, "shared memory of the tensor-core kernel");
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return e;
    }
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(args.ctas, 1, 1);
  cfg.blockDim = dim3(kTcThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, mx, mw, ms, mz, my, args);
  if (e != cudaSuccess) cudaGetLastError();   // report it once, here
  return e;
}

template <int MODE, bool BF16, bool GM1>
cudaError_t launch_bn(int bn, int ku, const CUtensorMap& mx, const CUtensorMap& mw, const CUtensorMap& ms,
                      const CUtensorMap& mz, const CUtensorMap& my, const TcArgs& args, cudaStream_t s) {
  // two k blocks per unit (the combinations TcCfg allows)
  constexpr bool kSplit = BF16 && (!GM1 || MODE == kLUT);
  constexpr bool kTable = MODE == kLUT;
  if constexpr (!(kSplit && kTable))
    if (ku == 2 && bn == 64) return launch_tc_t<MODE, BF16, 64, GM1, 2>(mx, mw, ms, mz, my, args, s);
  if constexpr (!kSplit && !kTable) {
    if (ku == 2 && bn == 128) return launch_tc_t<MODE, BF16, 128, GM1, 2>(mx, mw, ms, mz, my, args, s);
    if constexpr (MODE == kSYM)
      if (ku == 2 && bn == 256) return launch_tc_t<MODE, BF16, 256, GM1, 2>(mx, mw, ms, mz, my, args, s);
  }
  if (ku != 1) return cudaErrorInvalidValue;
  if (bn == 64) return launch_tc_t<MODE, BF16, 64, GM1, 1>(mx, mw, ms, mz, my, args, s);
  if (bn == 128) return launch_tc_t<MODE, BF16, 128, GM1, 1>(mx, mw, ms, mz, my, args, s);
  return launch_tc_t<MODE, BF16, 256, GM1, 1>(mx, mw, ms, mz, my, args, s);
}

template <int MODE>
cudaError_t launch_mode(bool bf16, bool gm1, int bn, int ku, const CUtensorMap& mx, const CUtensorMap& mw,
                        const CUtensorMap& ms, const CUtensorMap& mz, const CUtensorMap& my, const TcArgs& args,
                        cudaStream_t s) {
  if (bf16) return gm1 ? launch_bn<MODE, true, true>(bn, ku, mx, mw, ms, mz, my, args, s)
                       : launch_bn<MODE, true, false>(bn, ku, mx, mw, ms, mz, my, args, s);
  return gm1 ? launch_bn<MODE, false, true>(bn, ku, mx, mw, ms, mz, my, args, s)
             : launch_bn<MODE, false, false>(bn, ku, mx, mw, ms, mz, my, args, s);
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// Combinations the tensor path takes: 4-bit codes without the zero-point
// options.  fp16 activations: the operand is fp16((q - z) s) or fp16(T s), one
// rounding of 2^-11.  bf16 activations: per-row scales keep the exact integer
// q - z (the scale multiplies the fp32 result); group scales and tables split
// each weight into bf16 hi + lo parts (SPLIT above).
bool tc_supported(int bits, int mode, bool bf16, int group) {
  (void)bf16;
  (void)group;
  return bits == 4 && !zero_opts(mode);
}

TcPlan plan_tc(int M, int N, int K, int mode, bool bf16, int group, int sms) {
  TcPlan p{};
  p.bn = M <= 64 ? 64 : (M <= 128 ? 128 : 256);
  // two k blocks per unit where the kernel has them: 64 tokens unless a
  // table meets split operands; 128 tokens without a table or a split; 256
  // tokens SYM only, and only for more than one token tile (with a single one,
  // M = 256, the two A / B stages measured 1-2.5% slower than three of 64
  // columns).  A K that ends mid-unit is zero-filled.
  const bool split = bf16 && (group != -1 || mode == kLUT);
  const bool table = mode == kLUT;
  if (p.bn == 64)
    p.ku = (split && table) ? 1 : 2;
  else if (p.bn == 128)
    p.ku = (split || table) ? 1 : 2;
  else
    p.ku = (!split && mode == kSYM && M > 256) ? 2 : 1;
  p.tiles_n = (N + kRowsTile - 1) / kRowsTile;
  p.tiles_m = (M + p.bn - 1) / p.bn;
  p.nkb = (K / kKB + p.ku - 1) / p.ku;
  const long long units = (long long)p.tiles_n * p.tiles_m * p.nkb;
  long long ctas = sms;   // one CTA per SM (shared memory bound)
  if (ctas > units) ctas = units;
  p.ctas = (int)ctas;
  const int tiles = p.tiles_n * p.tiles_m;
  const bool partial = !(units % ctas == 0 && (units / ctas) % p.nkb == 0);
  p.ws_bytes = partial ? ((size_t)tiles * 4 + 255) / 256 * 256 +
                           (size_t)2 * p.ctas * p.bn * kRowsTile * sizeof(float)
                     : 0;
  return p;
}

cudaError_t launch_tc(const Problem& pr, const TcPlan& plan, void* workspace,
                      long long wait_limit, cudaStream_t stream) {
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap mx, mw;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)pr.K, (cuuint64_t)pr.M};
    const cuuint64_t strides[1] = {(cuuint64_t)pr.K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kKB, (cuuint32_t)plan.bn};
    const cuuint32_t es[2] = {1, 1};
    if (encode(&mx, pr.bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
               const_cast<void*>(pr.x), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const int nchunks = pr.K / 64;
    const cuuint64_t dims[2] = {(cuuint64_t)nchunks * 128, (cuuint64_t)(pr.N / 16)};
    const cuuint64_t strides[1] = {(cuuint64_t)nchunks * 512};
    const cuuint32_t box[2] = {(cuuint32_t)(128 * plan.ku), 8};   // the unit's chunks
    const cuuint32_t es[2] = {1, 1};
    if (encode(&mw, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(pr.qweight), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // group scales and zero-points ([N/16][G][16] fp16) as [G 16] x [N/16]: one
  // box = the sx slots of a unit's groups for 8 row blocks (the zero map is
  // only read for ASYM; without zeros it repeats the scale map)
  const int L = pr.group == -1 ? pr.K : pr.group;
  const int G = pr.K / L;
  const int sx = 16 * std::max(1, kKB * plan.ku / L);
  CUtensorMap ms, mz;
  for (int which = 0; which < 2; ++which) {
    const uint16_t* src = (which == 1 && pr.mode == kASYM) ? pr.zl : pr.scales;
    const cuuint64_t dims[2] = {(cuuint64_t)G * 16, (cuuint64_t)(pr.N / 16)};
    const cuuint64_t strides[1] = {(cuuint64_t)G * 32};
    const cuuint32_t box[2] = {(cuuint32_t)sx, 8};
    const cuuint32_t es[2] = {1, 1};
    if (encode(which ? &mz : &ms, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(src),
               dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // y as [M] x [N] (gated: [M] x [N/2]), one box = 32 tokens of a tile's
  // 128 rows (gated: its 64 outputs)
  CUtensorMap my;
  {
    const int ny = pr.gated ? pr.N / 2 : pr.N;
    const cuuint64_t dims[2] = {(cuuint64_t)ny, (cuuint64_t)pr.M};
    const cuuint64_t strides[1] = {(cuuint64_t)ny * 2};
    const cuuint32_t box[2] = {(cuuint32_t)(pr.gated ? kRowsTile / 2 : kRowsTile), 32};
    const cuuint32_t es[2] = {1, 1};
    if (encode(&my, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, pr.y, dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  TcArgs a{};
  a.sx = sx;
  a.scales = pr.scales;
  a.zl = pr.zl;
  a.y = reinterpret_cast<uint16_t*>(pr.y);
  a.M = pr.M;
  a.N = pr.N;
  a.K = pr.K;
  a.gated = pr.gated ? 1 : 0;
  a.L = pr.group == -1 ? pr.K : pr.group;
  a.G = pr.K / a.L;
  a.lg = pr.group == -1 ? 30 : __builtin_ctz((unsigned)pr.group);
  a.nrb = pr.N / 16;
  a.nkb = plan.nkb;
  a.tiles_n = plan.tiles_n;
  a.tiles_m = plan.tiles_m;
  a.tiles = plan.tiles_n * plan.tiles_m;
  a.units = (long long)a.tiles * plan.nkb;
  a.ctas = plan.ctas;
  a.wait_limit = wait_limit;
  if (plan.ws_bytes) {
    const size_t cbytes = ((size_t)a.tiles * 4 + 255) / 256 * 256;
    a.counters = reinterpret_cast<unsigned*>(workspace);
    a.slots = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + cbytes);
  }
  const bool gm1 = pr.group == -1;
  switch (pr.mode) {
    case kSYM: return launch_mode<kSYM>(pr.bf16, gm1, plan.bn, plan.ku, mx, mw, ms, mz, my, a, stream);
    case kASYM: return launch_mode<kASYM>(pr.bf16, gm1, plan.bn, plan.ku, mx, mw, ms, mz, my, a, stream);
    default: return launch_mode<kLUT>(pr.bf16, gm1, plan.bn, plan.ku, mx, mw, ms, mz, my, a, stream);
  }
}

unsigned tc_read_and_clear_error() {
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
  if (v) cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(zero));
  return v;
}

}  // namespace qk
