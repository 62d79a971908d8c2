// Bandwidth-bound decode path for few tokens (M <= 16 per launch slab).
//
// The product here is the quantized-matrix x full-precision-vector product the
// exllama discussion quotes from the GPTQ paper: limited by memory bandwidth,
// with weights de-quantized when needed and activations left unquantized.
// The kernel streams the packed codes exactly once, decodes them in registers
// (bit tricks for SYM/ASYM, a bank-replicated shared-memory pair table for
// LUT) and hands the exact small-integer (or table) values to the tensor cores
// as the A operand of m16n8k16 MMAs, the tokens being the N dimension.  Group
// scales multiply the fp32 partial sums after each group, so the MMA operands
// are exact.
//
// Memory pipeline: every warp owns a ring of shared-memory stages (one row
// tile x 128 columns of K each) and keeps all but one in flight with 16-byte
// cp.async copies (L2 only): a warp-wide copy instruction moves 512
// contiguous bytes of codes, so a stage costs the warp R x 2 code copies, one
// x copy per two token rows and one scale (and zero) copy.  (On this part the
// TMA bulk-copy engine was measured slower than cp.async for these small
// per-warp stages.)  x rows sit at a 288-byte pitch (72 words: rows g and
// g + 1 start 8 banks apart), so that the 8-byte B-fragment loads of each
// half-warp (rows g .. g + 3, 32 bytes per row) hit 32 distinct banks; token
// rows past M are zeroed once and never copied.
//
// Work split (stream-K): the (row tile, K stage) units are divided evenly over
// every warp of a grid of exactly the resident CTAs.  A warp whose range
// covers a whole tile stores y; otherwise it leaves an fp32 partial in the
// workspace and the last warp to finish the tile adds the partials in warp
// order (deterministic) and stores y.  No warp waits for another.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace qk {

// Device error word of the decode path.  Its waits are cp.async group waits,
// which always end, so nothing sets it today; qmm_check_error reads it with
// the tensor path's.
__device__ unsigned g_skinny_error = 0;

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxDevices = 64;
constexpr int kSC = 128;                 // K columns per stage (a "super-chunk"): 8 tiles of 16
constexpr int kTiles = kSC / 16;
constexpr int kXPitch = kSC * 2 + 32;    // bytes per x row in a stage (288: rows 8 banks apart)

// Row blocks (16 rows) per tile.
template <int NT>
constexpr int rb_per_tile() { return 2; }   // the fused gate / up epilogue relies on 2

// Zero-point bytes per row block and stage with zero-point options: up to 16
// zero groups (groups of 8 columns) of 16 fp16 values, or of 16 nibbles; one
// 8-byte record (padded to 16) when the zero group spans the stage.
template <int MODE>
constexpr int kZxRb = MODE == kASYMX ? 512 : (MODE == kASYMQ ? 128 : 16);

struct SkinnyArgs {
  const uint16_t* x;
  const uint8_t* qw;
  const uint16_t* scales;
  const uint16_t* zl;
  uint16_t* y;
  int M, N, K, G, nchunks, nrb, tiles, nsc;
  int lg;              // log2 of the group length; -1 for one group per row
  int lgz, GZ;         // zero-point options: log2 of the zero group, zero groups per row
  int gated;           // 1: rows are alternating 16-row gate / up blocks, y[M, N/2] = silu(gate) up
  int cta_tiles;       // 1: CTA b owns tile b, its warps take the super-chunks round-robin
  int stage_bytes;     // bytes of one ring stage
  long long units;     // tiles * nsc
  int ctas;            // CTAs per slab
  int warps;           // stream-K workers per slab (<= 8 ctas)
  double inv_units;     // 1 / units
  double inv_warps;     // 1 / warps
  float* slots;        // [slabs][2 * warps][rows * tokens]: a warp's first / last partial tile
  unsigned* counters;  // [slabs][tiles]
};

template <int MODE>
constexpr size_t kTabBytes = MODE == kLUT ? 256 * 32 * 4 : 0;

// Stage layout of one warp's ring slot: codes [R][CPS][CB] | x [TOK][288]
// | scales [R][GPS][32 B] | zeros: ASYM [R][GPS][32 B]; zero-point options
// [R][512 B] (the stage's zero groups, fp16 or 4-bit records).
template <int BITS, int MODE, int NT, int TPG>
struct Stage {
  static constexpr int R = rb_per_tile<NT>();
  static constexpr int TOK = 8 * NT;
  static constexpr int CPS = kSC / chunk_cols(BITS);   // chunks per stage
  static constexpr int GPS = kTiles / TPG;             // groups per stage
  static constexpr int CB = chunk_bytes(BITS);         // bytes per chunk
  static constexpr int X_OFF = R * CPS * CB;
  static constexpr int S_OFF = X_OFF + TOK * kXPitch;
  static constexpr int Z_OFF = S_OFF + R * GPS * 32;
  static constexpr int BYTES =
      Z_OFF + (MODE == kASYM ? R * GPS * 32 : (zero_opts(MODE) ? R * kZxRb<MODE> : 0));
  static_assert(BYTES % 16 == 0, "stages must stay 16-byte aligned");
};

// Ring depth per warp (stages in flight = depth - 1): 3 for one token tile
// where the 8 warps' rings still fit two CTAs per SM (228 KB, 1 KB reserved
// per CTA), else 2.  DEEP kernels run one CTA per SM (problems with at most
// one row tile per SM): as deep a ring as fits 227 KB, at most 6, so that a
// warp's whole share of a small matrix is requested at once.
template <int BITS, int MODE, int NT, int TPG, bool DEEP = false>
constexpr int ring_stages() {
  if constexpr (DEEP) {
    constexpr int tab = MODE == kLUT ? 256 * 32 * 4 : 0;
    constexpr int s = (227 * 1024 - tab) / (kWarps * Stage<BITS, MODE, NT, TPG>::BYTES);
    return s > 6 ? 6 : s;
  }
  if (NT != 1) return 2;
  if (MODE == kSYM || MODE == kASYM) return 3;
  if ((MODE == kASYMQ || MODE == kASYMQ1) &&
      2 * (3 * kWarps * Stage<BITS, MODE, NT, TPG>::BYTES + 1024) <= 228 * 1024)
    return 3;
  return 2;
}

// floor(a / d) for 0 <= a < 2^53, d > 0, from a double estimate (inv_d =
// 1 / d) and exact integer corrections: 64-bit integer division is a long
// software sequence on the GPU.
__device__ __forceinline__ long long floor_div(long long a, long long d, double inv_d) {
  long long q = (long long)((double)a * inv_d);
  if (q * d > a) --q;
  else if ((q + 1) * d <= a) ++q;
  return q;
}

// Worker of the stream-K range that holds unit u (worker b's range starts at
// floor(b U / W)): the largest b with b U < (u + 1) W.
__device__ __forceinline__ int owner_of(long long u, long long U, long long W, double inv_U) {
  return (int)floor_div((u + 1) * W - 1, U, inv_U);
}

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ void sts128_zero(uint32_t a) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(a), "r"(0u) : "memory");
}
// 8-byte asynchronous copy global -> shared; `valid` false writes zeros.
__device__ __forceinline__ void cp_async8(uint32_t saddr, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(saddr), "l"(src),
               "r"(valid ? 8 : 0)
               : "memory");
}
// 16-byte asynchronous copy global -> shared, L2 only; `valid` false writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async16_all(uint32_t saddr, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// D = A . B with a zero accumulator (first tile of a group).
template <bool BF16>
__device__ __forceinline__ void mma_16816_first(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                uint32_t b1) {
  const float z = 0.0f;
  if constexpr (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
  }
}

template <int BITS, int MODE, bool BF16, int NT, int TPG, bool DEEP>
__global__ void __launch_bounds__(kThreads, (DEEP || NT > 2) ? 1 : 2) skinny_kernel(const SkinnyArgs a) {
  using St = Stage<BITS, MODE, NT, TPG>;
  constexpr int S = ring_stages<BITS, MODE, NT, TPG, DEEP>();
  constexpr int R = St::R;
  constexpr int TOK = St::TOK;
  constexpr int CPS = St::CPS;
  constexpr int GPS = St::GPS;
  constexpr int NACC = R * NT * 4;        // fp32 values per lane per tile

  extern __shared__ __align__(128) unsigned char smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int slab = blockIdx.y;
  const int m_base = slab * TOK;
  const int mrows = min(TOK, a.M - m_base);   // token rows of this slab (>= 1)
  const int n = a.nsc;
  // this warp's stream-K range of (tile, super-chunk) units
  const int gw = blockIdx.x * kWarps + warp;
  const long long W = a.warps;
  int ub = 0, ue = 0;   // unit indices: at most 2^15 tiles x 2^13 stages, 32 bits
  // CTA-per-tile mode (problems with few row tiles): CTA b owns tile b, warp w
  // takes its super-chunks w, w + 8, ... and the warps' sums are added in
  // shared memory; otherwise warp-level stream-K over contiguous unit ranges
  const bool ctile = a.cta_tiles != 0;
  const int sc_step = ctile ? kWarps : 1;
  if (ctile) {
    ue = warp < n ? (n - warp + kWarps - 1) / kWarps : 0;
  } else if (gw < W) {
    ub = (int)floor_div((long long)gw * a.units, W, a.inv_warps);
    ue = (int)floor_div((long long)(gw + 1) * a.units, W, a.inv_warps);
  }
  const int lg = a.lg;

  unsigned char* tabp = smem;
  unsigned char* ring = smem + kTabBytes<MODE> + (size_t)warp * S * St::BYTES;
  const uint32_t ring_s = smem_u32(ring);

  // ---- per-warp setup: stage barriers; token rows past M zeroed in every
  // stage (they are never copied, and the fragment loads read all TOK rows)
  for (int s = 0; s < S; ++s) {
    const uint32_t xb = ring_s + s * St::BYTES + St::X_OFF + mrows * kXPitch;
    for (int i = lane; i < (TOK - mrows) * (kXPitch / 16); i += 32) sts128_zero(xb + 16 * i);
  }
  __syncwarp();

  pdl_wait();                 // inputs of this call may come from the previous grid
  pdl_launch_dependents();    // let the next grid get resident while this one runs

  if constexpr (MODE == kLUT) {
    // Pair table, replicated so that every lane reads its own bank.
    //  4-bit: entry[byte] = (T[lo nibble], T[hi nibble]), 32 copies of 4 bytes.
    //  2-bit: entry[byte] = 4 values from the 2-bit fields, 16 copies of 8 bytes.
    // With bf16 activations the fp16 entries do not fit bf16: each entry is
    // split exactly into hi = bf16(T) and lo = bf16(T - hi) (T - hi has at most
    // 3 significant bits), the entry doubles in size and the copies halve.
    uint32_t* tab = reinterpret_cast<uint32_t*>(smem);
    uint32_t hv[16], lv[16];
#pragma unroll
    for (int i = 0; i < (1 << BITS); ++i) {
      const uint16_t h = a.zl[i];
      if constexpr (BF16) {
        const float f = __half2float(__ushort_as_half(h));
        const __nv_bfloat16 hi = __float2bfloat16_rn(f);
        hv[i] = __bfloat16_as_ushort(hi);
        lv[i] = __bfloat16_as_ushort(__float2bfloat16_rn(f - __bfloat162float(hi)));
      } else {
        hv[i] = h;
        lv[i] = 0;
      }
    }
    //  3-bit: entry[6-bit field] = the pair (member 0 in bits 0..2, member 1
    //  in bits 3..5), 64 entries.
    constexpr int VALS = BITS == 2 ? 4 : 2;              // values per entry
    constexpr int WORDS = (BF16 ? 2 : 1) * VALS / 2;     // 32-bit words per entry copy
    constexpr int COPIES = 32 / WORDS;
    constexpr int NENT = BITS == 3 ? 64 : 256;
    for (int i = threadIdx.x; i < NENT * COPIES; i += kThreads) {
      const int e = i / COPIES;
      uint32_t v[4];
      if constexpr (BITS == 3) {
        v[0] = e & 7;
        v[1] = e >> 3;
      } else {
#pragma unroll
        for (int k = 0; k < VALS; ++k) v[k] = BITS == 4 ? ((e >> (4 * k)) & 15) : ((e >> (2 * k)) & 3);
      }
#pragma unroll
      for (int w = 0; w < VALS / 2; ++w) {
        tab[i * WORDS + w] = hv[v[2 * w]] | (hv[v[2 * w + 1]] << 16);
        if constexpr (BF16) tab[i * WORDS + VALS / 2 + w] = lv[v[2 * w]] | (lv[v[2 * w + 1]] << 16);
      }
    }
    __syncthreads();
  }

  if (ub >= ue && !ctile) return;   // no units (spare warps of the last CTA)

  const int nsc_full = a.K / kSC;         // super-chunks with no column past K

  // ---- copies of super-chunk (tile, sc) into ring stage st with 16-byte
  // cp.async pieces: per lane, R x CPS code pieces, one x piece per two token
  // rows, one scale (and zero) piece
  const int xrow0 = lane >> 4, xp = lane & 15;
  const int xi_n = (mrows + 1) >> 1;                       // warp-uniform
  const uint32_t xdst0 = St::X_OFF + xrow0 * kXPitch + xp * 16;
  // the lane's x sources, one per pair of token rows (rows past M are clamped
  // and copied with size 0); 32-token tiles recompute them instead of holding
  // 16 pointers
  constexpr bool kWide = NT > 2;
  constexpr int XP = (TOK + 1) / 2;
  const uint16_t* xsrc[kWide ? 1 : XP];
  auto xsrc_at = [&](int i) -> const uint16_t* {
    if constexpr (kWide)
      return a.x + (size_t)min(m_base + xrow0 + 2 * i, a.M - 1) * a.K + xp * 8;
    else
      return xsrc[i];
  };
  if constexpr (!kWide) {
#pragma unroll
    for (int i = 0; i < XP; ++i) {
      const int m = min(m_base + xrow0 + 2 * i, a.M - 1);
      xsrc[i] = a.x + (size_t)m * a.K + xp * 8;
    }
  }
  // zero-point options: bytes per zero group record (16 fp16 or 16 nibbles),
  // zero groups per stage, bytes of a row block's zeros per stage
  constexpr int zrec = MODE == kASYMX ? 32 : 8;
  const int zps = (MODE == kASYMQ1 || a.lgz >= 7) ? 1 : (kSC >> a.lgz);
  const uint8_t* zbytes = reinterpret_cast<const uint8_t*>(a.zl);
  // this lane's zero group inside a tile: columns 4t .. 4t + 3 lie in the
  // tile's half t / 2 (groups of 8 or more columns never split a half)
  const int zhalf = 8 * (t >> 1);
  const int lgzc = a.lgz < 7 ? a.lgz : 7;
  // this lane's zero-record pieces of a stage (at most two: pieces lane and
  // lane + 32 of R * zppr), row block and piece index fixed for the whole call
  constexpr int zppz = zrec == 32 ? 2 : 1;               // pieces per record
  const int zppr = zps * zppz;                           // pieces per row block (<= 32)
  int zr[2], zpc[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    zr[h] = (lane + 32 * h) / zppr;
    zpc[h] = lane + 32 * h - zr[h] * zppr;
  }
  const bool sq_on = lane < R * GPS * 2;
  const int sq_r = lane / (2 * GPS), sq_k = (lane >> 1) % GPS, sq_h = lane & 1;
  // steady-state copy parameters fixed for the call: source bytes of this
  // lane's x pieces (16, or 0 for a token row past M, which reads as zeros)
  // and the shift from a stage's first column to its first group
  uint32_t xsz[kWide ? 1 : XP];
  if constexpr (!kWide) {
#pragma unroll
    for (int i = 0; i < XP; ++i) xsz[i] = xrow0 + 2 * i < mrows ? 16u : 0u;
  }
  auto xsz_at = [&](int i) -> bool {
    if constexpr (kWide)
      return xrow0 + 2 * i < mrows;
    else
      return xsz[i] != 0;
  };
  const int lgs = lg < 0 ? 31 : lg;
  const uint8_t* cbase[R];
  bool rok[R];
  bool tile_ok = true;
  const uint16_t* sbase = a.scales;
  bool srok = false;
  int pf_tile = -1;
  auto set_tile = [&](int tile) {
    pf_tile = tile;
    tile_ok = true;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int rb = tile * R + r;
      rok[r] = rb < a.nrb;
      tile_ok = tile_ok && rok[r];
      cbase[r] = a.qw + (size_t)(rok[r] ? rb : 0) * a.nchunks * St::CB + lane * 16;
    }
    const int rbs = tile * R + sq_r;
    srok = sq_on && rbs < a.nrb;
    sbase = a.scales + (size_t)(srok ? rbs : 0) * a.G * 16 + sq_h * 8;
  };
  auto issue_zeros = [&](int tile, int k0, uint32_t base) {
    // the zps zero groups that meet the stage's 128 columns, per row block:
    // fp16 records (32 bytes) in two 16-byte pieces each, 4-bit records
    // (8 bytes) in one 8-byte piece each; a piece never spans two records,
    // so its validity is its record's and its source stays aligned
    const int zf = k0 >> a.lgz;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (lane + 32 * h < R * zppr) {   // warp-uniform for h = 0 once zppr >= 16
        const int r = zr[h], pc = zpc[h];
        const int rb = tile * R + r;
        const int zi = zf + pc / zppz;
        const bool ok = rb < a.nrb && zi < a.GZ;
        const uint8_t* src = zbytes + ((size_t)rb * a.GZ + zi) * zrec + (pc % zppz) * 16;
        if constexpr (zrec == 32)
          cp_async16(base + St::Z_OFF + r * kZxRb<MODE> + pc * 16, ok ? src : zbytes, ok);
        else
          cp_async8(base + St::Z_OFF + r * kZxRb<MODE> + pc * 8, ok ? src : zbytes, ok);
      }
    }
  };
  auto issue = [&](int tile, int sc, int st) {
    if (tile != pf_tile) set_tile(tile);
    const uint32_t base = ring_s + st * St::BYTES;
    const int k0 = sc * kSC;
    // a row block's codes of the stage: CPS chunks, contiguous, copied as
    // 512-byte warp-wide pieces (the last one partial for 3-bit chunks)
    constexpr int RB_BYTES = CPS * St::CB;
    constexpr int PIECES = (RB_BYTES + 511) / 512;
    if (tile_ok && sc < nsc_full) {
      // steady state (a whole stage of a tile inside N and K): every copy is
      // in bounds, no per-piece checks; 32-bit offsets from the row-block bases
      const uint32_t cofs = (uint32_t)sc * RB_BYTES;
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int i = 0; i < PIECES; ++i)
          if (RB_BYTES % 512 == 0 || i * 512 + lane * 16 < RB_BYTES)
            cp_async16_all(base + r * RB_BYTES + i * 512 + lane * 16, cbase[r] + cofs + i * 512);
#pragma unroll
      for (int i = 0; i < XP; ++i)
        if (i < xi_n)   // warp-uniform
          cp_async16(base + xdst0 + 2 * i * kXPitch, xsrc_at(i) + k0, xsz_at(i));
      if (sq_on) {
        const int off = ((k0 >> lgs) + sq_k) << 4;
        cp_async16(base + St::S_OFF + lane * 16, sbase + off, srok);
        if constexpr (MODE == kASYM)
          cp_async16(base + St::Z_OFF + lane * 16, a.zl + (sbase - a.scales) + off, srok);
      }
    } else {
      // a tile with row blocks past N, or the stage that K ends in: every
      // piece checked, the missing ones zero-filled
      const bool full = sc < nsc_full;
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int i = 0; i < PIECES; ++i) {
          if (RB_BYTES % 512 != 0 && i * 512 + lane * 16 >= RB_BYTES) continue;
          const int c = sc * CPS + (i * 512) / St::CB;      // chunk of the piece
          const bool ok = rok[r] && c < a.nchunks;
          cp_async16(base + r * RB_BYTES + i * 512 + lane * 16,
                     cbase[r] + (ok ? (size_t)sc * RB_BYTES + i * 512 : 0), ok);
        }
      const bool xk = full || k0 + xp * 8 < a.K;
#pragma unroll
      for (int i = 0; i < XP; ++i) {
        if (i < xi_n) {   // warp-uniform
          const bool ok = xrow0 + 2 * i < mrows && xk;
          cp_async16(base + xdst0 + 2 * i * kXPitch, xsrc_at(i) + (ok ? k0 : 0), ok);
        }
      }
      if (sq_on) {
        const int gi = (lg < 0 ? 0 : (k0 >> lg)) + sq_k;
        const bool ok = srok && gi < a.G;
        const size_t off = ok ? (size_t)gi * 16 : 0;
        cp_async16(base + St::S_OFF + lane * 16, sbase + off, ok);
        if constexpr (MODE == kASYM)
          cp_async16(base + St::Z_OFF + lane * 16, a.zl + (sbase - a.scales) + off, ok);
      }
    }
    if constexpr (zero_opts(MODE)) issue_zeros(tile, k0, base);
  };

  // ---- prologue: S - 1 super-chunks in flight (the warp's own units, in
  // order: consecutive super-chunks, then the next tile)
  int pf_u = ub;
  // the warp's first tile and super-chunk (ub < 2^31)
  const int tb = ctile ? (int)blockIdx.x : (int)((unsigned)ub / (unsigned)n);
  const int sb = ctile ? warp : ub - tb * n;
  int pf_t = tb, pf_s = sb;
  auto pf_next = [&]() {
    ++pf_u;
    pf_s += sc_step;
    if (pf_s >= n) {
      pf_s -= n;
      ++pf_t;
    }
  };
#pragma unroll
  for (int s = 0; s < S - 1; ++s) {
    if (pf_u < ue) {
      issue(pf_t, pf_s, s);
      pf_next();
    }
    cp_async_commit();
  }

  int tile = tb, sc = sb;
  int u = ub;
  // the current tile segment's sums; in CTA-per-tile mode they stay this
  // warp's contribution to the CTA's one tile after the loop
  float acc[R][NT][4];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[r][nt][i] = 0.0f;
  int st_c = 0;                          // ring stage being computed
  int st_f = S - 1;                      // ring stage being filled

  // y for the lane's fragments of `tile` (fused gate: silu(gate) * up)
  auto store_y = [&](const float (&acc)[R][NT][4], int tile) {
    if (a.gated) {
      // the tile's two row blocks are gate block `tile` (r = 0) and up block
      // `tile` (r = 1): each lane holds both values of its outputs
      const int ny = a.N >> 1;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int col = tile * 16 + g + 8 * (i >> 1);
          const int m = m_base + 8 * nt + 2 * t + (i & 1);
          if (col < ny && m < a.M) {
            const float v = silu(acc[0][nt][i]) * acc[1][nt][i];
            if constexpr (BF16)
              a.y[(size_t)m * ny + col] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            else
              a.y[(size_t)m * ny + col] = __half_as_ushort(__float2half_rn(v));
          }
        }
    } else {
      // fragment (r, nt, i) of this lane: row (tile R + r) 16 + g + 8 (i / 2),
      // token m_base + 8 nt + 2 t + (i % 2)
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int row = (tile * R + r) * 16 + g + 8 * (i >> 1);
            const int m = m_base + 8 * nt + 2 * t + (i & 1);
            if (row < a.N && m < a.M) {
              const float v = acc[r][nt][i];
              if constexpr (BF16)
                a.y[(size_t)m * a.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
              else
                a.y[(size_t)m * a.N + row] = __half_as_ushort(__float2half_rn(v));
            }
          }
    }
  };

  while (u < ue) {
    // this warp's segment of the tile: super-chunks [s0, s1)
    const int s0 = sc;
    const int tile_end = (tile + 1) * n;
    const int s1 = ctile ? n : (ue < tile_end ? ue : tile_end) - tile * n;

#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[r][nt][i] = 0.0f;

    for (; sc < s1; sc += sc_step, ++u) {
      // keep the ring full: the stage refilled here was drained last iteration
      if (pf_u < ue) {
        issue(pf_t, pf_s, st_f);
        pf_next();
      }
      cp_async_commit();
      cp_async_wait<S - 1>();
      __syncwarp();

      const unsigned char* st = ring + st_c * St::BYTES;
      const bool full = sc < nsc_full;   // else the stage holds only its first 64 columns

      // B fragments (tokens) of the eight tiles.  The packed layout gives lane
      // (g, t) the columns 4t .. 4t + 3 of each 16-column tile (the MMA's k
      // order permuted the same way for both operands), so its b0, b1 are the
      // 8 contiguous bytes at column 16 j + 4 t of token row g.
      // (all eight tiles' fragments up front for 8 and 16 tokens; 32 tokens
      // load each tile's when it is used, to keep the registers for the sums)
      const unsigned char* xa = st + St::X_OFF + g * kXPitch + 8 * t;
      uint32_t xf[kWide ? 1 : kTiles][NT][2];
      auto load_xf = [&](int j, uint32_t (&f)[NT][2]) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint2 v = *reinterpret_cast<const uint2*>(xa + nt * 8 * kXPitch + 32 * j);
          f[nt][0] = v.x;
          f[nt][1] = v.y;
        }
      };
      if constexpr (!kWide) {
#pragma unroll
        for (int j = 0; j < kTiles; ++j) load_xf(j, xf[j]);
      }
      // one 4-bit zero record per stage: each row block's (z_g, z_g8) pairs once
      uint32_t zq1[MODE == kASYMQ1 ? R : 1][2];
      if constexpr (MODE == kASYMQ1) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t b = st[St::Z_OFF + r * kZxRb<MODE> + g];
          const uint32_t zw =
              BF16 ? bsub2_u(lop3_and_or(b | (b << 12), 0x000F000Fu, 0x43004300u), 0x43004300u)
                   : hsub2_u(lop3_and_or(b | (b << 12), 0x000F000Fu, 0x64006400u), 0x64006400u);
          zq1[r][0] = __byte_perm(zw, 0, 0x1010);
          zq1[r][1] = __byte_perm(zw, 0, 0x3232);
        }
      }
      float gacc[R][NT][4];
      uint4 cw[R];
      uint32_t cw3[BITS == 3 ? R : 1][6];   // 3-bit: the lane's 24 bytes of the stage

#pragma unroll
      for (int j = 0; j < kTiles; ++j) {
        const int grp = j / TPG;            // group within the stage (compile-time)
        uint32_t xfw[NT][2];
        if constexpr (kWide) load_xf(j, xfw);
        const uint32_t(&xj)[NT][2] = *(kWide ? &xfw : &xf[kWide ? 0 : j]);
        // the lane's 16 code bytes of chunk j / 4 (4-bit) or of the stage (2-bit)
        if constexpr (BITS == 3) {
          if (j == 0) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
              for (int q = 0; q < 3; ++q) {
                const uint2 v = *reinterpret_cast<const uint2*>(st + r * St::CB + lane * 24 + 8 * q);
                cw3[r][2 * q] = v.x;
                cw3[r][2 * q + 1] = v.y;
              }
          }
        } else if ((BITS == 4 && (j & 3) == 0) || j == 0) {
#pragma unroll
          for (int r = 0; r < R; ++r)
            cw[r] = *reinterpret_cast<const uint4*>(st + (r * CPS + (BITS == 4 ? (j >> 2) : 0)) * 512 +
                                                    lane * 16);
        }
        if (full || j < 4) {
#pragma unroll
          for (int r = 0; r < R; ++r) {
            uint32_t af[4], aflo[4];
            if constexpr (BITS == 4) {
              // tile j: chunk j / 4 of the stage, word j % 4 of the lane
              const uint32_t w = (&cw[r].x)[j & 3];
              if constexpr (MODE == kSYM) {
                decode_int4<BF16, 8>(w, af);
              } else if constexpr (MODE == kASYM) {
                decode_int4<BF16, 0>(w, af);
                uint32_t zw = *reinterpret_cast<const uint32_t*>(st + St::Z_OFF +
                                                                 (r * GPS + grp) * 32 + 4 * g);
                if constexpr (BF16) {
                  const float2 zf = __half22float2(*reinterpret_cast<const __half2*>(&zw));
                  zw = pack2<true>(zf.x, zf.y);
                }
                sub_zero<BF16>(__byte_perm(zw, 0, 0x1010), __byte_perm(zw, 0, 0x3232), af);
              } else if constexpr (MODE == kASYMQ1) {
                decode_int4<BF16, 0>(w, af);
                sub_zero<BF16>(zq1[r][0], zq1[r][1], af);
              } else if constexpr (zero_opts(MODE)) {
                decode_int4<BF16, 0>(w, af);
                // zero group of (tile j, this lane's half) inside the stage
                const int zl = (16 * j + zhalf) >> lgzc;
                const unsigned char* zp = st + St::Z_OFF + r * kZxRb<MODE>;
                uint32_t zw;
                if constexpr (MODE == kASYMX) {
                  zw = *reinterpret_cast<const uint32_t*>(zp + zl * 32 + 4 * g);
                  if constexpr (BF16) {
                    const float2 zf2 = __half22float2(*reinterpret_cast<const __half2*>(&zw));
                    zw = pack2<true>(zf2.x, zf2.y);
                  }
                } else {
                  // rows g, g + 8 = the low and high nibble of byte g of the record
                  const uint32_t b = zp[zl * 8 + g];
                  if constexpr (BF16)   // (128 + z) - 128 in bf16, exact
                    zw = bsub2_u(lop3_and_or(b | (b << 12), 0x000F000Fu, 0x43004300u), 0x43004300u);
                  else                  // (1024 + z) - 1024 in fp16, exact
                    zw = hsub2_u(lop3_and_or(b | (b << 12), 0x000F000Fu, 0x64006400u), 0x64006400u);
                }
                sub_zero<BF16>(__byte_perm(zw, 0, 0x1010), __byte_perm(zw, 0, 0x3232), af);
              } else if constexpr (!BF16) {
                const uint32_t l4 = (uint32_t)lane << 2;
                af[0] = *reinterpret_cast<const uint32_t*>(tabp + lop3_and_or(w << 7, 0x7F80u, l4));
                af[1] = *reinterpret_cast<const uint32_t*>(tabp + lop3_and_or(w >> 1, 0x7F80u, l4));
                af[2] = *reinterpret_cast<const uint32_t*>(tabp + lop3_and_or(w >> 9, 0x7F80u, l4));
                af[3] = *reinterpret_cast<const uint32_t*>(tabp + lop3_and_or(w >> 17, 0x7F80u, l4));
              } else {
                // (hi, lo) per pair: 8-byte entries, 16 copies
                const uint32_t l8 = (uint32_t)(lane & 15) << 3;
                const uint2 e0 = *reinterpret_cast<const uint2*>(tabp + lop3_and_or(w << 7, 0x7F80u, l8));
                const uint2 e1 = *reinterpret_cast<const uint2*>(tabp + lop3_and_or(w >> 1, 0x7F80u, l8));
                const uint2 e2 = *reinterpret_cast<const uint2*>(tabp + lop3_and_or(w >> 9, 0x7F80u, l8));
                const uint2 e3 = *reinterpret_cast<const uint2*>(tabp + lop3_and_or(w >> 17, 0x7F80u, l8));
                af[0] = e0.x; af[1] = e1.x; af[2] = e2.x; af[3] = e3.x;
                aflo[0] = e0.y; aflo[1] = e1.y; aflo[2] = e2.y; aflo[3] = e3.y;
              }
            } else if constexpr (BITS == 3) {
              // 3-bit LUT: pair p of tile j is the 6-bit field at bit 24 j + 6 p
              // of the lane's 192-bit string, an index into the 64-entry pair
              // table (entries 128 bytes apart): one funnel shift brings it to
              // bits 7..12
#pragma unroll
              for (int p = 0; p < 4; ++p) {
                const int b = 24 * j + 6 * p, wi = b >> 5, sb = b & 31;
                const uint32_t lo = cw3[r][wi], hi = wi + 1 < 6 ? cw3[r][wi + 1] : 0u;
                const uint32_t f = sb >= 7 ? __funnelshift_r(lo, hi, sb - 7) : lo << (7 - sb);
                if constexpr (!BF16) {
                  const uint32_t l4 = (uint32_t)lane << 2;
                  af[p] = *reinterpret_cast<const uint32_t*>(tabp + lop3_and_or(f, 0x1F80u, l4));
                } else {
                  const uint32_t l8 = (uint32_t)(lane & 15) << 3;
                  const uint2 e = *reinterpret_cast<const uint2*>(tabp + lop3_and_or(f, 0x1F80u, l8));
                  af[p] = e.x;
                  aflo[p] = e.y;
                }
              }
            } else {
              // 2-bit LUT: word j/2 of the lane, bytes 2 (j % 2) and 2 (j % 2) + 1
              const uint32_t w = (&cw[r].x)[j >> 1];
              const int sh = 16 * (j & 1);
              const uint32_t s0w = sh >= 7 ? (w >> (sh - 7)) : (w << 7);
              const uint32_t s1w = w >> (sh + 1);
              if constexpr (!BF16) {
                const uint32_t l8 = (uint32_t)(lane & 15) << 3;
                const uint2 e0 = *reinterpret_cast<const uint2*>(tabp + lop3_and_or(s0w, 0x7F80u, l8));
                const uint2 e1 = *reinterpret_cast<const uint2*>(tabp + lop3_and_or(s1w, 0x7F80u, l8));
                af[0] = e0.x; af[1] = e0.y; af[2] = e1.x; af[3] = e1.y;
              } else {
                // (hi hi, lo lo) per byte: 16-byte entries, 8 copies
                const uint32_t l16 = (uint32_t)(lane & 7) << 4;
                const uint4 e0 = *reinterpret_cast<const uint4*>(tabp + lop3_and_or(s0w, 0x7F80u, l16));
                const uint4 e1 = *reinterpret_cast<const uint4*>(tabp + lop3_and_or(s1w, 0x7F80u, l16));
                af[0] = e0.x; af[1] = e0.y; af[2] = e1.x; af[3] = e1.y;
                aflo[0] = e0.z; aflo[1] = e0.w; aflo[2] = e1.z; aflo[3] = e1.w;
              }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              if (j % TPG == 0)
                mma_16816_first<BF16>(gacc[r][nt], af, xj[nt][0], xj[nt][1]);
              else
                mma_16816<BF16>(gacc[r][nt], af, xj[nt][0], xj[nt][1]);
              if constexpr (MODE == kLUT && BF16)
                mma_16816<BF16>(gacc[r][nt], aflo, xj[nt][0], xj[nt][1]);
            }
          }
        }
        // the group ends after this tile (position fixed at compile time): fold
        // its sums into acc with its scales (a group wholly past K is skipped)
        if ((j + 1) % TPG == 0 && (full || j + 1 - TPG < 4)) {
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const uint32_t sw = *reinterpret_cast<const uint32_t*>(st + St::S_OFF +
                                                                   (r * GPS + grp) * 32 + 4 * g);
            const float2 s = __half22float2(*reinterpret_cast<const __half2*>(&sw));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              acc[r][nt][0] = fmaf(s.x, gacc[r][nt][0], acc[r][nt][0]);
              acc[r][nt][1] = fmaf(s.x, gacc[r][nt][1], acc[r][nt][1]);
              acc[r][nt][2] = fmaf(s.y, gacc[r][nt][2], acc[r][nt][2]);
              acc[r][nt][3] = fmaf(s.y, gacc[r][nt][3], acc[r][nt][3]);
            }
          }
        }
      }
      __syncwarp();   // every lane is done with this stage before it is refilled
      st_c = st_c + 1 == S ? 0 : st_c + 1;
      st_f = st_f + 1 == S ? 0 : st_f + 1;
    }

    float* outv = &acc[0][0][0];
    if (ctile) break;
    // ---- this warp's result for the tile segment: store y (whole tile) or
    // hand a partial to the last warp that finishes the tile
    const bool whole = s0 == 0 && s1 == n;
    bool store = true;
    if (!whole) {
      const long long t_first = (long long)tile * n;
      const int first = owner_of(t_first, a.units, W, a.inv_units);
      const int nb = owner_of(t_first + n - 1, a.units, W, a.inv_units) - first + 1;
      // `first` started before this tile (its range start floor(first U / W)
      // is below t_first) exactly when first U < t_first W
      const int first_e = ((long long)first * a.units < t_first * W) ? 1 : 0;
      // slot 2 gw + e, e = 1 when the tile is not the warp's first; of the
      // contributors only `first` can have e = 1
      const int e = (tile == tb) ? 0 : 1;
      float* slots = a.slots + (size_t)slab * 2 * W * (NACC * 32);
      float4* mine = reinterpret_cast<float4*>(slots + (size_t)(2 * gw + e) * (NACC * 32) + lane * NACC);
#pragma unroll
      for (int i = 0; i < NACC / 4; ++i)
        mine[i] = make_float4(outv[4 * i], outv[4 * i + 1], outv[4 * i + 2], outv[4 * i + 3]);
      __syncwarp();
      unsigned* counter = a.counters + (size_t)slab * a.tiles + tile;
      unsigned prev = 0;
      if (lane == 0)
        asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(prev) : "l"(counter) : "memory");
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev != (unsigned)(nb - 1)) {
        store = false;
      } else {
#pragma unroll
        for (int i = 0; i < NACC; ++i) outv[i] = 0.0f;
        constexpr int KB = NT == 1 ? 4 : (NT == 2 ? 2 : 1);   // contributors loaded at a time
        for (int k0 = 0; k0 < nb; k0 += KB) {
          float4 v[KB][NACC / 4];
#pragma unroll
          for (int kk = 0; kk < KB; ++kk) {
            const int k = k0 + kk;
            if (k < nb) {
              const float4* src = reinterpret_cast<const float4*>(
                  slots + (size_t)(2 * (first + k) + (k == 0 ? first_e : 0)) * (NACC * 32) + lane * NACC);
#pragma unroll
              for (int i = 0; i < NACC / 4; ++i) v[kk][i] = __ldcg(src + i);
            }
          }
#pragma unroll
          for (int kk = 0; kk < KB; ++kk) {
            if (k0 + kk < nb) {
#pragma unroll
              for (int i = 0; i < NACC / 4; ++i) {
                outv[4 * i] += v[kk][i].x;
                outv[4 * i + 1] += v[kk][i].y;
                outv[4 * i + 2] += v[kk][i].z;
                outv[4 * i + 3] += v[kk][i].w;
              }
            }
          }
        }
        if (lane == 0) *counter = 0u;   // ready for the next call
      }
    }
    if (store) store_y(acc, tile);
    ++tile;
    sc = 0;
  }
  cp_async_wait<0>();   // nothing may still land in shared memory after exit
  if (ctile) {
    // the CTA's warps add their sums in warp order (deterministic) through
    // shared memory (the rings are free once every warp is past this barrier)
    __syncthreads();
    float* red = reinterpret_cast<float*>(smem + kTabBytes<MODE>);   // [kWarps][32][NACC]
    float4* mine = reinterpret_cast<float4*>(red + ((size_t)warp * 32 + lane) * NACC);
    const float* part = &acc[0][0][0];
#pragma unroll
    for (int i = 0; i < NACC / 4; ++i)
      mine[i] = make_float4(part[4 * i], part[4 * i + 1], part[4 * i + 2], part[4 * i + 3]);
    __syncthreads();
    if (warp == 0) {
      float sum[R][NT][4];
      float* outv = &sum[0][0][0];
#pragma unroll
      for (int i = 0; i < NACC; ++i) outv[i] = 0.0f;
      for (int w = 0; w < kWarps; ++w) {
        const float4* src = reinterpret_cast<const float4*>(red + ((size_t)w * 32 + lane) * NACC);
#pragma unroll
        for (int i = 0; i < NACC / 4; ++i) {
          const float4 v = src[i];
          outv[4 * i] += v.x;
          outv[4 * i + 1] += v.y;
          outv[4 * i + 2] += v.z;
          outv[4 * i + 3] += v.w;
        }
      }
      store_y(sum, (int)blockIdx.x);
    }
  }
}

template <int BITS, int MODE, int NT, int TPG, bool DEEP>
constexpr size_t smem_bytes() {
  using St = Stage<BITS, MODE, NT, TPG>;
  constexpr int S = ring_stages<BITS, MODE, NT, TPG, DEEP>();
  return kTabBytes<MODE> + (size_t)kWarps * S * St::BYTES;
}

// Opts the kernel into `smem` bytes of dynamic shared memory (once per device)
// and returns its resident CTAs per SM, or 0 if the size cannot be granted.
template <int BITS, int MODE, bool BF16, int NT, int TPG, bool DEEP>
int occupancy() {
  static int occ[kMaxDevices] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) dev = 0;
  if (occ[dev]) return occ[dev];
  auto k = skinny_kernel<BITS, MODE, BF16, NT, TPG, DEEP>;
  constexpr size_t smem = smem_bytes<BITS, MODE, NT, TPG, DEEP>();
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess) {
    cudaGetLastError();   // do not leave the failure behind as a sticky error
    return 0;
  }
  int o = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, k, kThreads, smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  occ[dev] = o;
  return o;
}

template <int BITS, int MODE, bool BF16, int NT, int TPG, bool DEEP>
cudaError_t launch(const SkinnyArgs& args, int slabs, cudaStream_t stream) {
  auto k = skinny_kernel<BITS, MODE, BF16, NT, TPG, DEEP>;
  if (occupancy<BITS, MODE, BF16, NT, TPG, DEEP>() < 1) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(args.ctas, slabs, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes<BITS, MODE, NT, TPG, DEEP>();
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, args);
  if (e != cudaSuccess) cudaGetLastError();   // report it once, here
  return e;
}
// Calls f.template operator()<BITS, MODE, BF16, NT, TPG, DEEP>() for the
// runtime values (the deep ring only for the plain SYM / ASYM / LUT formats).
template <int B, int MO, bool BF, int T, int TP, class F>
auto dispatch_deep(bool deep, F&& f) {
  if constexpr (!zero_opts(MO) && T <= 2) {
    if (deep) return f.template operator()<B, MO, BF, T, TP, true>();
  }
  return f.template operator()<B, MO, BF, T, TP, false>();
}

template <int B, int MO, bool BF, int T, class F>
auto dispatch_tpg(int tpg, bool deep, F&& f) {
  switch (tpg) {
    case 1: return dispatch_deep<B, MO, BF, T, 1>(deep, f);
    case 2: return dispatch_deep<B, MO, BF, T, 2>(deep, f);
    case 4: return dispatch_deep<B, MO, BF, T, 4>(deep, f);
    default: return dispatch_deep<B, MO, BF, T, 8>(deep, f);
  }
}

template <class F>
auto dispatch(int bits, int mode, bool bf16, int nt, int tpg, bool deep, F&& f) {
#define QMM_CASE(B, MO, BF, T) \
  if (bits == B && mode == MO && bf16 == BF && nt == T) return dispatch_tpg<B, MO, BF, T>(tpg, deep, f);
  QMM_CASE(4, kSYM, false, 1) QMM_CASE(4, kSYM, false, 2) QMM_CASE(4, kSYM, true, 1)
  QMM_CASE(4, kSYM, true, 2) QMM_CASE(4, kASYM, false, 1) QMM_CASE(4, kASYM, false, 2)
  QMM_CASE(4, kASYM, true, 1) QMM_CASE(4, kASYM, true, 2) QMM_CASE(4, kLUT, false, 1)
  QMM_CASE(4, kLUT, false, 2) QMM_CASE(4, kLUT, true, 1) QMM_CASE(4, kLUT, true, 2)
  QMM_CASE(2, kLUT, false, 1) QMM_CASE(2, kLUT, false, 2) QMM_CASE(2, kLUT, true, 1)
  QMM_CASE(2, kLUT, true, 2) QMM_CASE(3, kLUT, false, 1) QMM_CASE(3, kLUT, false, 2)
  QMM_CASE(3, kLUT, true, 1) QMM_CASE(3, kLUT, true, 2)
  QMM_CASE(4, kSYM, false, 4) QMM_CASE(4, kSYM, true, 4) QMM_CASE(4, kASYM, false, 4)
  QMM_CASE(4, kASYM, true, 4) QMM_CASE(4, kLUT, false, 4) QMM_CASE(4, kLUT, true, 4)
  QMM_CASE(2, kLUT, false, 4) QMM_CASE(2, kLUT, true, 4) QMM_CASE(3, kLUT, false, 4)
  QMM_CASE(3, kLUT, true, 4)
  QMM_CASE(4, kASYMX, false, 1) QMM_CASE(4, kASYMX, false, 2) QMM_CASE(4, kASYMX, true, 1)
  QMM_CASE(4, kASYMX, true, 2) QMM_CASE(4, kASYMQ, false, 1) QMM_CASE(4, kASYMQ, false, 2)
  QMM_CASE(4, kASYMQ, true, 1) QMM_CASE(4, kASYMQ, true, 2) QMM_CASE(4, kASYMQ1, false, 1)
  QMM_CASE(4, kASYMQ1, false, 2) QMM_CASE(4, kASYMQ1, true, 1) QMM_CASE(4, kASYMQ1, true, 2)
#undef QMM_CASE
  return dispatch_tpg<4, kSYM, false, 1>(tpg, deep, f);
}

// Tiles (of 16 columns) per group inside a 128-column stage: 8 for groups of
// 128 columns or more (and for one group per row), else group / 16.
int tiles_per_group(int group) { return (group == -1 || group >= kSC) ? 8 : group / 16; }

}  // namespace

SkinnyPlan plan_skinny(int M, int N, int K, int bits, int group, int mode, bool bf16, int sms,
                       bool force_streamk) {
  SkinnyPlan p{};
  // token tiles of 8: 1 up to 8 tokens, 2 up to 16, 4 up to 32 (the plain
  // formats; zero-point options stay at 16 tokens per slab)
  p.nt = M <= 8 ? 1 : (M <= 16 || zero_opts(mode) ? 2 : 4);
  const int R = p.nt == 1 ? rb_per_tile<1>() : rb_per_tile<2>();
  p.rows = 16 * R;
  const int nrb = N / 16;
  p.tiles_n = (nrb + R - 1) / R;
  p.slabs = std::max(1, (M + 8 * p.nt - 1) / (8 * p.nt));
  const int nsc = (K + kSC - 1) / kSC;
  const long long units = (long long)p.tiles_n * nsc;
  const int tpg = tiles_per_group(group);
  p.smem = dispatch(bits, mode, bf16, p.nt, tpg, false,
                    [&]<int B, int MO, bool BF, int T, int TP, bool D>() { return smem_bytes<B, MO, T, TP, D>(); });
  const int occ = dispatch(bits, mode, bf16, p.nt, tpg, false,
                           [&]<int B, int MO, bool BF, int T, int TP, bool D>() { return occupancy<B, MO, BF, T, TP, D>(); });
  // one resident wave of CTAs; every warp is a stream-K worker with >= 1 unit
  long long warps = (long long)sms * (occ > 0 ? occ : 1) * kWarps;
  const long long cap = std::max<long long>(1, units * 8 / nsc);
  if (!force_streamk && warps >= (long long)p.tiles_n * kWarps) {
    // few row tiles: one CTA per tile, its warps split K, sums added in
    // shared memory (no split-K workspace)
    p.cta_tiles = 1;
    p.splits = p.tiles_n;
    p.warps = p.tiles_n * kWarps;
    p.ws_bytes = 0;
    // at most one tile per SM: each CTA has an SM to itself, so it takes the
    // deep ring (its warps' stages all requested up front on small matrices)
    if (p.tiles_n <= sms && !zero_opts(mode) && p.nt <= 2) {
      p.deep = 1;
      p.smem = dispatch(bits, mode, bf16, p.nt, tpg, true,
                        [&]<int B, int MO, bool BF, int T, int TP, bool D>() { return smem_bytes<B, MO, T, TP, D>(); });
    }
    return p;
  }
  if (warps > cap) warps = cap;
  if (warps > units) warps = units;
  const long long ctas = (warps + kWarps - 1) / kWarps;
  p.splits = (int)ctas;
  p.warps = (int)warps;
  const bool split = !(units % warps == 0 && (units / warps) % nsc == 0);
  if (split) {
    const size_t counters = ((size_t)p.slabs * p.tiles_n * sizeof(unsigned) + 255) / 256 * 256;
    const size_t slots = (size_t)p.slabs * 2 * warps * p.rows * 8 * p.nt * sizeof(float);
    p.ws_bytes = counters + slots;
  } else {
    p.ws_bytes = 0;
  }
  return p;
}

cudaError_t launch_skinny(const Problem& pr, const SkinnyPlan& plan, void* workspace,
                          cudaStream_t stream) {
  SkinnyArgs a{};
  a.x = reinterpret_cast<const uint16_t*>(pr.x);
  a.qw = reinterpret_cast<const uint8_t*>(pr.qweight);
  a.scales = pr.scales;
  a.zl = pr.zl;
  a.y = reinterpret_cast<uint16_t*>(pr.y);
  a.M = pr.M;
  a.N = pr.N;
  a.K = pr.K;
  a.gated = pr.gated ? 1 : 0;
  a.cta_tiles = plan.cta_tiles;
  const int L = pr.group == -1 ? pr.K : pr.group;
  a.G = pr.K / L;
  a.lg = pr.group == -1 ? -1 : __builtin_ctz((unsigned)pr.group);
  {
    const int LZ = pr.zgroup == 0 ? L : (pr.zgroup == -1 ? pr.K : pr.zgroup);
    a.GZ = pr.K / LZ;
    // zero groups of 128 columns or more: one per stage (lgz only decides the
    // group's index, K >> lgz; a row-long group gets a shift past every k)
    a.lgz = pr.zgroup == -1 || (pr.zgroup == 0 && pr.group == -1) ? 30 : __builtin_ctz((unsigned)LZ);
  }
  a.nchunks = pr.K / chunk_cols(pr.bits);
  a.nsc = (pr.K + kSC - 1) / kSC;
  a.nrb = pr.N / 16;
  a.tiles = plan.tiles_n;
  a.units = (long long)plan.tiles_n * a.nsc;
  a.ctas = plan.splits;
  a.warps = plan.warps;
  a.inv_units = 1.0 / (double)a.units;
  a.inv_warps = 1.0 / (double)a.warps;
  if (plan.ws_bytes) {
    const size_t counters = ((size_t)plan.slabs * plan.tiles_n * sizeof(unsigned) + 255) / 256 * 256;
    a.counters = reinterpret_cast<unsigned*>(workspace);
    a.slots = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + counters);
  }
  return dispatch(pr.bits, pr.mode, pr.bf16, plan.nt, tiles_per_group(pr.group), plan.deep != 0,
                  [&]<int B, int MO, bool BF, int T, int TP, bool D>() {
                    a.stage_bytes = Stage<B, MO, T, TP>::BYTES;
                    return launch<B, MO, BF, T, TP, D>(a, plan.slabs, stream);
                  });
}

}  // namespace qk

// ---------------------------------------------------------------------------
// Decode path with a library-owned scratch buffer, for callers that cannot
// allocate device memory (see qmm_noalloc in qmm.h).
namespace qk {
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;   // 8 MiB per device
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device.  The symbol's
// name is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
cudaError_t static_scratch(void** out) {
  // atomics: host threads making their first call on a device at the same
  // time may both look the address up; they store the same value
  static std::atomic<void*> addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = addr[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return e;
    }
    addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

size_t static_scratch_bytes() { return kStaticScratchBytes; }

cudaError_t launch_skinny_static(const Problem& pr, int sms, cudaStream_t stream, bool* too_large) {
  *too_large = false;
  SkinnyPlan plan = plan_skinny(pr.M, pr.N, pr.K, pr.bits, pr.group, pr.mode, pr.bf16, sms);
  const size_t counters = ((size_t)plan.slabs * plan.tiles_n * sizeof(unsigned) + 255) / 256 * 256;
  const size_t slot2 = (size_t)plan.slabs * 2 * plan.rows * 8 * plan.nt * sizeof(float);  // per worker
  if (plan.ws_bytes > kStaticScratchBytes) {
    // fewer stream-K workers so that their partial-sum slots fit
    if (counters + slot2 > kStaticScratchBytes) {
      *too_large = true;
      return cudaSuccess;
    }
    const long long w = (long long)((kStaticScratchBytes - counters) / slot2);
    plan.warps = (int)std::min<long long>(plan.warps, w);
    plan.splits = (plan.warps + kWarps - 1) / kWarps;
    plan.ws_bytes = counters + slot2 * plan.warps;
  }
  void* ws = nullptr;
  if (plan.ws_bytes) {
    cudaError_t e = static_scratch(&ws);
    if (e != cudaSuccess) return e;
    // the arrival counters must start at zero; every call shares the buffer
    e = cudaMemsetAsync(ws, 0, counters, stream);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return e;
    }
  }
  return launch_skinny(pr, plan, ws, stream);
}

}  // namespace qk

namespace qk {
unsigned skinny_read_and_clear_error() {
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_skinny_error, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
  if (v) cudaMemcpyToSymbol(g_skinny_error, &zero, sizeof(zero));
  return v;
}
}  // namespace qk
