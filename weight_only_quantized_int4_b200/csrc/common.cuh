// Shared device helpers for the qmm kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "qmm.h"

namespace qk {

constexpr int kSYM = QMM_SYM, kASYM = QMM_ASYM, kLUT = QMM_LUT;
// Internal modes: ASYM with zero-point options (a zero group inside the scale
// group, or 4-bit integer zero-points); packed codes as for ASYM.  kASYMX has
// fp16 zero-points, kASYMQ 4-bit ones, kASYMQ1 4-bit ones in groups of 128
// columns or more (one zero record per 128-column stage of the decode path).
constexpr int kASYMX = 3, kASYMQ = 4, kASYMQ1 = 5;
__host__ __device__ constexpr bool zero_opts(int mode) {
  return mode == kASYMX || mode == kASYMQ || mode == kASYMQ1;
}

// Chunk of K covered by one block of codes (16 rows x KC columns): 512 bytes
// for 4- and 2-bit codes, 768 bytes for 3-bit codes.
__host__ __device__ constexpr int chunk_cols(int bits) { return bits == 4 ? 64 : 128; }
__host__ __device__ constexpr int chunk_bytes(int bits) { return bits == 3 ? 768 : 512; }

// Position of row r (0..15) of a row block inside its 16 scales.
__host__ __device__ constexpr int scale_slot(int r) { return 2 * (r & 7) + (r >> 3); }

// ------------------------------------------------------------------ PTX wrappers

// 128-bit load that caches in L2 only: codes are streamed once per call.
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_cg_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ld_u2(const void* p) {
  uint2 v;
  asm volatile("ld.global.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// Programmatic dependent launch: wait for the previous grid in the stream /
// allow the next grid to start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// D = A(16x16, row) . B(16x8, col) + C, fp32 accumulate.
template <bool BF16>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  if constexpr (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
  uint32_t r;
  // (a & mask) | orv  -> LUT = (0xF0 & 0xCC) | 0xAA = 0xEA
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(orv));
  return r;
}

__device__ __forceinline__ uint32_t hsub2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
__device__ __forceinline__ uint32_t bsub2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bfma2_u(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}


// --------------------------------------------------------- mbarrier / TMA helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of `bar`: false once `limit` clock cycles
// pass without the phase completing (the caller then abandons its work).
__device__ __forceinline__ bool mbar_wait_cycles(uint64_t* bar, uint32_t parity, long long limit) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try(bar, parity))
    if (clock64() - t0 > limit) return false;
  return true;
}

// 2D tensor-map load into shared memory, completing on `bar` (no multicast).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Orders this thread's generic-proxy global accesses with async-proxy (bulk
// copy) accesses of global memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// 2D tensor-map store from shared memory (bulk async group; out-of-range
// parts of the box are not written).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
// Contiguous shared -> global copy (bulk async group), same rules as bulk_load.
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The shared memory of every committed bulk store has been read.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Every committed bulk store has been performed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Contiguous global -> shared copy of `bytes` (a multiple of 16, both
// addresses 16-byte aligned), completing on `bar` (no multicast).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// SiLU (x times the logistic sigmoid of x) of the fused FFN gate.
__device__ __forceinline__ float silu(float v) { return v / (1.0f + __expf(-v)); }

// ------------------------------------------------------------- code decoding
//
// One 32-bit word of a 4-bit SYM/ASYM chunk holds a lane's 8 codes of one
// 16-column tile: pair p (the four MMA A-fragment registers a0..a3) at nibbles
// p (low member) and p + 4 (high member).  A nibble OR-ed under the exponent
// of 1024.0 (fp16 0x6400) or 128.0 (bf16 0x4300) reads as 1024 + q (128 + q);
// a nibble sitting 4 bits higher reads as 1024 + 16 q and is brought back with
// one fma by 1/16.  Subtracting the bias leaves the exact small integer q - z.

template <bool BF16>
struct Magic;
template <>
struct Magic<false> {
  static constexpr uint32_t kOr = 0x64006400u;   // 1024.0 in both halves
  static constexpr float kBase = 1024.0f;
};
template <>
struct Magic<true> {
  static constexpr uint32_t kOr = 0x43004300u;   // 128.0 in both halves
  static constexpr float kBase = 128.0f;
};

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

// Decode one word of a 4-bit SYM/ASYM chunk into the four A-fragment
// registers, as the exact integers q - ZI (ZI = 8 for SYM; 0 for ASYM, whose
// zero-point is taken off afterwards by sub_zero).
//   pair 0 (row g)     nibbles 0, 4      pair 1 (row g + 8) nibbles 1, 5
//   pair 2 (row g)     nibbles 2, 6      pair 3 (row g + 8) nibbles 3, 7
// fp16: the odd pairs are masked in place (value 1024 + 16 q) and brought back
// by one fma: (1024 + 16 q) / 16 - (64 + ZI).  bf16 has only 7 fraction bits,
// so there the odd pairs are shifted down first.
template <bool BF16, int ZI>
__device__ __forceinline__ void decode_int4(uint32_t w, uint32_t (&a)[4]) {
  constexpr uint32_t kOr = Magic<BF16>::kOr;
  const uint32_t w8 = w >> 8;
  if constexpr (BF16) {
    constexpr uint32_t kBias = 0x43004300u + (uint32_t)ZI * 0x00010001u;   // 128 + ZI
    a[0] = bsub2_u(lop3_and_or(w, 0x000F000Fu, kOr), kBias);
    a[1] = bsub2_u(lop3_and_or(w >> 4, 0x000F000Fu, kOr), kBias);
    a[2] = bsub2_u(lop3_and_or(w8, 0x000F000Fu, kOr), kBias);
    a[3] = bsub2_u(lop3_and_or(w >> 12, 0x000F000Fu, kOr), kBias);
  } else {
    constexpr uint32_t kBias = 0x64006400u + (uint32_t)ZI * 0x00010001u;   // 1024 + ZI
    // -(64 + ZI): 64 is 0x5400 with a step of 1/16, so ZI adds ZI*16 steps
    constexpr uint32_t kNegBias16 = 0xD400D400u + (uint32_t)(ZI * 16) * 0x00010001u;
    constexpr uint32_t kSixteenth = 0x2C002C00u;
    a[0] = hsub2_u(lop3_and_or(w, 0x000F000Fu, kOr), kBias);
    a[1] = hfma2_u(lop3_and_or(w, 0x00F000F0u, kOr), kSixteenth, kNegBias16);
    a[2] = hsub2_u(lop3_and_or(w8, 0x000F000Fu, kOr), kBias);
    a[3] = hfma2_u(lop3_and_or(w8, 0x00F000F0u, kOr), kSixteenth, kNegBias16);
  }
}

// ASYM: a[i] -= z for the row of each register (one rounding; exact for
// integer zero-points).
template <bool BF16>
__device__ __forceinline__ void sub_zero(uint32_t z_g, uint32_t z_g8, uint32_t (&a)[4]) {
  if constexpr (BF16) {
    a[0] = bsub2_u(a[0], z_g); a[1] = bsub2_u(a[1], z_g8);
    a[2] = bsub2_u(a[2], z_g); a[3] = bsub2_u(a[3], z_g8);
  } else {
    a[0] = hsub2_u(a[0], z_g); a[1] = hsub2_u(a[1], z_g8);
    a[2] = hsub2_u(a[2], z_g); a[3] = hsub2_u(a[3], z_g8);
  }
}

}  // namespace qk
