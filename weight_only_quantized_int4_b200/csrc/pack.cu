// Quantize/pack and debug-decode kernels.
//
// Quantization follows efrantar's reply in "Does Marlin support zero-point
// quantization?" (IST-DASLab/marlin issue 5: symmetric int4 with the zero fixed
// at 8 and fp16 scales; fp16 zero-points for the asymmetric variant) and the
// FLUTE summary's "How It Works" (nearest table entry, times a scale).  The
// arithmetic is the one documented for qmm_pack in qmm.h: fp32 group
// reductions, IEEE fp32 division, fp16 scale rounded before use, rint half to
// even.  This file is compiled with --fmad=false so that no product and sum is
// ever fused.
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace qk {
namespace {

// rint() result -> code in [0, qmax]; anything not above 0 (incl. NaN) -> 0.
__device__ __forceinline__ int clamp_code(float v, int qmax) {
  if (!(v > 0.0f)) return 0;
  if (v > (float)qmax) return qmax;
  return (int)v;
}

__device__ __forceinline__ uint16_t scale_to_half(float s32) {
  __half h = __float2half_rn(s32);
  uint16_t b = __half_as_ushort(h);
  if ((b & 0x7fff) == 0x7c00) b = (b & 0x8000) | 0x7bff;   // saturate, never inf
  return b;
}

// Column k of a source row; with an act-order permutation, packed column k
// takes original column perm[k] (entries outside [0, K) read column 0).
__device__ __forceinline__ float wcol(const float* row, const int* perm, int k, int K) {
  if (!perm) return row[k];
  const unsigned c = (unsigned)perm[k];
  return row[c < (unsigned)K ? c : 0u];
}

// Source row of packed row n.  With a second matrix W2 (the gated layout),
// 16-row blocks alternate: packed block 2b is block b of W, block 2b + 1 is
// block b of W2.
__device__ __forceinline__ const float* src_row(const float* W, const float* W2, int n, int K) {
  if (!W2) return W + (size_t)n * K;
  const int b = n >> 4;
  return ((b & 1) ? W2 : W) + (size_t)((b >> 1) * 16 + (n & 15)) * K;
}

// One warp per (row n, group gi): reduce |w| or (min, max) over the group,
// write the fp16 scale (and, if `zeros` is given, the zero) at the packed
// position.
__global__ void __launch_bounds__(256) pack_scales_kernel(const float* __restrict__ W,
                                                          const float* __restrict__ W2,
                                                          const int* __restrict__ perm, int N,
                                                          int K, int mode, int L, int G,
                                                          uint16_t* __restrict__ scales,
                                                          uint16_t* __restrict__ zeros) {
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (long long)N * G) return;
  const int n = (int)(warp / G), gi = (int)(warp % G);
  const float* row = src_row(W, W2, n, K);
  float amax = 0.0f, mn = INFINITY, mx = -INFINITY;
  for (int i = lane; i < L; i += 32) {
    float v = wcol(row, perm, gi * L + i, K);
    amax = fmaxf(amax, fabsf(v));
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  for (int o = 16; o; o >>= 1) {
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane) return;
  float s32;
  if (mode == kSYM) s32 = __fdiv_rn(amax, 7.0f);
  else if (mode == kASYM) s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
  else s32 = amax;
  const uint16_t s16 = scale_to_half(s32);
  const size_t idx = ((size_t)(n >> 4) * G + gi) * 16 + scale_slot(n & 15);
  scales[idx] = s16;
  if (mode == kASYM && zeros) {
    const float s = __half2float(__ushort_as_half(s16));
    const int z = (s == 0.0f) ? 0 : clamp_code(rintf(__fdiv_rn(-mn, s)), 15);
    zeros[idx] = __half_as_ushort(__int2half_rn(z));
  }
}

// Zero-point storage: fp16 values [N/16][GZ][16] (zbits 16), or the same
// integers in 4 bits, [N/16][GZ][8 bytes] with slot i at byte i / 2, the low
// nibble for even i (zbits 4).  Groups of LZ columns.
struct ZeroFmt {
  const void* z;
  int LZ, GZ, zbits;
};

__device__ __forceinline__ float zero_value(const ZeroFmt& f, int rb, int zi, int slot) {
  const size_t idx = ((size_t)rb * f.GZ + zi) * 16 + slot;
  if (f.zbits == 16) return __half2float(__ushort_as_half(static_cast<const uint16_t*>(f.z)[idx]));
  return (float)((static_cast<const uint8_t*>(f.z)[idx >> 1] >> (4 * (idx & 1))) & 15u);
}

// Zero-points of zero groups nested in the scale groups (efrantar's and
// mobicham's replies in the Marlin zero-point issue: integer zero-points,
// zero group smaller than the scale group): one thread per (row block, zero
// group, g) takes rows g and g + 8 (adjacent slots, one byte in 4-bit form):
// z = clamp(rint(-min / s), 0, 15) from the zero group's minimum and the fp16
// scale of the scale group around it.
__global__ void __launch_bounds__(256) pack_zeros_kernel(const float* __restrict__ W, int N, int K,
                                                         int L, int G, int LZ, int GZ, int zbits,
                                                         const uint16_t* __restrict__ scales,
                                                         void* __restrict__ zeros) {
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= (size_t)(N / 16) * GZ * 8) return;
  const int g = (int)(tid & 7);
  const size_t rz = tid >> 3;
  const int zi = (int)(rz % GZ), rb = (int)(rz / GZ);
  const int gi = (int)(((long long)zi * LZ) / L);
  int zv[2];
  for (int h = 0; h < 2; ++h) {
    const int n = rb * 16 + g + 8 * h;
    const float* w = W + (size_t)n * K + (size_t)zi * LZ;
    float mn = w[0];
    for (int i = 1; i < LZ; ++i) mn = fminf(mn, w[i]);
    const float s = __half2float(
        __ushort_as_half(scales[((size_t)rb * G + gi) * 16 + scale_slot(g + 8 * h)]));
    zv[h] = (s == 0.0f) ? 0 : clamp_code(rintf(__fdiv_rn(-mn, s)), 15);
  }
  const size_t idx = ((size_t)rb * GZ + zi) * 16 + 2 * g;   // slots 2g (row g), 2g + 1 (row g + 8)
  if (zbits == 16) {
    uint16_t* z = static_cast<uint16_t*>(zeros);
    z[idx] = __half_as_ushort(__int2half_rn(zv[0]));
    z[idx + 1] = __half_as_ushort(__int2half_rn(zv[1]));
  } else {
    static_cast<uint8_t*>(zeros)[idx >> 1] = (uint8_t)(zv[0] | (zv[1] << 4));
  }
}

struct CodeCtx {
  const float* W;
  const float* W2;   // gated layout: the second matrix (else null)
  const int* perm;   // act-order: packed column k takes original column perm[k] (else null)
  int K, mode, bits, L, G, nchunks;
  const uint16_t* scales;
  ZeroFmt zf;        // ASYM zero-points
  const uint16_t* lut;   // 2^bits fp16 entries (LUT mode)
  int nlut;
};

__device__ __forceinline__ int encode(float w, float s, float z, const CodeCtx& c,
                                     const float (&lut)[16]) {
  if (c.mode == kSYM) return s == 0.0f ? 8 : clamp_code(__fadd_rn(rintf(__fdiv_rn(w, s)), 8.0f), 15);
  if (c.mode == kASYM) return s == 0.0f ? 0 : clamp_code(__fadd_rn(rintf(__fdiv_rn(w, s)), z), 15);
  const float u = (s == 0.0f) ? 0.0f : __fdiv_rn(w, s);
  int best = 0;
  float bd = fabsf(__fsub_rn(u, lut[0]));
  for (int e = 1; e < c.nlut; ++e) {
    const float d = fabsf(__fsub_rn(u, lut[e]));
    if (d < bd) { bd = d; best = e; }
  }
  return best;
}

// One thread per 32-bit word of the packed codes.  Word id -> (row block,
// chunk, lane, word); the word's codes are gathered from W and placed at the
// nibble / 2-bit field the layout assigns them.
__global__ void __launch_bounds__(256) pack_codes_kernel(CodeCtx c, uint32_t* __restrict__ out,
                                                         size_t nwords) {
  const size_t wid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (wid >= nwords) return;
  const int word = wid & 3;
  const int lane = (wid >> 2) & 31;
  const size_t blk = wid >> 7;                       // 128 words per 512-byte chunk
  const int chunk = (int)(blk % c.nchunks);
  const int rb = (int)(blk / c.nchunks);
  const int g = lane >> 2, t = lane & 3;
  const int KC = chunk_cols(c.bits);
  float lut[16];
  for (int e = 0; e < 16; ++e)
    lut[e] = (c.mode == kLUT && e < c.nlut) ? __half2float(__ushort_as_half(c.lut[e])) : 0.0f;
  uint32_t v = 0;
  const int tiles_per_word = c.bits == 4 ? 1 : 2;
  for (int sub = 0; sub < tiles_per_word; ++sub) {
    const int j = word * tiles_per_word + sub;                   // 16-column tile
    const int k0 = chunk * KC + 16 * j + 4 * t;
    const int gi = k0 / c.L;
    for (int h = 0; h < 2; ++h) {
      const int n = rb * 16 + g + 8 * h;
      const size_t sidx = ((size_t)rb * c.G + gi) * 16 + scale_slot(g + 8 * h);
      const float s = __half2float(__ushort_as_half(c.scales[sidx]));
      const float z = c.mode == kASYM ? zero_value(c.zf, rb, k0 / c.zf.LZ, scale_slot(g + 8 * h))
                                      : 0.0f;
      float wc[4];
      const float* row = src_row(c.W, c.W2, n, c.K);
      if (c.perm) {
        for (int cc = 0; cc < 4; ++cc) wc[cc] = wcol(row, c.perm, k0 + cc, c.K);
      } else {
        const float4 wv = *reinterpret_cast<const float4*>(row + k0);
        wc[0] = wv.x; wc[1] = wv.y; wc[2] = wv.z; wc[3] = wv.w;
      }
      for (int cc = 0; cc < 4; ++cc) {
        const uint32_t q = (uint32_t)encode(wc[cc], s, z, c, lut);
        const int p = h + 2 * (cc >> 1), hi = cc & 1;
        int shift;
        if (c.bits == 4) {
          const int nib = (c.mode == kLUT) ? (2 * p + hi) : (p + 4 * hi);
          shift = 4 * nib;
        } else {
          shift = 8 * (2 * sub + (p >> 1)) + 2 * (2 * (p & 1) + hi);
        }
        v |= q << shift;
      }
    }
  }
  out[wid] = v;
  __threadfence();   // codes visible before this block retires (see qmm_pack)
}

// ---------------------------------------------------------------- dequant

// One thread per packed word: decode its codes to (q - z) * s (or T[q] * s),
// exact in fp32 for integer zero-points, then round once to fp16 / bf16.
// 3-bit codes: one thread per 32-bit word, six words per lane of a 768-byte
// chunk (128 columns).  The lane's six words are one 192-bit little-endian
// string: tile j at bits [24 j, 24 j + 24), pair p at [24 j + 6 p, + 6), member
// c % 2 at + 3 (c % 2).  Word w takes the bits [32 w, 32 w + 32) of it, i.e.
// parts of tiles 4w/3 .. (32w + 31)/24.
__global__ void __launch_bounds__(256) pack_codes3_kernel(CodeCtx c, uint32_t* __restrict__ out,
                                                          size_t nwords) {
  const size_t wid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (wid >= nwords) return;
  const int w6 = (int)(wid % 6);
  const int lane = (int)((wid / 6) % 32);
  const size_t blk = wid / 192;                      // 192 words per 768-byte chunk
  const int chunk = (int)(blk % c.nchunks);
  const int rb = (int)(blk / c.nchunks);
  const int g = lane >> 2, t = lane & 3;
  float lut[16];
  for (int e = 0; e < 16; ++e)
    lut[e] = e < c.nlut ? __half2float(__ushort_as_half(c.lut[e])) : 0.0f;
  const int lo_bit = 32 * w6;
  uint32_t v = 0;
  for (int j = (32 * w6) / 24; j <= (32 * w6 + 31) / 24 && j < 8; ++j) {   // 16-column tile
    const int k0 = chunk * 128 + 16 * j + 4 * t;
    const int gi = k0 / c.L;
    for (int h = 0; h < 2; ++h) {
      const int n = rb * 16 + g + 8 * h;
      const size_t sidx = ((size_t)rb * c.G + gi) * 16 + scale_slot(g + 8 * h);
      const float s = __half2float(__ushort_as_half(c.scales[sidx]));
      const float* row = src_row(c.W, c.W2, n, c.K);
      float wc[4];
      for (int cc = 0; cc < 4; ++cc) wc[cc] = wcol(row, c.perm, k0 + cc, c.K);
      for (int cc = 0; cc < 4; ++cc) {
        const uint32_t q = (uint32_t)encode(wc[cc], s, 0.0f, c, lut);
        const int p = h + 2 * (cc >> 1), hi = cc & 1;
        const int b = 24 * j + 6 * p + 3 * hi;            // the code's lowest bit
        for (int i = 0; i < 3; ++i) {
          const int pos = b + i - lo_bit;
          if (pos >= 0 && pos < 32) v |= ((q >> i) & 1u) << pos;
        }
      }
    }
  }
  out[wid] = v;
  __threadfence();   // visible to any kernel that starts after this grid
}

// 3-bit codes: one thread per (row block, chunk, lane) decodes its 64 codes.
__global__ void __launch_bounds__(256) dequant3_kernel(const uint32_t* __restrict__ qw,
                                                       const uint16_t* __restrict__ scales,
                                                       const uint16_t* __restrict__ lut, int K,
                                                       int L, int G, int nchunks, bool bf16,
                                                       void* out, size_t nthreads) {
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid >= nthreads) return;
  const int lane = (int)(tid % 32);
  const size_t blk = tid / 32;
  const int chunk = (int)(blk % nchunks);
  const int rb = (int)(blk / nchunks);
  const int g = lane >> 2, t = lane & 3;
  const uint32_t* w = qw + blk * 192 + (size_t)lane * 6;
  uint32_t lw[7];   // the lane's 192-bit string, one word of zero padding
  for (int i = 0; i < 6; ++i) lw[i] = w[i];
  lw[6] = 0;
  for (int j = 0; j < 8; ++j) {
    const int k0 = chunk * 128 + 16 * j + 4 * t;
    const int gi = k0 / L;
    for (int h = 0; h < 2; ++h) {
      const int n = rb * 16 + g + 8 * h;
      const size_t sidx = ((size_t)rb * G + gi) * 16 + scale_slot(g + 8 * h);
      const float s = __half2float(__ushort_as_half(scales[sidx]));
      float r[4];
      for (int cc = 0; cc < 4; ++cc) {
        const int p = h + 2 * (cc >> 1), hi = cc & 1;
        const int b = 24 * j + 6 * p + 3 * hi;             // the code's lowest bit
        const uint64_t win = (uint64_t)lw[b >> 5] | ((uint64_t)lw[(b >> 5) + 1] << 32);
        const uint32_t q = (uint32_t)(win >> (b & 31)) & 7u;
        r[cc] = __fmul_rn(__half2float(__ushort_as_half(lut[q])), s);
      }
      const size_t o = (size_t)n * K + k0;
      if (bf16) {
        __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(out) + o;
        for (int cc = 0; cc < 4; ++cc) p[cc] = __float2bfloat16_rn(r[cc]);
      } else {
        __half* p = reinterpret_cast<__half*>(out) + o;
        for (int cc = 0; cc < 4; ++cc) p[cc] = __float2half_rn(r[cc]);
      }
    }
  }
}

__global__ void __launch_bounds__(256) dequant_kernel(const uint32_t* __restrict__ qw,
                                                      const uint16_t* __restrict__ scales,
                                                      const uint16_t* __restrict__ zl, ZeroFmt zf,
                                                      int K, int bits, int mode, int L, int G,
                                                      int nchunks, bool bf16, void* out,
                                                      size_t nwords) {
  const size_t wid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (wid >= nwords) return;
  const int word = wid & 3;
  const int lane = (wid >> 2) & 31;
  const size_t blk = wid >> 7;
  const int chunk = (int)(blk % nchunks);
  const int rb = (int)(blk / nchunks);
  const int g = lane >> 2, t = lane & 3;
  const int KC = chunk_cols(bits);
  const uint32_t v = qw[wid];
  const int tiles_per_word = bits == 4 ? 1 : 2;
  for (int sub = 0; sub < tiles_per_word; ++sub) {
    const int j = word * tiles_per_word + sub;
    const int k0 = chunk * KC + 16 * j + 4 * t;
    const int gi = k0 / L;
    for (int h = 0; h < 2; ++h) {
      const int n = rb * 16 + g + 8 * h;
      const size_t sidx = ((size_t)rb * G + gi) * 16 + scale_slot(g + 8 * h);
      const float s = __half2float(__ushort_as_half(scales[sidx]));
      const float z = mode == kSYM    ? 8.0f
                      : mode == kASYM ? zero_value(zf, rb, k0 / zf.LZ, scale_slot(g + 8 * h))
                                      : 0.0f;
      float r[4];
      for (int cc = 0; cc < 4; ++cc) {
        const int p = h + 2 * (cc >> 1), hi = cc & 1;
        uint32_t q;
        if (bits == 4) {
          const int nib = (mode == kLUT) ? (2 * p + hi) : (p + 4 * hi);
          q = (v >> (4 * nib)) & 15u;
        } else {
          q = (v >> (8 * (2 * sub + (p >> 1)) + 2 * (2 * (p & 1) + hi))) & 3u;
        }
        if (mode == kLUT) r[cc] = __fmul_rn(__half2float(__ushort_as_half(zl[q])), s);
        else r[cc] = __fmul_rn(__fsub_rn((float)q, z), s);
      }
      const size_t o = (size_t)n * K + k0;
      if (bf16) {
        __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(out) + o;
        for (int cc = 0; cc < 4; ++cc) p[cc] = __float2bfloat16_rn(r[cc]);
      } else {
        __half* p = reinterpret_cast<__half*>(out) + o;
        for (int cc = 0; cc < 4; ++cc) p[cc] = __float2half_rn(r[cc]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_pack(const float* W, const float* W2, const int* perm, int N, int K, int mode,
                        int bits, int group, int zgroup, int zbits, const uint16_t* lut,
                        void* qweight, uint16_t* scales, void* zeros, cudaStream_t stream) {
  const int L = group == -1 ? K : group;
  const int G = K / L;
  const int LZ = zgroup == 0 ? L : (zgroup == -1 ? K : zgroup);
  const bool own_zeros = mode == kASYM && (LZ != L || zbits != 16);   // zero-point options
  const long long warps = (long long)N * G;
  pack_scales_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, stream>>>(
      W, W2, perm, N, K, mode, L, G, scales, own_zeros ? nullptr : static_cast<uint16_t*>(zeros));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (own_zeros) {
    const size_t threads = (size_t)(N / 16) * (K / LZ) * 8;
    pack_zeros_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(
        W, N, K, L, G, LZ, K / LZ, zbits, scales, zeros);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  CodeCtx c;
  c.W = W;
  c.W2 = W2;
  c.perm = perm;
  c.K = K;
  c.mode = mode;
  c.bits = bits;
  c.L = L;
  c.G = G;
  c.nchunks = K / chunk_cols(bits);
  c.scales = scales;
  c.zf = ZeroFmt{zeros, LZ, K / LZ, mode == kASYM ? zbits : 16};
  c.lut = lut;
  c.nlut = 1 << bits;
  const size_t nwords = (size_t)N * K * bits / 32;
  const unsigned blocks = (unsigned)((nwords + 255) / 256);
  if (bits == 3)
    pack_codes3_kernel<<<blocks, 256, 0, stream>>>(c, reinterpret_cast<uint32_t*>(qweight), nwords);
  else
    pack_codes_kernel<<<blocks, 256, 0, stream>>>(c, reinterpret_cast<uint32_t*>(qweight), nwords);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const void* qweight, const uint16_t* scales,
                           const void* zeros_or_lut, int N, int K, int bits, int group,
                           int zgroup, int zbits, int mode, int out_dtype, void* W_out,
                           cudaStream_t stream) {
  const int L = group == -1 ? K : group;
  const int G = K / L;
  const int LZ = zgroup == 0 ? L : (zgroup == -1 ? K : zgroup);
  const ZeroFmt zf{zeros_or_lut, LZ, K / LZ, zbits};
  const uint16_t* zl = static_cast<const uint16_t*>(zeros_or_lut);
  if (bits == 3) {
    const size_t nthreads = (size_t)(N / 16) * (K / 128) * 32;
    dequant3_kernel<<<(unsigned)((nthreads + 255) / 256), 256, 0, stream>>>(
        reinterpret_cast<const uint32_t*>(qweight), scales, zl, K, L, G, K / 128,
        out_dtype == QMM_BF16, W_out, nthreads);
    return cudaGetLastError();
  }
  const size_t nwords = (size_t)N * K * bits / 32;
  const unsigned blocks = (unsigned)((nwords + 255) / 256);
  dequant_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const uint32_t*>(qweight), scales,
                                             zl, zf, K, bits, mode, L, G,
                                             K / chunk_cols(bits), out_dtype == QMM_BF16, W_out,
                                             nwords);
  return cudaGetLastError();
}

}  // namespace qk
