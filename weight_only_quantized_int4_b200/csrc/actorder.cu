// Act-order support: the packed column order from per-column group indices,
// and the gather of activation columns into that order.
//
// The GPTQ-Triton project summary ("Limitations & Caveats") names GPTQ's
// act-order option.  Under act-order the quantizer forms its groups along a
// column order of its own, so column k of W belongs to group g_idx[k] and a
// group is any set of columns.  The packed layout keeps every group's columns
// together: packed column j holds original column perm[j], group i occupying
// packed columns [i L, (i + 1) L) in ascending original order.  A product then
// needs x with its columns in the same order, x'[m, j] = x[m, perm[j]], after
// which the kernels of the plain layout apply unchanged.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace qk {
namespace {

constexpr int kPermThreads = 256;

// One CTA per group gi: scan g_idx in column order, write the group's members
// to perm[gi L + rank] (rank = members seen before), count them.  A group that
// does not end with exactly L members adds 1 to *bad (its perm entries are
// then incomplete).  Values of g_idx outside [0, G) match no group.
__global__ void __launch_bounds__(kPermThreads) gidx_perm_kernel(const int* __restrict__ g_idx,
                                                                 int K, int L,
                                                                 int* __restrict__ perm,
                                                                 int* __restrict__ bad) {
  constexpr int kW = kPermThreads / 32;
  __shared__ int warp_counts[kW];
  const int gi = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int base = 0;   // members in the columns already scanned (same in every thread)
  for (int k0 = 0; k0 < K; k0 += kPermThreads) {
    const int k = k0 + threadIdx.x;
    const bool mine = k < K && g_idx[k] == gi;
    const unsigned b = __ballot_sync(0xffffffffu, mine);
    if (lane == 0) warp_counts[warp] = __popc(b);
    __syncthreads();
    int before = base, total = 0;
#pragma unroll
    for (int w = 0; w < kW; ++w) {
      before += w < warp ? warp_counts[w] : 0;
      total += warp_counts[w];
    }
    const int rank = before + __popc(b & ((1u << lane) - 1u));
    if (mine && rank < L) perm[(size_t)gi * L + rank] = k;
    base += total;
    __syncthreads();   // warp_counts is rewritten by the next round
  }
  if (threadIdx.x == 0 && base != L) atomicAdd(bad, 1);
}

// x'[m, j] = x[m, perm[j]]: one thread per 8 consecutive packed columns of one
// row (one 16-byte store).  perm entries outside [0, K) read column 0.
__global__ void __launch_bounds__(256) permute_x_kernel(const uint16_t* __restrict__ x,
                                                        const int* __restrict__ perm, int M, int K,
                                                        uint16_t* __restrict__ xp) {
  pdl_wait();                 // x (and perm) may come from the previous grid
  pdl_launch_dependents();    // the product may start getting resident
  const size_t pieces_per_row = (size_t)K / 8;
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)M * pieces_per_row) return;
  const size_t m = i / pieces_per_row;
  const int j0 = (int)(i - m * pieces_per_row) * 8;
  const int4 p0 = *reinterpret_cast<const int4*>(perm + j0);
  const int4 p1 = *reinterpret_cast<const int4*>(perm + j0 + 4);
  const int c[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
  const uint16_t* row = x + m * K;
  uint32_t v[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const unsigned lo = (unsigned)c[2 * q], hi = (unsigned)c[2 * q + 1];
    const uint32_t a = row[lo < (unsigned)K ? lo : 0u];
    const uint32_t b = row[hi < (unsigned)K ? hi : 0u];
    v[q] = a | (b << 16);
  }
  *reinterpret_cast<uint4*>(xp + m * K + j0) = make_uint4(v[0], v[1], v[2], v[3]);
}

}  // namespace

cudaError_t launch_gidx_perm(const int* g_idx, int K, int group, int* perm, int* bad,
                             cudaStream_t stream) {
  const int L = group == -1 ? K : group;
  cudaError_t e = cudaMemsetAsync(bad, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  gidx_perm_kernel<<<K / L, kPermThreads, 0, stream>>>(g_idx, K, L, perm, bad);
  return cudaGetLastError();
}

cudaError_t launch_permute_x(const void* x, const int* perm, int M, int K, void* xp,
                             cudaStream_t stream) {
  const size_t pieces = (size_t)M * (K / 8);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((pieces + 255) / 256), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e =
      cudaLaunchKernelEx(&cfg, permute_x_kernel, reinterpret_cast<const uint16_t*>(x), perm, M, K,
                         reinterpret_cast<uint16_t*>(xp));
  if (e != cudaSuccess) cudaGetLastError();
  return e;
}

}  // namespace qk
