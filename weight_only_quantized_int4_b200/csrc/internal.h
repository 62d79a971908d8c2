// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace qk {

struct Problem {
  const void* x;
  bool bf16;
  const void* qweight;
  const uint16_t* scales;
  const uint16_t* zl;     // zeros (ASYM) or table (LUT)
  int M, N, K, bits, group, mode;
  void* y;
  bool gated = false;     // fused gate/up rows: y[M, N/2] = silu(gate) * up
  // ASYM zero-point options (modes kASYMX / kASYMQ): zero group (columns; 0 =
  // the scale group, -1 = the row) and storage (16 = fp16, 4 = 4-bit integers)
  int zgroup = 0, zbits = 16;
};

// Split-K plan of the skinny (M <= 16 per slab) decode path.
struct SkinnyPlan {
  int nt;          // token tiles of 8 per slab (1 or 2)
  int cta_tiles;   // 1: one CTA per row tile, warps split K, no workspace
  int deep;        // 1: one CTA per SM with a deep ring (cta_tiles and tiles <= SMs)
  int rows;        // rows per CTA tile (16 * row blocks)
  int tiles_n;     // CTA tiles along N
  int slabs;       // token slabs (ceil(M / (8 nt)))
  int splits;      // CTAs per slab
  int warps;       // stream-K workers (warps) per slab
  size_t smem;     // dynamic shared memory per CTA
  size_t ws_bytes; // workspace needed (0 when every CTA owns whole tiles)
};

SkinnyPlan plan_skinny(int M, int N, int K, int bits, int group, int mode, bool bf16, int sms,
                       bool force_streamk = false);
cudaError_t launch_skinny(const Problem& p, const SkinnyPlan& plan, void* workspace,
                          cudaStream_t stream);
// Decode path on the library's static scratch buffer (no allocation); sets
// *too_large instead of launching when the problem does not fit it.
cudaError_t launch_skinny_static(const Problem& p, int sms, cudaStream_t stream, bool* too_large);
size_t static_scratch_bytes();
unsigned skinny_read_and_clear_error();

// Stream-K plan of the tensor-core path (tcgen05, 4-bit codes).
struct TcPlan {
  int bn;          // tokens per tile (UMMA N)
  int ku;          // 64-column k blocks per unit of work (1 or 2)
  int tiles_n, tiles_m, nkb, ctas;   // nkb: units per tile
  size_t ws_bytes;
};

bool tc_supported(int bits, int mode, bool bf16, int group);
TcPlan plan_tc(int M, int N, int K, int mode, bool bf16, int group, int sms);
cudaError_t launch_tc(const Problem& p, const TcPlan& plan, void* workspace, long long wait_limit,
                      cudaStream_t stream);

// Clock cycles a kernel's barrier wait may take before the call gives up
// (qmm_set_wait_limit).
long long wait_limit();
unsigned tc_read_and_clear_error();

// Quantize + pack.  W2: second matrix of the gated layout (else null); perm:
// act-order column permutation (else null); zgroup / zbits: ASYM zero-point
// options (0 / 16 for the plain format).
cudaError_t launch_pack(const float* W, const float* W2, const int* perm, int N, int K, int mode,
                        int bits, int group, int zgroup, int zbits, const uint16_t* lut,
                        void* qweight, uint16_t* scales, void* zeros, cudaStream_t stream);
cudaError_t launch_dequant(const void* qweight, const uint16_t* scales,
                           const void* zeros_or_lut, int N, int K, int bits, int group,
                           int zgroup, int zbits, int mode, int out_dtype, void* W_out,
                           cudaStream_t stream);

// Act-order: perm from per-column group indices (*bad counts groups without
// exactly `group` members), and x'[m, j] = x[m, perm[j]].
cudaError_t launch_gidx_perm(const int* g_idx, int K, int group, int* perm, int* bad,
                             cudaStream_t stream);
cudaError_t launch_permute_x(const void* x, const int* perm, int M, int K, void* xp,
                             cudaStream_t stream);

int device_sms();

// cuTensorMapEncodeTiled from the driver (looked up once), or nullptr.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

}  // namespace qk
