// C-ABI of libqmm: argument checks, path choice (M-based dispatch) and launch.
// The declarations, their meaning and the packed layout are in include/qmm.h.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace qk {

int device_sms() {
  static int sms[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!sms[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    sms[dev] = v > 0 ? v : 148;
  }
  return sms[dev];
}

// About 2 s of SM clock: a wait this long means something is wrong.
constexpr long long kDefaultWaitCycles = 4000000000ll;
std::atomic<long long> g_wait_cycles{kDefaultWaitCycles};

long long wait_limit() { return g_wait_cycles.load(std::memory_order_relaxed); }

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(int N, int K, int bits, int group, int mode) {
  if (N <= 0 || K <= 0) return QMM_ERR_ARG;
  if (mode != QMM_SYM && mode != QMM_ASYM && mode != QMM_LUT) return QMM_ERR_ARG;
  if (bits < 2 || bits > 4) return QMM_ERR_ARG;
  if (bits != 4 && mode != QMM_LUT) return QMM_ERR_UNSUPPORTED;   // 2- and 3-bit: LUT only
  if (N % 16 != 0 || K % chunk_cols(bits) != 0) return QMM_ERR_UNSUPPORTED;
  if (N > (1 << 20) || K > (1 << 20)) return QMM_ERR_UNSUPPORTED;   // 32-bit work indexing
  // groups: one per row (-1) or a power of two >= 16 dividing K
  if (group != -1 && (group < 16 || (group & (group - 1)) != 0 || K % group != 0))
    return QMM_ERR_UNSUPPORTED;
  return QMM_OK;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? QMM_OK : QMM_ERR_CUDA; }

// Zero-point options: zbits 16 (fp16) or 4; the zero group is -1 (the row) or
// a power of two >= 8 that divides K and nests inside the scale group.
int check_zopts(int K, int group, int zgroup, int zbits) {
  if (zbits != 16 && zbits != 4) return QMM_ERR_ARG;
  if (zgroup != -1 && (zgroup < 8 || (zgroup & (zgroup - 1)) != 0 || K % zgroup != 0))
    return QMM_ERR_UNSUPPORTED;
  const int L = group == -1 ? K : group, LZ = zgroup == -1 ? K : zgroup;
  if (LZ > L || L % LZ != 0) return QMM_ERR_UNSUPPORTED;
  return QMM_OK;
}

// Internal (mode, zgroup) of an ASYM format with zero-point options: the plain
// ASYM format when the zero group is the scale group and zeros are fp16.
void zero_mode(int K, int group, int zgroup, int zbits, int* mode, int* zg) {
  const int L = group == -1 ? K : group, LZ = zgroup == -1 ? K : zgroup;
  *zg = LZ == L ? 0 : zgroup;
  *mode = zbits == 4 ? (LZ >= 128 ? kASYMQ1 : kASYMQ) : (*zg == 0 ? QMM_ASYM : kASYMX);
}

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// Decode path while the product is bandwidth-bound (few tokens), tensor-core
// path once it becomes a dense contraction.  The crossover was measured on
// B200 (K = 4096 / 8192, N = 4096 .. 14336, SYM fp16, ASYM bf16, LUT, M = 24 ..
// 64): one 32-token slab of the decode path reads the weights once and wins or
// ties up to M = 32; above that it needs a second slab (a second read of the
// weights) and the tensor path, which reads them once, is 1.3-2x faster.
// Combinations the tensor path does not cover (2- and 3-bit codes; zero-point
// options) take the decode path, in slabs of 32 tokens.
int choose_path(int M, int N, int bits, int mode, bool bf16, int group) {
  (void)N;
  if (!tc_supported(bits, mode, bf16, group)) return QMM_PATH_SKINNY;
  if (M <= 32) return QMM_PATH_SKINNY;
  return QMM_PATH_TENSOR;
}

// The plan a call runs with; `ws_bytes` is what it needs from the workspace.
struct Plan {
  int path;
  SkinnyPlan sk;
  TcPlan tc;
  size_t ws_bytes() const { return path == QMM_PATH_TENSOR ? tc.ws_bytes : sk.ws_bytes; }
};

// `mode` may be an internal zero-point-options mode (kASYMX, kASYMQ, kASYMQ1).
Plan make_plan(int M, int N, int K, int bits, int group, int mode, bool bf16, int path) {
  Plan p{};
  const bool streamk = path == QMM_PATH_SKINNY_STREAMK;
  p.path = path == QMM_PATH_AUTO ? choose_path(M, N, bits, mode, bf16, group)
           : streamk            ? QMM_PATH_SKINNY
                                : path;
  if (p.path == QMM_PATH_TENSOR && !tc_supported(bits, mode, bf16, group)) p.path = QMM_PATH_SKINNY;
  if (p.path == QMM_PATH_TENSOR) p.tc = plan_tc(M, N, K, mode, bf16, group, device_sms());
  else p.sk = plan_skinny(M, N, K, bits, group, mode, bf16, device_sms(), streamk);
  return p;
}

}  // namespace
}  // namespace qk

using namespace qk;

static int run_qmm(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
                   const uint16_t* zeros_or_lut, int M, int N, int K, int bits, int group,
                   int mode, void* y, void* workspace, size_t workspace_bytes, void* stream,
                   int path, bool gated, int zgroup = 0, int zbits = 16) {
  if (M < 0) return QMM_ERR_ARG;
  int st = check_shape(N, K, bits, group, zero_opts(mode) ? QMM_ASYM : mode);
  if (st != QMM_OK) return st;
  if (xdtype != QMM_F16 && xdtype != QMM_BF16) return QMM_ERR_ARG;
  if (path < QMM_PATH_AUTO || path > QMM_PATH_SKINNY_STREAMK) return QMM_ERR_ARG;
  if (M == 0) return QMM_OK;
  if (!x || !qweight || !scales || !y) return QMM_ERR_ARG;
  if (mode != QMM_SYM && !zeros_or_lut) return QMM_ERR_ARG;
  if (!aligned(x, 16) || !aligned(qweight, 16) || !aligned(scales, 16) || !aligned(y, 2) ||
      ((mode == QMM_ASYM || zero_opts(mode)) && !aligned(zeros_or_lut, 16)) ||
      (workspace && !aligned(workspace, 256)))
    return QMM_ERR_ALIGN;
  {
    const char* xb = static_cast<const char*>(x);
    const char* yb = static_cast<const char*>(y);
    const size_t xs = (size_t)M * K * 2, ys = (size_t)M * (gated ? N / 2 : N) * 2;
    if (xb < yb + ys && yb < xb + xs) return QMM_ERR_ARG;   // y overlaps x
  }
  Problem p{x, xdtype == QMM_BF16, qweight, scales, zeros_or_lut, M, N, K, bits, group, mode, y};
  p.gated = gated;
  p.zgroup = zgroup;
  p.zbits = zbits;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Plan plan = make_plan(M, N, K, bits, group, mode, xdtype == QMM_BF16, path);
  if (plan.ws_bytes()) {
    if (!workspace) {
      // no workspace: every CTA owns whole tiles over all of K, no partial sums
      if (plan.path == QMM_PATH_TENSOR) {
        plan.tc.ctas = plan.tc.tiles_n * plan.tc.tiles_m;
        plan.tc.ws_bytes = 0;
      } else {
        plan.sk.warps = plan.sk.tiles_n;
        plan.sk.splits = (plan.sk.tiles_n + 7) / 8;
        plan.sk.ws_bytes = 0;
      }
    } else if (workspace_bytes < plan.ws_bytes()) {
      return QMM_ERR_WORKSPACE;
    }
  }
  if (plan.path == QMM_PATH_TENSOR)
    return status_of(launch_tc(p, plan.tc, workspace, wait_limit(), s));
  return status_of(launch_skinny(p, plan.sk, workspace, s));
}


extern "C" {

size_t qmm_packed_size(int N, int K, int bits, int group, int mode, size_t* scales_bytes,
                       size_t* zeros_bytes) {
  if (check_shape(N, K, bits, group, mode) != QMM_OK) return 0;
  const size_t G = group == -1 ? 1 : (size_t)(K / group);
  if (scales_bytes) *scales_bytes = (size_t)N * G * 2;
  if (zeros_bytes) *zeros_bytes = mode == QMM_ASYM ? (size_t)N * G * 2 : 0;
  return (size_t)N * K * bits / 8;
}

int qmm_pack(const float* W, int N, int K, int mode, int bits, int group, const uint16_t* lut,
             void* qweight, uint16_t* scales, uint16_t* zeros, void* stream) {
  int st = check_shape(N, K, bits, group, mode);
  if (st != QMM_OK) return st;
  if (!W || !qweight || !scales) return QMM_ERR_ARG;
  if (mode == QMM_ASYM && !zeros) return QMM_ERR_ARG;
  if (mode == QMM_LUT && !lut) return QMM_ERR_ARG;
  if (!aligned(W, 16) || !aligned(qweight, 16) || !aligned(scales, 16) ||
      (zeros && !aligned(zeros, 16)))
    return QMM_ERR_ALIGN;
  return status_of(launch_pack(W, nullptr, nullptr, N, K, mode, bits, group, 0, 16, lut, qweight,
                               scales, zeros, static_cast<cudaStream_t>(stream)));
}

int qmm_pack_gated(const float* Wg, const float* Wu, int I, int K, int mode, int bits, int group,
                   const uint16_t* lut, void* qweight, uint16_t* scales, uint16_t* zeros,
                   void* stream) {
  if (I <= 0 || I > (1 << 19)) return I <= 0 ? QMM_ERR_ARG : QMM_ERR_UNSUPPORTED;
  int st = check_shape(2 * I, K, bits, group, mode);
  if (st != QMM_OK) return st;
  if (I % 16 != 0) return QMM_ERR_UNSUPPORTED;
  if (!Wg || !Wu || !qweight || !scales) return QMM_ERR_ARG;
  if (mode == QMM_ASYM && !zeros) return QMM_ERR_ARG;
  if (mode == QMM_LUT && !lut) return QMM_ERR_ARG;
  if (!aligned(Wg, 16) || !aligned(Wu, 16) || !aligned(qweight, 16) || !aligned(scales, 16) ||
      (zeros && !aligned(zeros, 16)))
    return QMM_ERR_ALIGN;
  return status_of(launch_pack(Wg, Wu, nullptr, 2 * I, K, mode, bits, group, 0, 16, lut, qweight,
                               scales, zeros, static_cast<cudaStream_t>(stream)));
}

int qmm_path(int M, int N, int K, int bits, int group, int mode) {
  if (M < 0) return QMM_ERR_ARG;
  int st = check_shape(N, K, bits, group, mode);
  if (st != QMM_OK) return st;
  return choose_path(M, N, bits, mode, false, group);
}

int qmm_path_ex(int M, int N, int K, int bits, int group, int mode, int xdtype, int path) {
  if (M < 0) return QMM_ERR_ARG;
  int st = check_shape(N, K, bits, group, mode);
  if (st != QMM_OK) return st;
  if (xdtype != QMM_F16 && xdtype != QMM_BF16) return QMM_ERR_ARG;
  if (path < QMM_PATH_AUTO || path > QMM_PATH_SKINNY_STREAMK) return QMM_ERR_ARG;
  return make_plan(std::max(M, 1), N, K, bits, group, mode, xdtype == QMM_BF16, path).path;
}

size_t qmm_workspace_size_for(int M, int N, int K, int bits, int group, int mode, int path) {
  if (M <= 0 || check_shape(N, K, bits, group, mode) != QMM_OK) return 0;
  if (path < QMM_PATH_AUTO || path > QMM_PATH_SKINNY_STREAMK) return 0;
  // the activation dtype is not an argument here: size for the larger of the two
  return std::max(make_plan(M, N, K, bits, group, mode, false, path).ws_bytes(),
                  make_plan(M, N, K, bits, group, mode, true, path).ws_bytes());
}

size_t qmm_workspace_size(int M, int N, int K, int bits, int group, int mode) {
  return qmm_workspace_size_for(M, N, K, bits, group, mode, QMM_PATH_AUTO);
}

int qmm_with_path(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
                  const uint16_t* zeros_or_lut, int M, int N, int K, int bits, int group,
                  int mode, void* y, void* workspace, size_t workspace_bytes, void* stream,
                  int path) {
  return run_qmm(x, xdtype, qweight, scales, zeros_or_lut, M, N, K, bits, group, mode, y,
                 workspace, workspace_bytes, stream, path, false);
}

int qmm_gated(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
              const uint16_t* zeros_or_lut, int M, int I, int K, int bits, int group, int mode,
              void* y, void* workspace, size_t workspace_bytes, void* stream) {
  if (I <= 0) return QMM_ERR_ARG;
  if (I % 16 != 0 || I > (1 << 19)) return QMM_ERR_UNSUPPORTED;
  return run_qmm(x, xdtype, qweight, scales, zeros_or_lut, M, 2 * I, K, bits, group, mode, y,
                 workspace, workspace_bytes, stream, QMM_PATH_AUTO, true);
}

int qmm(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
        const uint16_t* zeros_or_lut, int M, int N, int K, int bits, int group, int mode, void* y,
        void* workspace, size_t workspace_bytes, void* stream) {
  return qmm_with_path(x, xdtype, qweight, scales, zeros_or_lut, M, N, K, bits, group, mode, y,
                       workspace, workspace_bytes, stream, QMM_PATH_AUTO);
}

int qmm_noalloc(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
                const uint16_t* zeros_or_lut, int M, int N, int K, int bits, int group, int mode,
                void* y, void* stream) {
  if (M < 0) return QMM_ERR_ARG;
  int st = check_shape(N, K, bits, group, mode);
  if (st != QMM_OK) return st;
  if (xdtype != QMM_F16 && xdtype != QMM_BF16) return QMM_ERR_ARG;
  if (M > 16) return QMM_ERR_TOO_LARGE;
  if (M == 0) return QMM_OK;
  if (!x || !qweight || !scales || !y) return QMM_ERR_ARG;
  if (mode != QMM_SYM && !zeros_or_lut) return QMM_ERR_ARG;
  if (!aligned(x, 16) || !aligned(qweight, 16) || !aligned(scales, 16) || !aligned(y, 2) ||
      (mode == QMM_ASYM && !aligned(zeros_or_lut, 16)))
    return QMM_ERR_ALIGN;
  {
    const char* xb = static_cast<const char*>(x);
    const char* yb = static_cast<const char*>(y);
    const size_t xs = (size_t)M * K * 2, ys = (size_t)M * N * 2;
    if (xb < yb + ys && yb < xb + xs) return QMM_ERR_ARG;   // y overlaps x
  }
  Problem p{x, xdtype == QMM_BF16, qweight, scales, zeros_or_lut, M, N, K, bits, group, mode, y};
  bool too_large = false;
  const cudaError_t e =
      launch_skinny_static(p, device_sms(), static_cast<cudaStream_t>(stream), &too_large);
  if (too_large) return QMM_ERR_TOO_LARGE;
  return status_of(e);
}

int qmm_dequant(const void* qweight, const uint16_t* scales, const uint16_t* zeros_or_lut, int N,
                int K, int bits, int group, int mode, int out_dtype, void* W_out, void* stream) {
  int st = check_shape(N, K, bits, group, mode);
  if (st != QMM_OK) return st;
  if (out_dtype != QMM_F16 && out_dtype != QMM_BF16) return QMM_ERR_ARG;
  if (!qweight || !scales || !W_out) return QMM_ERR_ARG;
  if (mode != QMM_SYM && !zeros_or_lut) return QMM_ERR_ARG;
  if (!aligned(qweight, 16) || !aligned(W_out, 8)) return QMM_ERR_ALIGN;
  return status_of(launch_dequant(qweight, scales, zeros_or_lut, N, K, bits, group, 0, 16, mode,
                                  out_dtype, W_out, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------ zero-point options

size_t qmm_zeros_size(int N, int K, int group, int zgroup, int zbits) {
  if (check_shape(N, K, 4, group, QMM_ASYM) != QMM_OK) return 0;
  if (check_zopts(K, group, zgroup, zbits) != QMM_OK) return 0;
  const size_t GZ = (size_t)K / (zgroup == -1 ? K : zgroup);
  return zbits == 4 ? (size_t)N * GZ / 2 : (size_t)N * GZ * 2;
}

int qmm_pack_asym(const float* W, int N, int K, int group, int zgroup, int zbits, void* qweight,
                  uint16_t* scales, void* zeros, void* stream) {
  int st = check_shape(N, K, 4, group, QMM_ASYM);
  if (st != QMM_OK) return st;
  st = check_zopts(K, group, zgroup, zbits);
  if (st != QMM_OK) return st;
  if (!W || !qweight || !scales || !zeros) return QMM_ERR_ARG;
  if (!aligned(W, 16) || !aligned(qweight, 16) || !aligned(scales, 16) || !aligned(zeros, 16))
    return QMM_ERR_ALIGN;
  int mode, zg;
  zero_mode(K, group, zgroup, zbits, &mode, &zg);
  return status_of(launch_pack(W, nullptr, nullptr, N, K, QMM_ASYM, 4, group, zg, zbits, nullptr,
                               qweight, scales, zeros, static_cast<cudaStream_t>(stream)));
}

size_t qmm_workspace_size_asym(int M, int N, int K, int group, int zgroup, int zbits) {
  if (M <= 0 || check_shape(N, K, 4, group, QMM_ASYM) != QMM_OK) return 0;
  if (check_zopts(K, group, zgroup, zbits) != QMM_OK) return 0;
  int mode, zg;
  zero_mode(K, group, zgroup, zbits, &mode, &zg);
  return std::max(make_plan(M, N, K, 4, group, mode, false, QMM_PATH_AUTO).ws_bytes(),
                  make_plan(M, N, K, 4, group, mode, true, QMM_PATH_AUTO).ws_bytes());
}

int qmm_asym(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
             const void* zeros, int M, int N, int K, int group, int zgroup, int zbits, void* y,
             void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_shape(N, K, 4, group, QMM_ASYM);
  if (st != QMM_OK) return st;
  st = check_zopts(K, group, zgroup, zbits);
  if (st != QMM_OK) return st;
  int mode, zg;
  zero_mode(K, group, zgroup, zbits, &mode, &zg);
  return run_qmm(x, xdtype, qweight, scales, static_cast<const uint16_t*>(zeros), M, N, K, 4,
                 group, mode, y, workspace, workspace_bytes, stream, QMM_PATH_AUTO, false, zg,
                 zbits);
}

int qmm_dequant_asym(const void* qweight, const uint16_t* scales, const void* zeros, int N, int K,
                     int group, int zgroup, int zbits, int out_dtype, void* W_out, void* stream) {
  int st = check_shape(N, K, 4, group, QMM_ASYM);
  if (st != QMM_OK) return st;
  st = check_zopts(K, group, zgroup, zbits);
  if (st != QMM_OK) return st;
  if (out_dtype != QMM_F16 && out_dtype != QMM_BF16) return QMM_ERR_ARG;
  if (!qweight || !scales || !zeros || !W_out) return QMM_ERR_ARG;
  if (!aligned(qweight, 16) || !aligned(W_out, 8)) return QMM_ERR_ALIGN;
  int mode, zg;
  zero_mode(K, group, zgroup, zbits, &mode, &zg);
  return status_of(launch_dequant(qweight, scales, zeros, N, K, 4, group, zg, zbits, QMM_ASYM,
                                  out_dtype, W_out, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- act-order

int qmm_actorder_perm(const int32_t* g_idx, int K, int group, int32_t* perm, int32_t* bad_groups,
                      void* stream) {
  if (K <= 0 || K > (1 << 20)) return K <= 0 ? QMM_ERR_ARG : QMM_ERR_UNSUPPORTED;
  if (group != -1 && (group < 16 || (group & (group - 1)) != 0 || K % group != 0))
    return QMM_ERR_UNSUPPORTED;
  if (!g_idx || !perm || !bad_groups) return QMM_ERR_ARG;
  if (!aligned(g_idx, 4) || !aligned(perm, 4) || !aligned(bad_groups, 4)) return QMM_ERR_ALIGN;
  return status_of(launch_gidx_perm(g_idx, K, group, perm, bad_groups,
                                    static_cast<cudaStream_t>(stream)));
}

int qmm_pack_actorder(const float* W, const int32_t* perm, int N, int K, int mode, int bits,
                      int group, const uint16_t* lut, void* qweight, uint16_t* scales,
                      uint16_t* zeros, void* stream) {
  int st = check_shape(N, K, bits, group, mode);
  if (st != QMM_OK) return st;
  if (!W || !perm || !qweight || !scales) return QMM_ERR_ARG;
  if (mode == QMM_ASYM && !zeros) return QMM_ERR_ARG;
  if (mode == QMM_LUT && !lut) return QMM_ERR_ARG;
  if (!aligned(W, 16) || !aligned(perm, 16) || !aligned(qweight, 16) || !aligned(scales, 16) ||
      (zeros && !aligned(zeros, 16)))
    return QMM_ERR_ALIGN;
  return status_of(launch_pack(W, nullptr, perm, N, K, mode, bits, group, 0, 16, lut, qweight,
                               scales, zeros, static_cast<cudaStream_t>(stream)));
}

size_t qmm_workspace_size_actorder(int M, int N, int K, int bits, int group, int mode) {
  if (M <= 0 || check_shape(N, K, bits, group, mode) != QMM_OK) return 0;
  return round256(qmm_workspace_size(M, N, K, bits, group, mode)) + round256((size_t)M * K * 2);
}

int qmm_actorder(const void* x, int xdtype, const int32_t* perm, const void* qweight,
                 const uint16_t* scales, const uint16_t* zeros_or_lut, int M, int N, int K,
                 int bits, int group, int mode, void* y, void* workspace, size_t workspace_bytes,
                 void* stream) {
  if (M < 0) return QMM_ERR_ARG;
  int st = check_shape(N, K, bits, group, mode);
  if (st != QMM_OK) return st;
  if (xdtype != QMM_F16 && xdtype != QMM_BF16) return QMM_ERR_ARG;
  if (M == 0) return QMM_OK;
  if (!x || !perm || !y || !qweight || !scales) return QMM_ERR_ARG;
  if (mode != QMM_SYM && !zeros_or_lut) return QMM_ERR_ARG;
  if (!aligned(x, 16) || !aligned(perm, 16) || !aligned(qweight, 16) || !aligned(scales, 16) ||
      !aligned(y, 2) || (mode == QMM_ASYM && !aligned(zeros_or_lut, 16)) ||
      (workspace && !aligned(workspace, 256)))
    return QMM_ERR_ALIGN;
  // the workspace holds the product's own workspace, then x in packed column order
  const size_t plain = round256(qmm_workspace_size(M, N, K, bits, group, mode));
  if (!workspace || workspace_bytes < plain + (size_t)M * K * 2) return QMM_ERR_WORKSPACE;
  {
    const char* xb = static_cast<const char*>(x);
    const char* yb = static_cast<const char*>(y);
    const char* wb = static_cast<const char*>(workspace);
    const size_t xs = (size_t)M * K * 2, ys = (size_t)M * N * 2, ws = plain + xs;
    if (xb < yb + ys && yb < xb + xs) return QMM_ERR_ARG;   // y overlaps x
    if (wb < yb + ys && yb < wb + ws) return QMM_ERR_ARG;   // y overlaps the workspace
  }
  void* xp = static_cast<char*>(workspace) + plain;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = status_of(launch_permute_x(x, perm, M, K, xp, s));
  if (st != QMM_OK) return st;
  return run_qmm(xp, xdtype, qweight, scales, zeros_or_lut, M, N, K, bits, group, mode, y,
                 workspace, plain, stream, QMM_PATH_AUTO, false);
}

long long qmm_set_wait_limit(long long cycles) {
  const long long v = cycles > 0 ? cycles : kDefaultWaitCycles;
  return g_wait_cycles.exchange(v, std::memory_order_relaxed);
}

int qmm_check_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QMM_ERR_CUDA;
  const unsigned v = tc_read_and_clear_error();
  const unsigned w = skinny_read_and_clear_error();
  if (v == 0xFFFFFFFFu || w == 0xFFFFFFFFu) return QMM_ERR_CUDA;
  return (v | w) ? QMM_ERR_TIMEOUT : QMM_OK;
}

const char* qmm_strerror(int status) {
  switch (status) {
    case QMM_OK: return "ok";
    case QMM_ERR_ARG: return "invalid argument (null pointer, negative size or bad enum value)";
    case QMM_ERR_UNSUPPORTED: return "unsupported shape, mode or bit width";
    case QMM_ERR_ALIGN: return "pointer not aligned as required";
    case QMM_ERR_CUDA: return "CUDA runtime error";
    case QMM_ERR_TIMEOUT: return "a kernel abandoned a bounded wait";
    case QMM_ERR_WORKSPACE: return "workspace smaller than qmm_workspace_size";
    case QMM_ERR_TOO_LARGE:
      return "problem does not fit the library's static scratch buffer (qmm_noalloc: M <= 16)";
    default: return "unknown status";
  }
}

}  // extern "C"
