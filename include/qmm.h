/* qmm -- weight-only quantized matrix multiply for NVIDIA B200 (sm_100a).
 *
 *   y[M, N] = x[M, K] . dequant(Wq)[N, K]^T
 *
 * x and y are fp16 or bf16; Wq holds 4-bit (or 2- or 3-bit, LUT mode) codes, decoded
 * on the fly inside the kernels as
 *   QMM_SYM   (q - 8) * s           symmetric, zero-point fixed at 8
 *   QMM_ASYM  (q - z) * s           fp16 zero-point per group
 *   QMM_LUT   T[q] * s              fp16 table of 2^bits entries
 * with one fp16 scale s (and zero z) per group of `group` weights along K, or
 * one per output row when group == -1.
 *
 * Sources for the operation:
 *  - "Does Marlin support zero-point quantization?" (IST-DASLab/marlin issue 5),
 *    reply by efrantar: fp16 x int4 matmul, symmetric linear quantization with
 *    the zero-point fixed at 8, column-wise or groupsize 128, fp16 scales; fp16
 *    zero-points as the asymmetric extension.
 *  - FLUTE project summary (sourcepulse.org), "How It Works": lookup-table
 *    quantization, value = table entry times a scale factor; 2-, 3- and 4-bit codes.
 *  - GPTQ-Triton project summary (sourcepulse.org), "How It Works": the
 *    quantized weights are decoded on the fly right before the multiply.
 *  - exllama discussion 24 (quoting the GPTQ paper): activations stay in
 *    floating point; the small-M product is bound by memory bandwidth.
 *
 * Conventions for every entry point:
 *  - Pointers named as device pointers must point to memory of the current CUDA
 *    device.  The caller allocates and owns every buffer; the library keeps no
 *    reference after the call returns.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call
 *    is asynchronous on that stream and never synchronizes the device.
 *  - The return value is a qmm_status.  Argument errors are detected on the
 *    host before anything is launched; launch errors come from
 *    cudaGetLastError right after the launch.  Errors raised later by a kernel
 *    (a bounded wait that ran out) are reported by qmm_check_error.
 *  - Shapes the GPU kernels accept: N % 16 == 0; K % 64 == 0 (4-bit) or
 *    K % 128 == 0 (2- and 3-bit); group == -1 or a power of two >= 16 that divides K;
 *    N, K <= 2^20; M >= 0.  Other shapes return QMM_ERR_UNSUPPORTED.
 *
 * Packed layout (written by qmm_pack, read by qmm and qmm_dequant):
 *  - qweight: N*K*bits/8 bytes.  Rows are taken in blocks of 16; each block is
 *    a run of K/KC chunks of 512 bytes (KC = 64 columns for 4-bit, 128 for
 *    2-bit).  Inside a chunk, lane l = 4g + t (g = 0..7, t = 0..3) owns bytes
 *    [16 l, 16 l + 16): rows g and g + 8 of the block and, in every 16-column
 *    tile j of the chunk, columns 16 j + 4 t + c (c = 0..3).  Those eight codes
 *    of a tile form four pairs p = h + 2 (c / 2) (h = 0 for row g, 1 for row
 *    g + 8) with member c % 2.  4-bit SYM/ASYM: tile j is 32-bit word j of the
 *    lane, pair p's members at nibbles p and p + 4.  4-bit LUT: word j, nibbles
 *    2p and 2p + 1.  2-bit LUT: word j / 2, byte 2 (j % 2) + p / 2, 2-bit field
 *    2 (p % 2) + (c % 2).  Words are little-endian; field f holds bits
 *    [bits*f, bits*f + bits).
 *    3-bit LUT (the FLUTE summary's 2/3/4-bit tables): chunks of 128 columns
 *    and 768 bytes, lane l owning bytes [24 l, 24 l + 24), read as one 192-bit
 *    little-endian string: tile j at bits [24 j, 24 j + 24), pair p at
 *    [24 j + 6 p, + 6), member c % 2 at + 3 (c % 2) -- each pair one 6-bit field.
 *  - scales (and zeros): fp16, G = K/group groups (1 for group -1), stored as
 *    [N/16][G][16] with row r of a block at position 2 (r % 8) + r / 8, i.e.
 *    rows g and g + 8 side by side.
 *  - LUT (zeros_or_lut in QMM_LUT mode): 2^bits fp16 entries in code order.
 */
#ifndef QMM_H
#define QMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { QMM_SYM = 0, QMM_ASYM = 1, QMM_LUT = 2 } qmm_mode;
typedef enum { QMM_F16 = 0, QMM_BF16 = 1 } qmm_dtype;
typedef enum {
  QMM_OK = 0,
  QMM_ERR_ARG = -1,          /* null pointer, negative size, bad enum value      */
  QMM_ERR_UNSUPPORTED = -2,  /* shape / mode / bits combination not implemented  */
  QMM_ERR_ALIGN = -3,        /* pointer not aligned as documented                */
  QMM_ERR_CUDA = -4,         /* a CUDA runtime call failed                       */
  QMM_ERR_TIMEOUT = -5,      /* a kernel gave up a bounded wait (qmm_check_error) */
  QMM_ERR_WORKSPACE = -6,    /* workspace smaller than qmm_workspace_size        */
  QMM_ERR_TOO_LARGE = -7     /* qmm_noalloc: problem exceeds the static scratch  */
} qmm_status;

/* Paths for qmm_with_path. */
/* Paths.  QMM_PATH_SKINNY_STREAMK is the decode path with its split-K plan
 * forced: for problems with few row tiles the decode path normally gives each
 * tile one CTA (its warps split K and add their sums in shared memory); this
 * value keeps the warp-level stream-K split with workspace partials instead
 * (for tests and tuning; same results within rounding). */
enum { QMM_PATH_AUTO = 0, QMM_PATH_SKINNY = 1, QMM_PATH_TENSOR = 2, QMM_PATH_SKINNY_STREAMK = 3 };

/* Byte sizes of the packed buffers for an [N, K] weight.  Returns the size of
 * qweight (N*K*bits/8) and writes the scale and zero buffer sizes (zeros: 0
 * unless QMM_ASYM) when the pointers are non-NULL.  Returns 0 for shapes the
 * packed layout does not cover. */
size_t qmm_packed_size(int N, int K, int bits, int group, int mode,
                       size_t* scales_bytes, size_t* zeros_bytes);

/* Quantize and pack fp32 weights (round to nearest, per group along K):
 *   SYM  s = absmax / 7,       q = clamp(rint(w / s) + 8, 0, 15)
 *   ASYM s = (max - min) / 15, z = clamp(rint(-min / s), 0, 15),
 *                              q = clamp(rint(w / s) + z, 0, 15)
 *   LUT  s = absmax,           q = argmin_i |w / s - T[i]| (lowest i on ties)
 * s is rounded to fp16 (saturating at 65504) before the codes are computed; all
 * divisions are IEEE fp32 and rint rounds half to even.  A group whose fp16
 * scale is 0 encodes every weight as 0 (SYM q = 8; ASYM z = q = 0; LUT the
 * entry nearest 0).
 *   W        device, fp32 [N, K] row-major, finite values.
 *   lut      device, 2^bits fp16 entries (QMM_LUT), else NULL.
 *   qweight  device, qmm_packed_size bytes, 16-byte aligned (written).
 *   scales   device, fp16, scales_bytes, 16-byte aligned (written).
 *   zeros    device, fp16, zeros_bytes, 16-byte aligned (QMM_ASYM, written), else NULL.
 * bits: 4 for SYM/ASYM; 4, 3 or 2 for LUT. */
int qmm_pack(const float* W, int N, int K, int mode, int bits, int group,
             const uint16_t* lut, void* qweight, uint16_t* scales, uint16_t* zeros,
             void* stream);

/* Bytes of workspace qmm needs for this problem (any path).  The workspace
 * holds split-K partial sums and per-tile arrival counters.  It must be zero
 * filled once before its first use; every completed call leaves the counters
 * at zero again, so it can be reused by later calls on the same stream.  Calls
 * that run at the same time (other streams) need separate workspaces.
 * 0 means the problem needs none. */
size_t qmm_workspace_size(int M, int N, int K, int bits, int group, int mode);

/* Workspace bytes for a call that takes path `path` (QMM_PATH_*); with
 * QMM_PATH_AUTO this is qmm_workspace_size. */
size_t qmm_workspace_size_for(int M, int N, int K, int bits, int group, int mode, int path);

/* y = x . dequant(Wq)^T.
 *   x             device, [M, K] row-major, xdtype (fp16 or bf16), 16-byte aligned.
 *   qweight, scales, zeros_or_lut
 *                 device, as written by qmm_pack (zeros for ASYM, the table
 *                 for LUT, NULL for SYM); scales and ASYM zeros 16-byte
 *                 aligned (they are copied in 16-byte pieces).  ASYM zeros are exact for integer
 *                 zero-points; a fractional zero is applied with one fp16 rounding.
 *   y             device, [M, N] row-major, same dtype as x, must not overlap x.
 *   workspace     device, workspace_bytes >= qmm_workspace_size(...), zero
 *                 filled before first use (see above); may be NULL with
 *                 workspace_bytes 0, in which case no cross-CTA split-K is used.
 * The accumulation is fp32.  M <= 32 runs the bandwidth-bound decode path
 * (one slab of up to 32 tokens; larger M in slabs of 32 where the tensor path
 * does not apply), larger M the tcgen05 tensor-core path, which takes 4-bit codes with
 * fp16 or bf16 activations in every mode and group (with bf16 activations and
 * group scales or a table, each weight enters as two bf16 parts, hi + lo).
 * Other combinations stay on the decode path.  qmm_path and qmm_path_ex tell
 * which.  The tensor path reads x through a TMA
 * tensor map, so x's row pitch (K * 2 bytes) must be a multiple of 16 -- true
 * for every K the packed layout allows. */
int qmm(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
        const uint16_t* zeros_or_lut, int M, int N, int K, int bits, int group, int mode,
        void* y, void* workspace, size_t workspace_bytes, void* stream);

/* qmm with the path chosen by the caller (QMM_PATH_*); QMM_PATH_AUTO is qmm. */
int qmm_with_path(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
                  const uint16_t* zeros_or_lut, int M, int N, int K, int bits, int group,
                  int mode, void* y, void* workspace, size_t workspace_bytes, void* stream,
                  int path);

/* The path qmm picks for this problem with fp16 activations (QMM_PATH_SKINNY
 * or QMM_PATH_TENSOR), or a negative qmm_status for an unsupported problem. */
int qmm_path(int M, int N, int K, int bits, int group, int mode);

/* The kernel a call runs (QMM_PATH_SKINNY or QMM_PATH_TENSOR) for activations
 * of type xdtype when the caller asks for `path` (QMM_PATH_*): QMM_PATH_AUTO
 * gives qmm's own choice, and a request for the tensor path reports
 * QMM_PATH_SKINNY where the tensor-core kernel does not take the combination
 * (2- and 3-bit codes; bf16 with group scales or a table; zero-point
 * options).  A negative qmm_status for invalid arguments. */
int qmm_path_ex(int M, int N, int K, int bits, int group, int mode, int xdtype, int path);

/* qmm for callers that cannot allocate device memory.  (This entry point is
 * an addition of this library; the sources describe no counterpart.)
 *
 * Some callers cannot call cudaMalloc: code that records work into a CUDA
 * graph under stream capture (allocation is not a capturable operation), or an
 * engine whose device memory is planned once at start-up and may not grow.
 * qmm needs a caller-provided workspace for its split-K partial sums; this
 * variant runs the same decode-path kernel on a scratch buffer the library
 * owns instead: a static device array of 8 MiB that every GPU which loads
 * the library holds until the process exits.  No call allocates: nothing here
 * calls cudaMalloc, cudaFree or an allocating library routine.
 *
 * Arguments are those of qmm without the workspace.  M must be at most 16
 * (one token slab of the decode path) and the problem's arrival counters must
 * fit the buffer; otherwise the call returns QMM_ERR_TOO_LARGE without
 * launching.  When the partial-sum slots of the usual plan do not fit, the
 * call uses fewer stream-K workers (slower, same result within rounding).
 *
 * The first call on a device looks up the buffer's device address
 * (cudaGetSymbolAddress, once per device, with that device current); make
 * that first call outside any stream capture.  Every call clears the buffer's
 * arrival counters (cudaMemsetAsync on `stream`) and then reuses the buffer,
 * which keeps the previous call's partial sums.  All calls share the one
 * buffer: calls that can run at the same time on the GPU (different streams
 * without ordering between them) race and may return wrong results. */
int qmm_noalloc(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
                const uint16_t* zeros_or_lut, int M, int N, int K, int bits, int group, int mode,
                void* y, void* stream);

/* Fused feed-forward gate: the GPTQ-Triton summary ("How It Works") fuses
 * the FFN layers into the quantized matmul.  For a LLaMA-style FFN with gate
 * and up projections Wg, Wu [I, K]:
 *
 *     y[M, I] = silu(x . dequant(Wg)^T) * (x . dequant(Wu)^T),  silu(v) = v / (1 + e^-v)
 *
 * in one pass over the codes of both matrices.
 *
 * qmm_pack_gated packs Wg and Wu (device, fp32 [I, K] row-major each, 16-byte
 * aligned) as one [2I, K] matrix in the layout of qmm_pack whose 16-row blocks
 * alternate: packed block 2b is rows 16b .. 16b + 15 of Wg, block 2b + 1 the
 * same rows of Wu.  Quantization is per row as in qmm_pack, so the codes,
 * scales and zeros equal those qmm_pack writes for that interleaved matrix.
 * Buffer sizes: qmm_packed_size(2 I, K, ...).  I must be a multiple of 16.
 *
 * qmm_gated runs the product on such a buffer (qweight, scales, zeros_or_lut
 * as written by qmm_pack_gated; I as given to it) and writes y [M, I] (same
 * dtype as x, must not overlap x); the sums are fp32 and the gate, the SiLU
 * and the product are taken in fp32 before the single rounding to y's type.
 * Workspace: qmm_workspace_size(M, 2 I, K, bits, group, mode) bytes, same
 * rules as qmm (NULL / 0 allowed).  Paths and statuses are those of qmm on
 * the [2I, K] problem. */
int qmm_pack_gated(const float* Wg, const float* Wu, int I, int K, int mode, int bits, int group,
                   const uint16_t* lut, void* qweight, uint16_t* scales, uint16_t* zeros,
                   void* stream);
int qmm_gated(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
              const uint16_t* zeros_or_lut, int M, int I, int K, int bits, int group, int mode,
              void* y, void* workspace, size_t workspace_bytes, void* stream);

/* ---- Zero-point options (asymmetric 4-bit codes).
 *
 * "Does Marlin support zero-point quantization?" (IST-DASLab/marlin issue 5):
 * efrantar's reply names zero-points quantized to low-bit integers, and
 * mobicham's reports HQQ+ runs with a zero-point group smaller than the
 * scale group (scale per row, zero-point per 8 weights).  Both are supported
 * for QMM_ASYM codes:
 *   zgroup  the zero-point group along K: -1 (the whole row) or a power of two
 *           >= 8 that divides K and the scale group (a zero group never
 *           straddles two scale groups; group -1 counts as K).  Equal to
 *           `group` gives the plain ASYM format.
 *   zbits   16: fp16 zero-points, [N/16][K/zgroup][16] in the slot order of
 *           the scales;  4: the integer zero-points 0..15 in 4 bits,
 *           [N/16][K/zgroup][8 bytes], slot i at byte i / 2, low nibble for
 *           even i.  Buffer size: qmm_zeros_size.
 * Codes, code layout and scales are those of QMM_ASYM.  Decode:
 *   w = (q - z[n, k / zgroup]) * s[n, k / group].
 * qmm_pack_asym quantizes: s = (max - min) / 15 over the scale group (rounded
 * to fp16 as in qmm_pack), then per zero group z = clamp(rint(-min_zg / s),
 * 0, 15) from the zero group's own minimum, q = clamp(rint(w / s) + z, 0, 15).
 * With zgroup == group and zbits == 16 every function below equals its plain
 * QMM_ASYM counterpart byte for byte.
 * qmm_asym runs the decode path for every M (the tensor-core path does not
 * take these formats; M > 16 runs in slabs of 16 tokens); zeros must be
 * 16-byte aligned; other arguments and statuses as for qmm. */
size_t qmm_zeros_size(int N, int K, int group, int zgroup, int zbits);
int qmm_pack_asym(const float* W, int N, int K, int group, int zgroup, int zbits, void* qweight,
                  uint16_t* scales, void* zeros, void* stream);
size_t qmm_workspace_size_asym(int M, int N, int K, int group, int zgroup, int zbits);
int qmm_asym(const void* x, int xdtype, const void* qweight, const uint16_t* scales,
             const void* zeros, int M, int N, int K, int group, int zgroup, int zbits, void* y,
             void* workspace, size_t workspace_bytes, void* stream);
int qmm_dequant_asym(const void* qweight, const uint16_t* scales, const void* zeros, int N, int K,
                     int group, int zgroup, int zbits, int out_dtype, void* W_out, void* stream);

/* ---- Act-order (GPTQ-Triton summary, "Limitations & Caveats": the act-order
 * option).  A GPTQ quantizer run with act-order forms its groups along its own
 * column order, so column k of W belongs to group g_idx[k] (int32, 0 .. K/group
 * - 1) and every group holds `group` columns.  The packed layout keeps each
 * group's columns together:
 *   perm    int32 [K], device, 16-byte aligned: packed column j holds original
 *           column perm[j]; group i occupies packed columns [i group,
 *           (i + 1) group), its members in ascending original column.
 * qmm_actorder_perm computes perm from g_idx on the device and writes to the
 * device int *bad_groups the number of groups that do not hold exactly
 * `group` columns (perm is incomplete unless it reads 0).  O(K^2 / group) work.
 * qmm_pack_actorder is qmm_pack for the weight whose packed column j is
 * W[:, perm[j]]: scales (zeros) are per act-order group, codes in packed
 * order (qmm_dequant of the result gives W~ in packed column order).
 * qmm_actorder computes y = x . W~^T over the original columns: it writes
 * x'[m, j] = x[m, perm[j]] into the workspace and runs qmm on x'.  Workspace:
 * qmm_workspace_size_actorder bytes (required; the first
 * qmm_workspace_size(...) bytes, rounded up to 256, follow qmm's rules, the rest
 * holds x'); y must overlap neither x nor the workspace.  perm entries
 * outside [0, K) read column 0 (no access outside W or x).  Other arguments
 * and statuses as for qmm_pack / qmm. */
int qmm_actorder_perm(const int32_t* g_idx, int K, int group, int32_t* perm, int32_t* bad_groups,
                      void* stream);
int qmm_pack_actorder(const float* W, const int32_t* perm, int N, int K, int mode, int bits,
                      int group, const uint16_t* lut, void* qweight, uint16_t* scales,
                      uint16_t* zeros, void* stream);
size_t qmm_workspace_size_actorder(int M, int N, int K, int bits, int group, int mode);
int qmm_actorder(const void* x, int xdtype, const int32_t* perm, const void* qweight,
                 const uint16_t* scales, const uint16_t* zeros_or_lut, int M, int N, int K,
                 int bits, int group, int mode, void* y, void* workspace, size_t workspace_bytes,
                 void* stream);

/* Decode the packed weights into W_out[N, K] row-major (fp16 or bf16 by
 * out_dtype): W_out = round_to_nearest_even((q - z) * s) (SYM z = 8) or
 * round(T[q] * s), the product taken exactly in fp32 (exact for integer
 * zero-points).  For tests and inspection; not on the matmul path. */
int qmm_dequant(const void* qweight, const uint16_t* scales, const uint16_t* zeros_or_lut,
                int N, int K, int bits, int group, int mode, int out_dtype, void* W_out,
                void* stream);

/* Synchronizes `stream`, then reads and clears the library's device error word
 * on the current device: QMM_OK, or QMM_ERR_TIMEOUT if a kernel abandoned a
 * bounded wait since the last check.  The output of such a call is undefined,
 * and a workspace it used may hold nonzero arrival counters: zero it again
 * before reusing it. */
int qmm_check_error(void* stream);

/* Failure detection.  Every wait a kernel makes on another part of itself
 * (a copy landing, a stage being freed, an MMA finishing) is bounded: after
 * `cycles` SM clock cycles without progress the CTA gives up, drains the
 * copies and MMAs it has issued (those waits have a fixed bound of about
 * 2 s), frees its tensor memory and exits, and qmm_check_error reports
 * QMM_ERR_TIMEOUT.  The default is about 2 s at B200 clocks; cycles <= 0
 * restores it.  A tiny value makes a call give up on purpose, which is how the
 * error path is tested.  Applies to calls launched afterwards, process-wide;
 * returns the previous value.  (Waits of the tensor-core path; the decode path
 * waits only for its own asynchronous copies, which always complete.) */
long long qmm_set_wait_limit(long long cycles);

/* Static description of a status code. */
const char* qmm_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* QMM_H */
