// CPU oracle for the weight-only quantized matmul  y = x . dequant(Wq)^T.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
// baseline of the benchmark may load this library.  It shares no code, header,
// table or constant with the CUDA library; the two meet only at the byte
// layout that both implement from its written definition.
//
// Plain, slow and direct on purpose: one element at a time, the steps in the
// order the sources give them, double precision for the matmul sums.
//
// Sources (web pages on weight-only low-bit quantization):
//  [MZ]  "Does Marlin support zero-point quantization?" (githubissues.com,
//        IST-DASLab/marlin issue 5), reply by efrantar: a general fp16 x int4
//        matmul with symmetric linear quantization, column-wise or groupsize 128,
//        fp16 scales; zero-point fixed to 8; fp16 zero-points as the natural
//        extension.
//  [FL]  FLUTE project summary (sourcepulse.org, project 1846613), "How It
//        Works": a lookup table maps each code to a de-quantized value, which a
//        scale factor multiplies; 2/3/4-bit codes; NF4-style tables.
//  [GT]  GPTQ-Triton project summary (sourcepulse.org, project 1838626),
//        "How It Works" / "Highlighted Details": weights decoded on the fly
//        before the matmul; group size -1 (one group per output column).
//  [EX]  exllama discussion 24, "Regarding comment on benchmark memory
//        bandwidth speeds" (quoting the GPTQ paper): activations are not
//        quantized; only the weights are, and are de-quantized when needed.
//
// Readings where the sources are silent (each also listed in the design notes):
//  R1 round() is round-half-to-even (rintf in the default rounding mode).
//  R2 the scale is rounded to fp16 first; codes are computed with that fp16
//     scale, so encode and decode agree.  An fp16 overflow saturates to 65504.
//  R3 true IEEE fp32 division w / s (no reciprocal multiply, no FMA contraction).
//  R4 asymmetric zero-point z = clamp(rint(-min / s), 0, 15), an integer held
//     in fp16.
//  R5 a group whose fp16 scale is 0 encodes every value as 0: SYM q = 8,
//     ASYM z = 0 and q = 0, LUT q = index of the entry nearest 0.
//  R6 LUT encode: q = argmin_i |w/s - T[i]| in fp32, the lowest index on ties.
//  R7 group = -1 means one group spanning the whole row (all of K).
//
// Packed layout (the library's documented format, restated here from its
// definition; see the functions code_place and scale_index):
//  * codes: row blocks of 16 rows; per row block, K/KC chunks of KC columns
//    (KC = 64 for 4-bit, 128 for 2-bit), each chunk 512 bytes.  Inside a chunk
//    lane l = 4g + t (g = 0..7, t = 0..3) owns bytes [16 l, 16 l + 16): rows g
//    and g + 8 of the block, and in every 16-column tile j of the chunk the
//    four columns 16 j + 4 t + c, c = 0..3.  The eight codes of one tile for one
//    lane form four pairs p = 0..3: p = h + 2 (c / 2) where h = 0 for row g and
//    1 for row g + 8, and (c % 2) selects the low or high member of the pair.
//      4-bit SYM/ASYM: word j of the lane; pair p low -> nibble p, high ->
//                      nibble p + 4.
//      4-bit LUT:      word j of the lane; pair p low -> nibble 2p, high ->
//                      nibble 2p + 1.
//      2-bit LUT:      word j/2 of the lane, byte 2 (j % 2) + p / 2; inside the
//                      byte the 2-bit field 2 (p % 2) + (c % 2).
//      3-bit LUT:      chunks of 128 columns and 768 bytes, lane l owning bytes
//                      [24 l, 24 l + 24), read as one 192-bit little-endian
//                      string: tile j at bits [24 j, 24 j + 24), pair p at
//                      [24 j + 6 p, + 6), member c % 2 at + 3 (c % 2) -- a pair is
//                      one 6-bit field.
//    Words are little-endian uint32; nibble/field f occupies bits [b f, b f + b).
//  * scales (and ASYM zeros): fp16, [N/16][G][16]; inside the 16 the row r of
//    the block sits at 2 (r % 8) + r / 8.
//  * LUT: 2^bits fp16 entries, plain order.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <cstddef>

namespace {

enum { MODE_SYM = 0, MODE_ASYM = 1, MODE_LUT = 2 };
enum { DT_F16 = 0, DT_BF16 = 1 };
enum { OK = 0, ERR_ARG = -1 };

// ---------------------------------------------------------------- conversions

// fp16 bits -> exact value.
double half_value(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0)
    v = std::ldexp((double)m, -24);                  // subnormal: m * 2^-24
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = std::ldexp((double)(1024 + m), e - 25);      // (1 + m/1024) * 2^(e-15)
  return sign ? -v : v;
}

// bf16 bits -> exact value (the upper half of an fp32).
double bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// Round a finite double to the nearest multiple of `quantum`, ties to even
// multiple.  `quantum` is a power of two, so v / quantum is exact.
double round_to_quantum(double v, double quantum) {
  double q = v / quantum;
  double f = std::floor(q);
  double d = q - f;
  if (d > 0.5 || (d == 0.5 && std::fmod(f, 2.0) != 0.0)) f += 1.0;
  return f * quantum;
}

// Value -> fp16 bits, round to nearest even (IEEE binary16: 10 fraction bits,
// exponent -14..15, subnormal quantum 2^-24, overflow to infinity).
uint16_t half_bits(double v) {
  if (std::isnan(v)) return 0x7e00;
  uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  double a = std::fabs(v);
  if (a == 0.0) return sign;
  int e;
  std::frexp(a, &e);                       // a in [2^(e-1), 2^e)
  int exp = e - 1;                         // a in [2^exp, 2^(exp+1))
  if (exp < -14) exp = -14;                // subnormal range shares 2^-24 quantum
  double r = round_to_quantum(a, std::ldexp(1.0, exp - 10));
  if (r >= 65536.0) return sign | 0x7c00;  // rounded past the largest finite
  if (r < std::ldexp(1.0, -14))            // subnormal (or zero)
    return sign | (uint16_t)(r / std::ldexp(1.0, -24));
  std::frexp(r, &e);
  exp = e - 1;                             // rounding may have bumped the binade
  uint16_t frac = (uint16_t)(r / std::ldexp(1.0, exp - 10) - 1024.0);
  return sign | (uint16_t)((exp + 15) << 10) | frac;
}

// Value -> bf16 bits, round to nearest even (8 significant bits, fp32 range).
uint16_t bf16_bits(double v) {
  if (std::isnan(v)) return 0x7fc0;
  uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  double a = std::fabs(v);
  if (a == 0.0) return sign;
  int e;
  std::frexp(a, &e);
  int exp = e - 1;
  if (exp < -126) exp = -126;
  double r = round_to_quantum(a, std::ldexp(1.0, exp - 7));
  if (r >= std::ldexp(1.0, 128)) return sign | 0x7f80;
  if (r < std::ldexp(1.0, -126))
    return sign | (uint16_t)(r / std::ldexp(1.0, -133));
  std::frexp(r, &e);
  exp = e - 1;
  uint16_t frac = (uint16_t)(r / std::ldexp(1.0, exp - 7) - 128.0);
  return sign | (uint16_t)((exp + 127) << 7) | frac;
}

// R2: fp16 scale, saturated to the largest finite fp16 instead of infinity.
uint16_t scale_bits(float s32) {
  uint16_t h = half_bits((double)s32);
  if ((h & 0x7fff) == 0x7c00) h = (h & 0x8000) | 0x7bff;
  return h;
}

// ------------------------------------------------------------------- layout

int n_groups(int K, int group) { return group == -1 ? 1 : K / group; }
int group_len(int K, int group) { return group == -1 ? K : group; }
int chunk_cols(int bits) { return bits == 4 ? 64 : 128; }
int chunk_bytes(int bits) { return bits == 3 ? 768 : 512; }

// Shapes the quantizer and the logical decode accept: any N, K > 0 with the
// group dividing K.
bool logical_ok(int N, int K, int mode, int bits, int group) {
  if (N <= 0 || K <= 0) return false;
  if (mode != MODE_SYM && mode != MODE_ASYM && mode != MODE_LUT) return false;
  if (bits != 4 && !((bits == 2 || bits == 3) && mode == MODE_LUT)) return false;
  if (group != -1 && (group <= 0 || K % group != 0)) return false;
  return true;
}

// Shapes the packed layout is defined for: whole row blocks and chunks, groups
// made of whole 16-column tiles.
bool shape_ok(int N, int K, int mode, int bits, int group) {
  if (!logical_ok(N, K, mode, bits, group)) return false;
  if (N % 16 != 0 || K % chunk_cols(bits) != 0) return false;
  if (group != -1 && group % 16 != 0) return false;
  return true;
}

// Byte offset and bit shift of code (n, k) in the packed code buffer (2- and
// 4-bit codes).
void code_place(int n, int k, int K, int mode, int bits, size_t* byte, int* shift) {
  int kc_cols = chunk_cols(bits);
  int rb = n / 16, r = n % 16;
  int g = r % 8, h = r / 8;
  int chunk = k / kc_cols, kk = k % kc_cols;
  int j = kk / 16, t = (kk % 16) / 4, c = kk % 4;
  int lane = 4 * g + t;
  int p = h + 2 * (c / 2);
  int hi = c % 2;
  size_t chunk_base = ((size_t)rb * (K / kc_cols) + chunk) * chunk_bytes(bits) +
                      (size_t)lane * (chunk_bytes(bits) / 32);
  if (bits == 4) {
    int nib = (mode == MODE_LUT) ? (2 * p + hi) : (p + 4 * hi);
    *byte = chunk_base + (size_t)j * 4 + nib / 2;
    *shift = 4 * (nib % 2);
  } else {
    int byte_in_word = 2 * (j % 2) + p / 2;
    int field = 2 * (p % 2) + hi;
    *byte = chunk_base + (size_t)(j / 2) * 4 + byte_in_word;
    *shift = 2 * field;
  }
}

// 3-bit codes: bit offset of code (n, k)'s lowest bit in the packed buffer.
// The lane's 24 bytes are one 192-bit little-endian string: tile j at bits
// [24 j, 24 j + 24), pair p at [24 j + 6 p, + 6), member c % 2 at + 3 (c % 2).
size_t code_bit3(int n, int k, int K) {
  int rb = n / 16, r = n % 16;
  int g = r % 8, h = r / 8;
  int chunk = k / 128, kk = k % 128;
  int j = kk / 16, t = (kk % 16) / 4, c = kk % 4;
  int lane = 4 * g + t;
  int p = h + 2 * (c / 2);
  size_t lane_base = ((size_t)rb * (K / 128) + chunk) * 768 + (size_t)lane * 24;
  return lane_base * 8 + 24 * j + 6 * p + 3 * (c % 2);
}

int get_code(const uint8_t* qw, int n, int k, int K, int mode, int bits) {
  if (bits == 3) {
    int q = 0;
    size_t b = code_bit3(n, k, K);
    for (int i = 0; i < 3; ++i) q |= ((qw[(b + i) / 8] >> ((b + i) % 8)) & 1) << i;
    return q;
  }
  size_t byte;
  int shift;
  code_place(n, k, K, mode, bits, &byte, &shift);
  return (qw[byte] >> shift) & ((1 << bits) - 1);
}

void put_code(uint8_t* qw, int n, int k, int K, int mode, int bits, int q) {
  if (bits == 3) {
    size_t b = code_bit3(n, k, K);
    for (int i = 0; i < 3; ++i) qw[(b + i) / 8] |= (uint8_t)(((q >> i) & 1) << ((b + i) % 8));
    return;
  }
  size_t byte;
  int shift;
  code_place(n, k, K, mode, bits, &byte, &shift);
  qw[byte] |= (uint8_t)((q & ((1 << bits) - 1)) << shift);
}

// Index of (row n, group gi) in the packed scale / zero buffers.
size_t scale_index(int n, int gi, int G) {
  int rb = n / 16, r = n % 16;
  return ((size_t)rb * G + gi) * 16 + 2 * (r % 8) + r / 8;
}

// ------------------------------------------------------------------- quantize

// Clamp-and-truncate for a float that rint() has already made integral.
int clamp_code(float v, int qmax) {
  if (!(v > 0.0f)) return 0;               // also catches -inf
  if (v > (float)qmax) return qmax;
  return (int)v;
}

}  // namespace

extern "C" {

size_t oracle_packed_bytes(int N, int K, int bits) { return (size_t)N * K * bits / 8; }

// Per group of `group` weights along K in each row n ([MZ], [FL], [GT]):
//   SYM  s = absmax / 7,            q = clamp(rint(w / s) + 8, 0, 15)
//   ASYM s = (max - min) / 15,      z = clamp(rint(-min / s), 0, 15),
//                                   q = clamp(rint(w / s) + z, 0, 15)
//   LUT  s = absmax,                q = argmin_i |w / s - T[i]|
// with s rounded to fp16 before use (R2) and the readings R1, R3-R7.
// Outputs are logical (unpacked): codes[N*K], scales[N*G], zeros[N*G] (ASYM).
int oracle_quantize(const float* W, int N, int K, int mode, int bits, int group,
                    const uint16_t* lut, uint8_t* codes, uint16_t* scales, uint16_t* zeros) {
  if (!W || !codes || !scales || !logical_ok(N, K, mode, bits, group)) return ERR_ARG;
  if (mode == MODE_ASYM && !zeros) return ERR_ARG;
  if (mode == MODE_LUT && !lut) return ERR_ARG;
  const int G = n_groups(K, group), L = group_len(K, group);
  const int qmax = (1 << bits) - 1;
  const int nlut = 1 << bits;
  for (int n = 0; n < N; ++n) {
    for (int gi = 0; gi < G; ++gi) {
      const float* w = W + (size_t)n * K + (size_t)gi * L;
      uint8_t* q = codes + (size_t)n * K + (size_t)gi * L;
      // (i) reduce the group in fp32 (max and min are exact)
      float amax = 0.0f, mn = w[0], mx = w[0];
      for (int i = 0; i < L; ++i) {
        float a = std::fabs(w[i]);
        if (a > amax) amax = a;
        if (w[i] < mn) mn = w[i];
        if (w[i] > mx) mx = w[i];
      }
      // (ii) the fp32 scale, (iii) rounded to fp16
      float s32;
      if (mode == MODE_SYM) s32 = amax / 7.0f;
      else if (mode == MODE_ASYM) s32 = (mx - mn) / 15.0f;
      else s32 = amax;
      uint16_t s16 = scale_bits(s32);
      float s = (float)half_value(s16);
      scales[(size_t)n * G + gi] = s16;
      if (mode == MODE_SYM) {
        for (int i = 0; i < L; ++i)
          q[i] = (uint8_t)(s == 0.0f ? 8 : clamp_code(std::rint(w[i] / s) + 8.0f, qmax));
      } else if (mode == MODE_ASYM) {
        int z = (s == 0.0f) ? 0 : clamp_code(std::rint(-mn / s), qmax);
        zeros[(size_t)n * G + gi] = half_bits((double)z);
        for (int i = 0; i < L; ++i)
          q[i] = (uint8_t)(s == 0.0f ? 0 : clamp_code(std::rint(w[i] / s) + (float)z, qmax));
      } else {
        for (int i = 0; i < L; ++i) {
          float u = (s == 0.0f) ? 0.0f : w[i] / s;
          int best = 0;
          float bd = std::fabs(u - (float)half_value(lut[0]));
          for (int e = 1; e < nlut; ++e) {
            float d = std::fabs(u - (float)half_value(lut[e]));
            if (d < bd) { bd = d; best = e; }
          }
          q[i] = (uint8_t)best;
        }
      }
    }
  }
  return OK;
}

// Logical codes/scales/zeros -> packed buffers (layout in the header comment).
int oracle_pack(const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros,
                int N, int K, int mode, int bits, int group,
                uint8_t* qweight, uint16_t* scales_p, uint16_t* zeros_p) {
  if (!codes || !scales || !qweight || !scales_p || !shape_ok(N, K, mode, bits, group))
    return ERR_ARG;
  if (mode == MODE_ASYM && (!zeros || !zeros_p)) return ERR_ARG;
  const int G = n_groups(K, group);
  std::memset(qweight, 0, oracle_packed_bytes(N, K, bits));
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) put_code(qweight, n, k, K, mode, bits, codes[(size_t)n * K + k]);
  for (int n = 0; n < N; ++n)
    for (int gi = 0; gi < G; ++gi) {
      scales_p[scale_index(n, gi, G)] = scales[(size_t)n * G + gi];
      if (mode == MODE_ASYM) zeros_p[scale_index(n, gi, G)] = zeros[(size_t)n * G + gi];
    }
  return OK;
}

// Packed buffers -> logical codes/scales/zeros (inverse of oracle_pack).
int oracle_unpack(const uint8_t* qweight, const uint16_t* scales_p, const uint16_t* zeros_p,
                  int N, int K, int mode, int bits, int group,
                  uint8_t* codes, uint16_t* scales, uint16_t* zeros) {
  if (!qweight || !codes || !shape_ok(N, K, mode, bits, group)) return ERR_ARG;
  const int G = n_groups(K, group);
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) codes[(size_t)n * K + k] = (uint8_t)get_code(qweight, n, k, K, mode, bits);
  for (int n = 0; n < N; ++n)
    for (int gi = 0; gi < G; ++gi) {
      if (scales && scales_p) scales[(size_t)n * G + gi] = scales_p[scale_index(n, gi, G)];
      if (mode == MODE_ASYM && zeros && zeros_p)
        zeros[(size_t)n * G + gi] = zeros_p[scale_index(n, gi, G)];
    }
  return OK;
}

// Decoded weight of one code ([MZ] symmetric / fp16 zero-point, [FL] table):
//   SYM (q - 8) s,  ASYM (q - z) s,  LUT T[q] s.  Exact in double (and in fp32).
static double decode(int q, double s, double z, const uint16_t* lut, int mode) {
  if (mode == MODE_SYM) return ((double)q - 8.0) * s;
  if (mode == MODE_ASYM) return ((double)q - z) * s;
  return half_value(lut[q]) * s;
}

// Logical codes -> W~[N*K] as exact doubles.
int oracle_dequant(const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros_or_lut,
                   int N, int K, int mode, int bits, int group, double* out) {
  if (!codes || !scales || !out || !logical_ok(N, K, mode, bits, group)) return ERR_ARG;
  if (mode != MODE_SYM && !zeros_or_lut) return ERR_ARG;
  const int G = n_groups(K, group), L = group_len(K, group);
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) {
      int gi = k / L;
      double s = half_value(scales[(size_t)n * G + gi]);
      double z = (mode == MODE_ASYM) ? half_value(zeros_or_lut[(size_t)n * G + gi]) : 0.0;
      out[(size_t)n * K + k] = decode(codes[(size_t)n * K + k], s, z, zeros_or_lut, mode);
    }
  return OK;
}

// Values -> fp16 (dtype 0) or bf16 (dtype 1) bits, round to nearest even.
int oracle_round(const double* in, size_t n, int dtype, uint16_t* out) {
  if (!in || !out || (dtype != DT_F16 && dtype != DT_BF16)) return ERR_ARG;
  for (size_t i = 0; i < n; ++i) out[i] = dtype == DT_F16 ? half_bits(in[i]) : bf16_bits(in[i]);
  return OK;
}

// fp16 / bf16 bits -> exact values.
int oracle_widen(const uint16_t* in, size_t n, int dtype, double* out) {
  if (!in || !out || (dtype != DT_F16 && dtype != DT_BF16)) return ERR_ARG;
  for (size_t i = 0; i < n; ++i) out[i] = dtype == DT_F16 ? half_value(in[i]) : bf16_value(in[i]);
  return OK;
}

// W~[n, k] for k = 0 .. K-1 of packed row n, into w.
static void dequant_row(int n, const uint8_t* qweight, const uint16_t* scales_p,
                        const uint16_t* zeros_or_lut, int K, int mode, int bits, int G, int L,
                        double* w) {
  for (int k = 0; k < K; ++k) {
    int q = get_code(qweight, n, k, K, mode, bits);
    int gi = k / L;
    double s = half_value(scales_p[scale_index(n, gi, G)]);
    double z = (mode == MODE_ASYM) ? half_value(zeros_or_lut[scale_index(n, gi, G)]) : 0.0;
    w[k] = decode(q, s, z, zeros_or_lut, mode);
  }
}

// y[m, n] = sum_k x[m, k] * W~[n, k] for output columns n in [n0, n1), read
// straight from the packed buffers ([GT] decode-then-multiply, [EX] the
// activations stay in their fp16/bf16 input precision).  The sum runs over k in
// ascending order in double; y is [M, n1 - n0] row-major doubles.
int oracle_qmm(const uint16_t* x, int xdtype, const uint8_t* qweight, const uint16_t* scales_p,
               const uint16_t* zeros_or_lut, int M, int N, int K, int mode, int bits, int group,
               int n0, int n1, double* y) {
  if (!x || !qweight || !scales_p || !y || M < 0 || n0 < 0 || n1 > N || n0 > n1) return ERR_ARG;
  if (!shape_ok(N, K, mode, bits, group)) return ERR_ARG;
  if (mode != MODE_SYM && !zeros_or_lut) return ERR_ARG;
  const int G = n_groups(K, group), L = group_len(K, group);
  double* xv = new double[(size_t)M * K];
  double* w = new double[(size_t)K];
  for (size_t i = 0; i < (size_t)M * K; ++i)
    xv[i] = xdtype == DT_BF16 ? bf16_value(x[i]) : half_value(x[i]);
  for (int n = n0; n < n1; ++n) {
    dequant_row(n, qweight, scales_p, zeros_or_lut, K, mode, bits, G, L, w);
    for (int m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += xv[(size_t)m * K + k] * w[k];
      y[(size_t)m * (n1 - n0) + (n - n0)] = acc;
    }
  }
  delete[] xv;
  delete[] w;
  return OK;
}

// Fused feed-forward gate ([GT] "How It Works": the FFN layers are fused into
// the quantized matmul).  The packed matrix has 2I rows whose 16-row blocks
// alternate gate and up: output i reads gate row 32 (i / 16) + i % 16 and the
// up row 16 below it.  y[m, i] = silu(g) * u with g, u the two rows' sums as in
// oracle_qmm and silu(v) = v / (1 + exp(-v)), all in double; outputs
// i in [i0, i1), y is [M, i1 - i0] row-major.
int oracle_qmm_gated(const uint16_t* x, int xdtype, const uint8_t* qweight,
                     const uint16_t* scales_p, const uint16_t* zeros_or_lut, int M, int I, int K,
                     int mode, int bits, int group, int i0, int i1, double* y) {
  if (!x || !qweight || !scales_p || !y || M < 0 || I <= 0 || I % 16 || i0 < 0 || i1 > I ||
      i0 > i1)
    return ERR_ARG;
  const int N = 2 * I;
  if (!shape_ok(N, K, mode, bits, group)) return ERR_ARG;
  if (mode != MODE_SYM && !zeros_or_lut) return ERR_ARG;
  const int G = n_groups(K, group), L = group_len(K, group);
  double* xv = new double[(size_t)M * K];
  double* wg = new double[(size_t)K];
  double* wu = new double[(size_t)K];
  for (size_t i = 0; i < (size_t)M * K; ++i)
    xv[i] = xdtype == DT_BF16 ? bf16_value(x[i]) : half_value(x[i]);
  for (int i = i0; i < i1; ++i) {
    const int ng = 32 * (i / 16) + i % 16, nu = ng + 16;
    dequant_row(ng, qweight, scales_p, zeros_or_lut, K, mode, bits, G, L, wg);
    dequant_row(nu, qweight, scales_p, zeros_or_lut, K, mode, bits, G, L, wu);
    for (int m = 0; m < M; ++m) {
      double g = 0.0, u = 0.0;
      for (int k = 0; k < K; ++k) {
        g += xv[(size_t)m * K + k] * wg[k];
        u += xv[(size_t)m * K + k] * wu[k];
      }
      y[(size_t)m * (i1 - i0) + (i - i0)] = g / (1.0 + std::exp(-g)) * u;
    }
  }
  delete[] xv;
  delete[] wg;
  delete[] wu;
  return OK;
}

// ------------------------------------------------ zero-point options ([MZ])
//
// [MZ] (mobicham's and efrantar's replies) raises two variants of the fp16
// zero-point: zero-points quantized to low-bit integers, and a zero-point group
// size different from the scale group size (scale per row with a zero-point per
// 8 weights).  Readings taken here:
//  R18 the zero-point group zg nests inside the scale group (zg divides the
//      scale group, group -1 counting as K); the reverse nesting is the one
//      the page reports as useless and is not defined.
//  R19 quantizer: s = (max - min) / 15 over the scale group (as R4), rounded to
//      fp16; per zero-point group z = clamp(rint(-min_zg / s), 0, 15) from that
//      group's own minimum; q = clamp(rint(w / s) + z, 0, 15).  With zg equal
//      to the scale group this is the plain asymmetric quantizer.
//  R20 zero storage: zbits 16 = fp16 value (as R4); zbits 4 = the same integer
//      in 4 bits, packed [N/16][Gz][8 bytes]: the block's rows in the order of
//      the scales (row r at slot 2 (r % 8) + r / 8), slot i at byte i / 2, the
//      low nibble for even i.
// Logical zeros are fp16 bit patterns [N, Gz] in every case.

static int zgroup_len(int K, int zgroup) { return zgroup == -1 ? K : zgroup; }

static bool zopts_ok(int K, int group, int zgroup, int zbits) {
  if (zbits != 16 && zbits != 4) return false;
  const int L = group_len(K, group);
  if (zgroup != -1 && (zgroup <= 0 || K % zgroup != 0)) return false;
  const int LZ = zgroup_len(K, zgroup);
  return LZ <= L && L % LZ == 0;
}

// Per row: scale per group of `group`, zero-point per group of `zgroup` (R18,
// R19).  codes[N*K], scales[N*G], zeros[N*Gz] (fp16 bits of integers).
int oracle_quantize_asym(const float* W, int N, int K, int group, int zgroup, uint8_t* codes,
                         uint16_t* scales, uint16_t* zeros) {
  if (!W || !codes || !scales || !zeros || !logical_ok(N, K, MODE_ASYM, 4, group)) return ERR_ARG;
  if (!zopts_ok(K, group, zgroup, 16)) return ERR_ARG;
  const int G = n_groups(K, group), L = group_len(K, group);
  const int LZ = zgroup_len(K, zgroup), GZ = K / LZ;
  for (int n = 0; n < N; ++n) {
    const float* row = W + (size_t)n * K;
    for (int gi = 0; gi < G; ++gi) {
      // the scale from the scale group's range
      float mn = row[gi * L], mx = row[gi * L];
      for (int i = gi * L; i < (gi + 1) * L; ++i) {
        if (row[i] < mn) mn = row[i];
        if (row[i] > mx) mx = row[i];
      }
      const uint16_t s16 = scale_bits((mx - mn) / 15.0f);
      const float s = (float)half_value(s16);
      scales[(size_t)n * G + gi] = s16;
      // a zero-point per zero group inside it, from that group's minimum
      for (int zi = gi * L / LZ; zi < (gi + 1) * L / LZ; ++zi) {
        float zmn = row[zi * LZ];
        for (int i = zi * LZ; i < (zi + 1) * LZ; ++i)
          if (row[i] < zmn) zmn = row[i];
        const int z = (s == 0.0f) ? 0 : clamp_code(std::rint(-zmn / s), 15);
        zeros[(size_t)n * GZ + zi] = half_bits((double)z);
        for (int i = zi * LZ; i < (zi + 1) * LZ; ++i)
          codes[(size_t)n * K + i] =
              (uint8_t)(s == 0.0f ? 0 : clamp_code(std::rint(row[i] / s) + (float)z, 15));
      }
    }
  }
  return OK;
}

// Packed zero buffer bytes (R20).
size_t oracle_zeros_bytes(int N, int K, int zgroup, int zbits) {
  const size_t GZ = (size_t)K / zgroup_len(K, zgroup);
  return zbits == 4 ? (size_t)N * GZ / 2 : (size_t)N * GZ * 2;
}

// The integer zero-point of row n, zero group zi, as a double, from the packed
// zero buffer (fp16 value, or the 4-bit integer of R20).
static double packed_zero(const uint8_t* zeros_p, int n, int zi, int GZ, int zbits) {
  const size_t idx = scale_index(n, zi, GZ);
  if (zbits == 16) {
    uint16_t h;
    std::memcpy(&h, zeros_p + 2 * idx, 2);
    return half_value(h);
  }
  return (double)((zeros_p[idx / 2] >> (4 * (idx % 2))) & 15);
}

// Logical (codes, scales, zeros) -> packed buffers; zeros written per R20.
// A zero that is not an integer in [0, 15] cannot be stored in 4 bits (ERR_ARG).
int oracle_pack_asym(const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros, int N,
                     int K, int group, int zgroup, int zbits, uint8_t* qweight,
                     uint16_t* scales_p, uint8_t* zeros_p) {
  if (!codes || !scales || !zeros || !qweight || !scales_p || !zeros_p) return ERR_ARG;
  if (!shape_ok(N, K, MODE_ASYM, 4, group) || !zopts_ok(K, group, zgroup, zbits)) return ERR_ARG;
  const int LZ = zgroup_len(K, zgroup), GZ = K / LZ;
  if (LZ % 8 != 0) return ERR_ARG;
  int st = oracle_pack(codes, scales, scales, N, K, MODE_SYM, 4, group, qweight, scales_p, nullptr);
  if (st != OK) return st;
  // SYM and ASYM place 4-bit codes identically; the zeros go separately
  std::memset(zeros_p, 0, oracle_zeros_bytes(N, K, zgroup, zbits));
  for (int n = 0; n < N; ++n)
    for (int zi = 0; zi < GZ; ++zi) {
      const uint16_t zb = zeros[(size_t)n * GZ + zi];
      const size_t idx = scale_index(n, zi, GZ);
      if (zbits == 16) {
        std::memcpy(zeros_p + 2 * idx, &zb, 2);
      } else {
        const double z = half_value(zb);
        if (!(z >= 0.0 && z <= 15.0 && z == std::floor(z))) return ERR_ARG;
        zeros_p[idx / 2] |= (uint8_t)((int)z << (4 * (idx % 2)));
      }
    }
  return OK;
}

// Logical codes -> exact W~[N*K] = (q - z[n, k / zg]) s[n, k / group].
int oracle_dequant_asym(const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros, int N,
                        int K, int group, int zgroup, double* out) {
  if (!codes || !scales || !zeros || !out || !logical_ok(N, K, MODE_ASYM, 4, group)) return ERR_ARG;
  if (!zopts_ok(K, group, zgroup, 16)) return ERR_ARG;
  const int G = n_groups(K, group), L = group_len(K, group);
  const int LZ = zgroup_len(K, zgroup), GZ = K / LZ;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) {
      const double s = half_value(scales[(size_t)n * G + k / L]);
      const double z = half_value(zeros[(size_t)n * GZ + k / LZ]);
      out[(size_t)n * K + k] = decode(codes[(size_t)n * K + k], s, z, nullptr, MODE_ASYM);
    }
  return OK;
}

// y[m, n] = sum_k x[m, k] (q - z) s read from the packed buffers, columns
// [n0, n1), double sums in ascending k (as oracle_qmm).
int oracle_qmm_asym(const uint16_t* x, int xdtype, const uint8_t* qweight,
                    const uint16_t* scales_p, const uint8_t* zeros_p, int M, int N, int K,
                    int group, int zgroup, int zbits, int n0, int n1, double* y) {
  if (!x || !qweight || !scales_p || !zeros_p || !y || M < 0 || n0 < 0 || n1 > N || n0 > n1)
    return ERR_ARG;
  if (!shape_ok(N, K, MODE_ASYM, 4, group) || !zopts_ok(K, group, zgroup, zbits)) return ERR_ARG;
  const int G = n_groups(K, group), L = group_len(K, group);
  const int LZ = zgroup_len(K, zgroup), GZ = K / LZ;
  double* xv = new double[(size_t)M * K];
  double* w = new double[(size_t)K];
  for (size_t i = 0; i < (size_t)M * K; ++i)
    xv[i] = xdtype == DT_BF16 ? bf16_value(x[i]) : half_value(x[i]);
  for (int n = n0; n < n1; ++n) {
    for (int k = 0; k < K; ++k) {
      const double s = half_value(scales_p[scale_index(n, k / L, G)]);
      const double z = packed_zero(zeros_p, n, k / LZ, GZ, zbits);
      w[k] = decode(get_code(qweight, n, k, K, MODE_ASYM, 4), s, z, nullptr, MODE_ASYM);
    }
    for (int m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += xv[(size_t)m * K + k] * w[k];
      y[(size_t)m * (n1 - n0) + (n - n0)] = acc;
    }
  }
  delete[] xv;
  delete[] w;
  return OK;
}

// ------------------------------------------------------------- act-order
//
// [GT] "Limitations & Caveats" names GPTQ's act-order option without
// describing it.  Reading R21 (GPTQ's convention): the quantizer visits the
// columns in a chosen order and forms its groups along that order, so the
// group of column k is g_idx[k] and a group is any set of columns; the weight
// keeps its column order.  W~[n, k] = decode(q[n, k], s[n, g_idx[k]],
// z[n, g_idx[k]]).  Packed layout: the codes of group i occupy packed columns
// [i L, (i + 1) L), members in ascending original column (so every group must
// hold exactly L columns); scales and zeros stay per group.

static bool gidx_ok(const int* g_idx, int K, int G) {
  for (int k = 0; k < K; ++k)
    if (g_idx[k] < 0 || g_idx[k] >= G) return false;
  return true;
}

// Packed column of every original column: pos[k] = g_idx[k] L + (number of
// earlier columns in the same group).  False if a group does not hold exactly
// L columns.
static bool packed_columns(const int* g_idx, int K, int G, int L, int* pos) {
  int* cnt = new int[G]();
  bool ok = true;
  for (int k = 0; k < K; ++k) pos[k] = g_idx[k] * L + cnt[g_idx[k]]++;
  for (int i = 0; i < G; ++i) ok = ok && cnt[i] == L;
  delete[] cnt;
  return ok;
}

// Quantize with groups given by g_idx (R21); otherwise oracle_quantize's
// arithmetic.  Reductions run over the group's members in ascending column.
int oracle_quantize_gidx(const float* W, int N, int K, int mode, int bits, int group,
                         const int* g_idx, const uint16_t* lut, uint8_t* codes, uint16_t* scales,
                         uint16_t* zeros) {
  if (!W || !g_idx || !codes || !scales || !logical_ok(N, K, mode, bits, group)) return ERR_ARG;
  if (mode == MODE_ASYM && !zeros) return ERR_ARG;
  if (mode == MODE_LUT && !lut) return ERR_ARG;
  const int G = n_groups(K, group);
  if (!gidx_ok(g_idx, K, G)) return ERR_ARG;
  // the members of every group, in ascending column: group gi's are
  // members[first[gi] .. first[gi + 1])
  int* first = new int[G + 1]();
  int* members = new int[K];
  for (int k = 0; k < K; ++k) ++first[g_idx[k] + 1];
  for (int gi = 0; gi < G; ++gi) first[gi + 1] += first[gi];
  {
    int* fill = new int[G];
    for (int gi = 0; gi < G; ++gi) fill[gi] = first[gi];
    for (int k = 0; k < K; ++k) members[fill[g_idx[k]]++] = k;
    delete[] fill;
  }
  // gather each group's members into a contiguous row, quantize that row with
  // the plain quantizer (one group per row), scatter the codes back
  float* gw = new float[K];
  uint8_t* gq = new uint8_t[K];
  int st = OK;
  for (int n = 0; n < N && st == OK; ++n)
    for (int gi = 0; gi < G && st == OK; ++gi) {
      const int* mem = members + first[gi];
      const int cnt = first[gi + 1] - first[gi];
      for (int i = 0; i < cnt; ++i) gw[i] = W[(size_t)n * K + mem[i]];
      if (cnt == 0) {   // an empty group: no weights, scale 0
        scales[(size_t)n * G + gi] = 0;
        if (mode == MODE_ASYM) zeros[(size_t)n * G + gi] = 0;
        continue;
      }
      uint16_t s16, z16 = 0;
      st = oracle_quantize(gw, 1, cnt, mode, bits, -1, lut, gq, &s16,
                           mode == MODE_ASYM ? &z16 : nullptr);
      scales[(size_t)n * G + gi] = s16;
      if (mode == MODE_ASYM) zeros[(size_t)n * G + gi] = z16;
      for (int i = 0; i < cnt; ++i) codes[(size_t)n * K + mem[i]] = gq[i];
    }
  delete[] gw;
  delete[] gq;
  delete[] members;
  delete[] first;
  return st;
}

// Logical codes -> exact W~ with per-column groups g_idx.
int oracle_dequant_gidx(const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros_or_lut,
                        int N, int K, int mode, int bits, int group, const int* g_idx,
                        double* out) {
  if (!codes || !scales || !g_idx || !out || !logical_ok(N, K, mode, bits, group)) return ERR_ARG;
  if (mode != MODE_SYM && !zeros_or_lut) return ERR_ARG;
  const int G = n_groups(K, group);
  if (!gidx_ok(g_idx, K, G)) return ERR_ARG;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) {
      const int gi = g_idx[k];
      const double s = half_value(scales[(size_t)n * G + gi]);
      const double z = (mode == MODE_ASYM) ? half_value(zeros_or_lut[(size_t)n * G + gi]) : 0.0;
      out[(size_t)n * K + k] = decode(codes[(size_t)n * K + k], s, z, zeros_or_lut, mode);
    }
  return OK;
}

// Logical codes (original column order) -> packed buffers with the act-order
// column placement of R21.
int oracle_pack_gidx(const uint8_t* codes, const uint16_t* scales, const uint16_t* zeros,
                     const int* g_idx, int N, int K, int mode, int bits, int group,
                     uint8_t* qweight, uint16_t* scales_p, uint16_t* zeros_p) {
  if (!codes || !g_idx || !shape_ok(N, K, mode, bits, group)) return ERR_ARG;
  const int G = n_groups(K, group), L = group_len(K, group);
  if (!gidx_ok(g_idx, K, G)) return ERR_ARG;
  int* pos = new int[K];
  uint8_t* moved = new uint8_t[(size_t)N * K];
  const bool ok = packed_columns(g_idx, K, G, L, pos);
  int st = ERR_ARG;
  if (ok) {
    for (int n = 0; n < N; ++n)
      for (int k = 0; k < K; ++k) moved[(size_t)n * K + pos[k]] = codes[(size_t)n * K + k];
    st = oracle_pack(moved, scales, zeros, N, K, mode, bits, group, qweight, scales_p, zeros_p);
  }
  delete[] pos;
  delete[] moved;
  return st;
}

// y[m, n] = sum_k x[m, k] W~[n, k] in original column order, the code of column
// k read at its packed column and its scale (zero) at group g_idx[k].
int oracle_qmm_gidx(const uint16_t* x, int xdtype, const uint8_t* qweight,
                    const uint16_t* scales_p, const uint16_t* zeros_or_lut, const int* g_idx,
                    int M, int N, int K, int mode, int bits, int group, int n0, int n1,
                    double* y) {
  if (!x || !qweight || !scales_p || !g_idx || !y || M < 0 || n0 < 0 || n1 > N || n0 > n1)
    return ERR_ARG;
  if (!shape_ok(N, K, mode, bits, group)) return ERR_ARG;
  if (mode != MODE_SYM && !zeros_or_lut) return ERR_ARG;
  const int G = n_groups(K, group), L = group_len(K, group);
  if (!gidx_ok(g_idx, K, G)) return ERR_ARG;
  int* pos = new int[K];
  if (!packed_columns(g_idx, K, G, L, pos)) {
    delete[] pos;
    return ERR_ARG;
  }
  double* xv = new double[(size_t)M * K];
  double* w = new double[(size_t)K];
  for (size_t i = 0; i < (size_t)M * K; ++i)
    xv[i] = xdtype == DT_BF16 ? bf16_value(x[i]) : half_value(x[i]);
  for (int n = n0; n < n1; ++n) {
    for (int k = 0; k < K; ++k) {
      const int gi = g_idx[k];
      const double s = half_value(scales_p[scale_index(n, gi, G)]);
      const double z = (mode == MODE_ASYM) ? half_value(zeros_or_lut[scale_index(n, gi, G)]) : 0.0;
      w[k] = decode(get_code(qweight, n, pos[k], K, mode, bits), s, z, zeros_or_lut, mode);
    }
    for (int m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += xv[(size_t)m * K + k] * w[k];
      y[(size_t)m * (n1 - n0) + (n - n0)] = acc;
    }
  }
  delete[] pos;
  delete[] xv;
  delete[] w;
  return OK;
}

}  // extern "C"
