// Plain CPU oracle for the rotated token-wise INT4 paged KV cache.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may include, link or
// call this file: only tests/, the smoke check and the benchmark's CPU
// baseline use it. It shares no source, header, table or helper with the CUDA
// library; the two meet only through seeded inputs generated elsewhere.
//
// What it follows:
//  * "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
//    Serving", Summary and Method: token-wise INT4 quantization of the KV cache
//    behind a block-diagonal Hadamard rotation, fused into paged KV-cache
//    layouts.
//  * "UltraQuant: 4-bit KV caching for long agents" (Traditional Chinese page),
//    section on how the method works: a Walsh-Hadamard rotation of the K/V
//    vectors spreads outlier channels before quantization.
//  * "IsoQuant: Hardware-Aligned SO(4) Isoclinic Rotations for LLM KV Cache
//    Compression", Abstract: each 4-D block is a quaternion v and is mapped to
//    qL * v * conj(qR).
// Where the pages leave a step open, the reading taken is the one written
// beside the step below; the same readings are listed in the design notes.
//
// Build: g++ -O2 -ffp-contract=off -fno-fast-math -frounding-math -fopenmp
// -shared -fPIC. No fused multiply-add is formed implicitly
// (-ffp-contract=off), so every float expression below is a sequence of
// IEEE-754 binary32 operations with round-to-nearest-even, exactly as
// written; the two operations that round upward switch the hardware rounding
// mode around themselves (-frounding-math keeps the compiler from moving or
// folding them).

#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// ---------------------------------------------------------------------------
// IEEE-754 binary16, written from the format definition (1 sign bit, 5
// exponent bits with bias 15, 10 fraction bits; subnormals have quantum 2^-24).
// ---------------------------------------------------------------------------

double orc_half_to_double(uint16_t h) {
  const int sign = h >> 15;
  const int e = (h >> 10) & 0x1f;
  const int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = std::ldexp((double)m, -24);
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = std::ldexp((double)(1024 + m), e - 25);
  }
  return sign ? -v : v;
}

// Rounding modes for binary32 -> binary16.
enum { ORC_RN = 0, ORC_RD = 1, ORC_RU = 2 };

// Converts a value to binary16 bits under one of three rounding modes: to
// nearest (ties to even), toward -inf, toward +inf. All double arithmetic
// below is exact: x is only scaled by powers of two, floored, subtracted from
// its own floor and compared.
uint16_t orc_double_to_half(double x, int mode) {
  if (std::isnan(x)) return 0x7e00;
  const bool neg = std::signbit(x);
  const uint16_t sign = neg ? 0x8000 : 0;
  if (std::isinf(x)) return sign | 0x7c00;
  double a = std::fabs(x);
  if (a == 0.0) return sign;
  // Direction in which the MAGNITUDE moves: toward -inf on a negative number
  // makes the magnitude larger.
  enum { NEAREST, DOWN, UP } dir = NEAREST;
  if (mode == ORC_RD) dir = neg ? UP : DOWN;
  if (mode == ORC_RU) dir = neg ? DOWN : UP;

  int e2;
  std::frexp(a, &e2);              // a = f * 2^e2 with f in [0.5, 1)
  int E = e2 - 1;                  // a in [2^E, 2^(E+1))
  if (E < -14) E = -14;            // subnormals share the quantum of binade -14
  const double q = std::ldexp(1.0, E - 10);  // spacing of binary16 values here
  const double n = a / q;          // exact
  const double fl = std::floor(n);
  double r;
  if (dir == DOWN) {
    r = fl;
  } else if (dir == UP) {
    r = (n == fl) ? fl : fl + 1.0;
  } else {
    const double frac = n - fl;
    if (frac > 0.5) r = fl + 1.0;
    else if (frac < 0.5) r = fl;
    else r = (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
  }
  const double v = r * q;
  if (v > 65504.0) {               // past the largest finite binary16
    if (dir == DOWN) return sign | 0x7bff;
    return sign | 0x7c00;          // nearest: only reached when a >= 65520
  }
  // r in [0, 2048]; r == 2048 carries into the next binade naturally.
  const int bits = ((E + 15) << 10) + ((int)r - 1024);
  return (uint16_t)(sign | (uint16_t)bits);
}

uint16_t orc_float_to_half(float x, int mode) { return orc_double_to_half((double)x, mode); }

float orc_half_to_float(uint16_t h) { return (float)orc_half_to_double(h); }

// ---------------------------------------------------------------------------
// Block-diagonal Walsh-Hadamard rotation (SAW-INT4 Summary/Method; UltraQuant
// method section). Blocks are contiguous runs of b channels; within a block
// y = (1/sqrt(b)) * H_b * x with H_b the Sylvester Hadamard matrix,
// H_b[i][j] = (-1)^popcount(i & j). It is computed by the fast transform:
// stages h = 1, 2, 4, ..., b/2 in ascending order; at each stage every pair
// (i, i+h) with (i & h) == 0 becomes (x_i + x_{i+h}, x_i - x_{i+h}), each one
// binary32 operation; then every element is multiplied by c_b, the binary32
// value nearest 1/sqrt(b).
// ---------------------------------------------------------------------------

float orc_hadamard_scale(int b) {
  // 1/sqrt(b) for b a power of two: 2^(-k) when b = 4^k, sqrt(2) * 2^(-k)
  // when b = 2 * 4^(k-1) (i.e. b = 2^(2k-1)). sqrt(2.0) is correctly rounded
  // in double and lies far from a binary32 rounding boundary, so this is the
  // binary32 value nearest 1/sqrt(b).
  int lg = 0;
  while ((1 << lg) < b) ++lg;
  if (lg % 2 == 0) return std::ldexp(1.0f, -lg / 2);
  return (float)std::ldexp(std::sqrt(2.0), -(lg + 1) / 2);
}

void orc_fwht_unscaled(float* x, int b) {
  for (int h = 1; h < b; h <<= 1) {
    for (int i = 0; i < b; ++i) {
      if ((i & h) == 0) {
        const float a = x[i];
        const float c = x[i + h];
        x[i] = a + c;
        x[i + h] = a - c;
      }
    }
  }
}

void orc_rotate_hadamard_f32(float* x, int d, int b) {
  const float cb = orc_hadamard_scale(b);
  for (int t = 0; t < d; t += b) {
    orc_fwht_unscaled(x + t, b);
    for (int i = 0; i < b; ++i) x[t + i] = x[t + i] * cb;
  }
}

// ---------------------------------------------------------------------------
// Quaternion block rotation (IsoQuant Abstract: T(v) = qL v conj(qR), full
// SO(4) variant). Channels 4j..4j+3 of a head are the quaternion
// (w, x, y, z). The table holds, per block j, qL[j] then qR[j], each as
// (w, x, y, z) in binary32. Each component of a Hamilton product a*b is the
// textbook formula evaluated as fma(t3, fma(t2, fma(t1, t0))) with t0 a plain
// product and the terms in this order:
//   w: ( a.w b.w, -a.x b.x, -a.y b.y, -a.z b.z)
//   x: ( a.w b.x,  a.x b.w,  a.y b.z, -a.z b.y)
//   y: ( a.w b.y, -a.x b.z,  a.y b.w,  a.z b.x)
//   z: ( a.w b.z,  a.x b.y, -a.y b.x,  a.z b.w)
// ---------------------------------------------------------------------------

void orc_hamilton_f32(const float* a, const float* b, float* out) {
  const float aw = a[0], ax = a[1], ay = a[2], az = a[3];
  const float bw = b[0], bx = b[1], by = b[2], bz = b[3];
  float w = aw * bw;
  w = std::fma(-ax, bx, w);
  w = std::fma(-ay, by, w);
  w = std::fma(-az, bz, w);
  float x = aw * bx;
  x = std::fma(ax, bw, x);
  x = std::fma(ay, bz, x);
  x = std::fma(-az, by, x);
  float y = aw * by;
  y = std::fma(-ax, bz, y);
  y = std::fma(ay, bw, y);
  y = std::fma(az, bx, y);
  float z = aw * bz;
  z = std::fma(ax, by, z);
  z = std::fma(-ay, bx, z);
  z = std::fma(az, bw, z);
  out[0] = w; out[1] = x; out[2] = y; out[3] = z;
}

void orc_rotate_quat_f32(float* x, int d, const float* quat) {
  for (int j = 0; j < d / 4; ++j) {
    const float* qL = quat + j * 8;
    const float* qR = quat + j * 8 + 4;
    const float qRc[4] = {qR[0], -qR[1], -qR[2], -qR[3]};
    float t[4];
    orc_hamilton_f32(qL, x + 4 * j, t);
    orc_hamilton_f32(t, qRc, x + 4 * j);
  }
}

// IsoQuant-Fast (IsoQuant Abstract: "keeps only one isoclinic factor"):
// T(v) = qL v, one Hamilton product per 4-channel block (16 multiply-adds),
// qL[j] from the same table layout as the full map (qR[j] unused).
void orc_rotate_quat_fast_f32(float* x, int d, const float* quat) {
  for (int j = 0; j < d / 4; ++j) {
    float t[4];
    orc_hamilton_f32(quat + j * 8, x + 4 * j, t);
    for (int i = 0; i < 4; ++i) x[4 * j + i] = t[i];
  }
}

// Randomised-sign Hadamard (a reading of the randomised Hadamard transform
// the pages' rotation sources build on): every channel is first multiplied
// by its sign s_i in {+1, -1} (exact), then the block Hadamard rotation
// above; the signs are a caller-supplied binary32 table [d] shared by every
// row, like the quaternion table.
void orc_rotate_signed_hadamard_f32(float* x, int d, int b, const float* signs) {
  for (int i = 0; i < d; ++i) x[i] = x[i] * signs[i];
  orc_rotate_hadamard_f32(x, d, b);
}

// IsoQuant-Full folded into one 4x4 matrix per block (IsoQuant page,
// Abstract: the map v -> qL v conj(qR) is linear in v, so it is a 4x4 real
// matrix M = Rm(conj qR) Lm(qL), Lm(a) the matrix of v -> a v and Rm(b) the
// matrix of t -> t b). Reading: M is built in binary32 from the table's
// quaternions, each entry M[r][c] = sum over k of Rm[r][k] Lm[k][c] as
// fma(t3, fma(t2, fma(t1, t0))) with t0 the plain product and k ascending;
// the map is then y_r = fma(M[r][3] v3, fma(M[r][2] v2, fma(M[r][1] v1,
// M[r][0] v0))): 16 multiply-adds per block instead of 32, with a rounding
// that differs from the two Hamilton products'.
//   Lm(a) rows: ( a.w, -a.x, -a.y, -a.z), ( a.x,  a.w, -a.z,  a.y),
//               ( a.y,  a.z,  a.w, -a.x), ( a.z, -a.y,  a.x,  a.w)
//   Rm(b) rows: ( b.w, -b.x, -b.y, -b.z), ( b.x,  b.w,  b.z, -b.y),
//               ( b.y, -b.z,  b.w,  b.x), ( b.z,  b.y, -b.x,  b.w)
void orc_quat_matrix_f32(const float* q8, float* M) {
  const float* a = q8;
  const float b[4] = {q8[4], -q8[5], -q8[6], -q8[7]};  // conj(qR)
  const float Lm[4][4] = {{a[0], -a[1], -a[2], -a[3]},
                          {a[1], a[0], -a[3], a[2]},
                          {a[2], a[3], a[0], -a[1]},
                          {a[3], -a[2], a[1], a[0]}};
  const float Rm[4][4] = {{b[0], -b[1], -b[2], -b[3]},
                          {b[1], b[0], b[3], -b[2]},
                          {b[2], -b[3], b[0], b[1]},
                          {b[3], b[2], -b[1], b[0]}};
  for (int r = 0; r < 4; ++r)
    for (int c = 0; c < 4; ++c) {
      float m = Rm[r][0] * Lm[0][c];
      for (int k = 1; k < 4; ++k) m = std::fma(Rm[r][k], Lm[k][c], m);
      M[4 * r + c] = m;
    }
}

void orc_rotate_quat_mat_f32(float* x, int d, const float* quat) {
  for (int j = 0; j < d / 4; ++j) {
    float M[16];
    orc_quat_matrix_f32(quat + j * 8, M);
    const float* v = x + 4 * j;
    float y[4];
    for (int r = 0; r < 4; ++r) {
      float t = M[4 * r] * v[0];
      for (int c = 1; c < 4; ++c) t = std::fma(M[4 * r + c], v[c], t);
      y[r] = t;
    }
    for (int r = 0; r < 4; ++r) x[4 * j + r] = y[r];
  }
}

// Rotation kinds (same numbering as the library's public enum, restated).
enum { ORC_ROT_NONE = 0, ORC_ROT_HADAMARD = 1, ORC_ROT_QUAT = 2, ORC_ROT_QUAT_FAST = 3,
       ORC_ROT_HADAMARD_SIGNED = 4, ORC_ROT_QUAT_MAT = 5 };

void orc_rotate_f32(float* x, int d, int kind, int b, const float* quat) {
  if (kind == ORC_ROT_HADAMARD) orc_rotate_hadamard_f32(x, d, b);
  else if (kind == ORC_ROT_QUAT) orc_rotate_quat_f32(x, d, quat);
  else if (kind == ORC_ROT_QUAT_FAST) orc_rotate_quat_fast_f32(x, d, quat);
  else if (kind == ORC_ROT_HADAMARD_SIGNED) orc_rotate_signed_hadamard_f32(x, d, b, quat);
  else if (kind == ORC_ROT_QUAT_MAT) orc_rotate_quat_mat_f32(x, d, quat);
}

// ---------------------------------------------------------------------------
// Token-wise asymmetric INT4 quantizer (SAW-INT4 page, Summary: one scale and
// one zero-point per (token, head) row, 16 levels).
// Readings: the minimum is stored rounded toward -inf; the scale is
// (max - m16)/15 with the binary32 subtraction, the binary32 division and the
// final binary16 conversion all rounded toward +inf, so every x lies in
// [m16, m16 + 15 s16] exactly; the code is the nearest integer (ties to even)
// to the exact product RN(x - m16) * RN(1/s16), clamped to [0, 15] (one
// rounding of the product; the clamp never acts given that range, and is
// kept as the definition); a row
// with max == m16 has s16 = 0 and all codes 0; -0 is normalised to +0 in both
// the minimum and the maximum so the stored bits do not depend on reduction
// order.
// ---------------------------------------------------------------------------

// Binary32 subtraction and division rounded toward +inf (IEEE-754 directed
// rounding, done by the FPU in that mode).
float orc_sub_ru(float a, float b) {
  const int old = std::fegetround();
  std::fesetround(FE_UPWARD);
  volatile float va = a, vb = b;
  volatile float r = va - vb;
  std::fesetround(old);
  return r;
}

float orc_div_ru(float a, float b) {
  const int old = std::fegetround();
  std::fesetround(FE_UPWARD);
  volatile float va = a, vb = b;
  volatile float r = va / vb;
  std::fesetround(old);
  return r;
}

// Nearest integer, ties to even, of a double (exact: floor and the
// fraction of a double below 2^52 are exact).
static double rint_half_even(double t) {
  const double fl = std::floor(t);
  const double fr = t - fl;
  if (fr > 0.5) return fl + 1.0;
  if (fr < 0.5) return fl;
  return (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

// Codes of `bits` bits (2, 3 or 4) are packed into a little-endian bit
// stream: code i of the row occupies bits [i*bits, (i+1)*bits) of the row's
// d*bits/8 bytes (for 4 bits: the even channel in the low nibble).
static void pack_codes(const int* c, int d, int bits, uint8_t* out) {
  const int nbytes = d * bits / 8;
  for (int k = 0; k < nbytes; ++k) out[k] = 0;
  for (int i = 0; i < d; ++i) {
    const int bit = i * bits;
    const unsigned v = (unsigned)c[i] << (bit % 8);
    out[bit / 8] |= (uint8_t)(v & 0xFF);
    if ((bit % 8) + bits > 8) out[bit / 8 + 1] |= (uint8_t)(v >> 8);
  }
}

void orc_unpack_codes(const uint8_t* codes, int d, int bits, int* c) {
  for (int i = 0; i < d; ++i) {
    const int bit = i * bits;
    unsigned v = codes[bit / 8];
    if ((bit % 8) + bits > 8) v |= (unsigned)codes[bit / 8 + 1] << 8;
    c[i] = (int)((v >> (bit % 8)) & ((1u << bits) - 1));
  }
}

// The row statistics shared by the integer and table formats: the minimum
// rounded down to binary16 (m16) and the scale (max - m16)/Q rounded up at
// every step (s16); Q = 2^bits - 1, or 15 for the 16-level table.
static void row_stats(const float* y, int d, int Q, uint16_t* s16_out, uint16_t* m16_out) {
  float mn = y[0], mx = y[0];
  for (int i = 1; i < d; ++i) {
    if (y[i] < mn) mn = y[i];
    if (y[i] > mx) mx = y[i];
  }
  mn = mn + 0.0f;
  mx = mx + 0.0f;
  const uint16_t m16 = orc_float_to_half(mn, ORC_RD);
  const float m = orc_half_to_float(m16);
  const float diff = orc_sub_ru(mx, m);
  const float s32 = orc_div_ru(diff, (float)Q);
  *s16_out = orc_float_to_half(s32, ORC_RU);
  *m16_out = m16;
}

// Token-wise asymmetric integer codes of `bits` bits (2, 3 or 4; the 2- and
// 3-bit forms follow IsoQuant's bit widths {2, 3, 4}, page "IsoQuant:
// Hardware-Aligned SO(4) Isoclinic Rotations for LLM KV Cache Compression",
// Abstract): as the INT4 rule above with Q = 2^bits - 1 levels above zero.
void orc_quantize_row_bits(const float* y, int d, int bits, uint8_t* codes,
                           uint16_t* s16_out, uint16_t* m16_out) {
  const int Q = (1 << bits) - 1;
  row_stats(y, d, Q, s16_out, m16_out);
  const float m = orc_half_to_float(*m16_out);
  const float s = orc_half_to_float(*s16_out);
  std::vector<int> c(d, 0);
  if (s != 0.0f) {
    const float inv = 1.0f / s;
    for (int i = 0; i < d; ++i) {
      const float t0 = y[i] - m;
      const double prod = (double)t0 * (double)inv;  // exact: 24 x 24 bits
      double r = rint_half_even(prod);
      if (r < 0.0) r = 0.0;
      if (r > Q) r = Q;
      c[i] = (int)r;
    }
  }
  pack_codes(c.data(), d, bits, codes);
}

void orc_quantize_row(const float* y, int d, uint8_t* codes,
                      uint16_t* s16_out, uint16_t* m16_out) {
  orc_quantize_row_bits(y, d, 4, codes, s16_out, m16_out);
}

// Calibrated 16-entry table in place of the uniform INT4 levels (UltraQuant
// page, method section: the 16 centroids refitted on activations instead of
// the theoretical Lloyd-Max ones). Reading: the table replaces the levels
// 0..15 of u = (x - m16)/s16 with the row statistics of INT4 unchanged;
// `levels` holds 16 non-decreasing binary16-exact values in [0, 15] on the
// 1/16 grid; the code is the index of the level nearest to the exact
// u* = RN(x - m16) * RN(1/s16), a tie going to the lower index (the count of
// midpoints (t_k + t_k+1)/2 that u* exceeds); x^ = t[c] s16 + m16.
void orc_quantize_row_lut(const float* y, int d, const float* levels, uint8_t* codes,
                          uint16_t* s16_out, uint16_t* m16_out) {
  row_stats(y, d, 15, s16_out, m16_out);
  const float m = orc_half_to_float(*m16_out);
  const float s = orc_half_to_float(*s16_out);
  std::vector<int> c(d, 0);
  if (s != 0.0f) {
    const float inv = 1.0f / s;
    for (int i = 0; i < d; ++i) {
      const float t0 = y[i] - m;
      const double u = (double)t0 * (double)inv;  // exact
      int code = 0;
      for (int k = 0; k < 15; ++k)
        if (u > 0.5 * ((double)levels[k] + (double)levels[k + 1])) code = k + 1;
      c[i] = code;
    }
  }
  pack_codes(c.data(), d, 4, codes);
}

// Unpacks one row of codes (d/2 bytes) into d integers.
void orc_unpack_row(const uint8_t* codes, int d, int* c) {
  for (int k = 0; k < d / 2; ++k) {
    c[2 * k] = codes[k] & 0xf;
    c[2 * k + 1] = codes[k] >> 4;
  }
}

// ---------------------------------------------------------------------------
// Microscaled FP4 cache, a second format of the same paged cache (UltraQuant
// page, method section: FP4 KV tensors with UE8M0 group scales and FP8
// queries, taken by the matrix cores' scaled multiply-accumulate).
// Readings: the Open Compute Project microscaling (MX) formats, which both
// scaled matrix-core paths implement: blocks of 32 consecutive channels of a
// rotated (token, head) row share one power-of-two scale 2^X stored as the
// UE8M0 byte X + 127, with X = floor(log2(amax)) - emax, amax the block's
// largest |x| and emax the element format's largest exponent (2 for E2M1, 8
// for E4M3); X is clamped to [-127, 127] and an all-zero block takes
// X = -127. Each element x / 2^X (exact: a power-of-two scaling) is rounded
// to the nearest value of the element format, ties to even, saturating at
// the format's largest finite value (6 for E2M1, 448 for E4M3), keeping the
// sign of x (a negative value that rounds to zero becomes -0). E2M1 codes:
// bit 3 sign, bits 2-0 index into {0, 0.5, 1, 1.5, 2, 3, 4, 6}; packed two
// per byte, the even channel in the low nibble. E4M3: bit 7 sign, 4 exponent
// bits (bias 7), 3 mantissa bits, subnormals m 2^-9.
// ---------------------------------------------------------------------------

int orc_mx_exponent(float amax, int emax) {
  if (!(amax > 0.0f)) return -127;
  int e2;
  std::frexp((double)amax, &e2);  // amax = f 2^e2 with f in [0.5, 1)
  int x = e2 - 1 - emax;          // floor(log2 amax) - emax
  if (x < -127) x = -127;
  if (x > 127) x = 127;
  return x;
}

// Nearest value, ties to even, of a >= 0 on a grid with `mbits` mantissa
// bits and smallest normal exponent emin, saturating at vmax.
static double round_minifloat(double a, int mbits, int emin, double vmax) {
  if (a >= vmax) return vmax;
  if (a == 0.0) return 0.0;
  int e2;
  std::frexp(a, &e2);
  int E = e2 - 1;
  if (E < emin) E = emin;
  const double quantum = std::ldexp(1.0, E - mbits);
  const double r = rint_half_even(a / quantum) * quantum;
  return r > vmax ? vmax : r;
}

static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

int orc_e2m1_encode(double t) {
  const double r = round_minifloat(std::fabs(t), 1, 0, 6.0);
  int m = 0;
  while (kE2M1[m] != r) ++m;
  return (std::signbit(t) ? 8 : 0) | m;
}

double orc_e2m1_value(int code) {
  const double v = kE2M1[code & 7];
  return (code & 8) ? -v : v;
}

int orc_e4m3_encode(double t) {
  const double r = round_minifloat(std::fabs(t), 3, -6, 448.0);
  int bits = 0;
  if (r != 0.0) {
    int e2;
    std::frexp(r, &e2);
    const int E = e2 - 1;
    if (E < -6) {
      bits = (int)std::ldexp(r, 9);  // subnormal: m 2^-9
    } else {
      bits = ((E + 7) << 3) | (int)((std::ldexp(r, -E) - 1.0) * 8.0);
    }
  }
  return (std::signbit(t) ? 0x80 : 0) | bits;
}

double orc_e4m3_value(int code) {
  const int e = (code >> 3) & 15, m = code & 7;
  const double v = e == 0 ? std::ldexp((double)m, -9) : std::ldexp(1.0 + m / 8.0, e - 7);
  return (code & 0x80) ? -v : v;
}

// One rotated binary32 row -> d/2 bytes of E2M1 codes and d/32 UE8M0 bytes.
void orc_mxfp4_quantize_row(const float* y, int d, uint8_t* codes, uint8_t* scales) {
  std::vector<int> c(d);
  for (int g = 0; g < d / 32; ++g) {
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(y[32 * g + i]));
    const int X = orc_mx_exponent(amax, 2);
    scales[g] = (uint8_t)(X + 127);
    for (int i = 0; i < 32; ++i) c[32 * g + i] = orc_e2m1_encode(std::ldexp((double)y[32 * g + i], -X));
  }
  for (int k = 0; k < d / 2; ++k) codes[k] = (uint8_t)(c[2 * k] | (c[2 * k + 1] << 4));
}

// The query side: a rotated binary32 row -> its MX E4M3 values (exact, in
// double), blocks of 32 channels with their own shared exponent.
void orc_mxfp8_row_values(const float* y, int d, double* out) {
  for (int g = 0; g < d / 32; ++g) {
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(y[32 * g + i]));
    const int X = orc_mx_exponent(amax, 8);
    for (int i = 0; i < 32; ++i) {
      const int code = orc_e4m3_encode(std::ldexp((double)y[32 * g + i], -X));
      out[32 * g + i] = std::ldexp(orc_e4m3_value(code), X);
    }
  }
}

// Storage formats (same numbering as the library's public enum, restated).
enum { ORC_FMT_INT4 = 0, ORC_FMT_MXFP4 = 1, ORC_FMT_INT2 = 2, ORC_FMT_INT3 = 3,
       ORC_FMT_LUT4 = 4 };

// Bits per code and bytes of one row's codes and parameters: (s16, m16) for
// the integer and table formats, d/32 scale bytes for MX FP4 (a params row of
// the pool is 4 bytes at d <= 128).
static inline int code_bits(int fmt) {
  return fmt == ORC_FMT_INT2 ? 2 : (fmt == ORC_FMT_INT3 ? 3 : 4);
}
static inline int code_row_bytes(int fmt, int d) { return d * code_bits(fmt) / 8; }
static inline int params_row_bytes(int fmt, int d) {
  return fmt == ORC_FMT_MXFP4 ? (d / 32 < 4 ? 4 : d / 32) : 4;
}

// Dequantized row (double) of one stored row in any format (`levels`: the
// table of the LUT4 format).
static void deq_row(int fmt, const float* levels, const uint8_t* codes_row,
                    const uint8_t* params_row, int d, double* x) {
  if (fmt == ORC_FMT_MXFP4) {
    for (int k = 0; k < d / 2; ++k)
      for (int n = 0; n < 2; ++n) {
        const int i = 2 * k + n;
        const int code = n ? codes_row[k] >> 4 : codes_row[k] & 0xf;
        x[i] = std::ldexp(orc_e2m1_value(code), (int)params_row[i / 32] - 127);
      }
  } else {
    uint16_t s16, m16;
    std::memcpy(&s16, params_row, 2);
    std::memcpy(&m16, params_row + 2, 2);
    const double s = orc_half_to_double(s16), m = orc_half_to_double(m16);
    std::vector<int> c(d);
    orc_unpack_codes(codes_row, d, code_bits(fmt), c.data());
    for (int i = 0; i < d; ++i)
      x[i] = (fmt == ORC_FMT_LUT4 ? (double)levels[c[i]] : (double)c[i]) * s + m;
  }
}

// ---------------------------------------------------------------------------
// Rotary position embedding, optionally applied to each key row and to the
// query in front of the block rotation (the step before the method's path in
// a decode step; the pages do not describe it, so this is a reading).
// Adjacent channel pairs (2i, 2i+1) turn by the angle of the pair at the
// token's position, whose cosine and sine the caller supplies as one row of a
// binary32 table: cs[2i] = cos, cs[2i+1] = sin. Binary32, every product and
// the difference / sum rounded on its own (no fused multiply-add):
//   x'_{2i} = RN(RN(x_{2i} c) - RN(x_{2i+1} s)),
//   x'_{2i+1} = RN(RN(x_{2i} s) + RN(x_{2i+1} c)).
void orc_rope_row_f32(float* x, int d, const float* cs) {
  for (int i = 0; i < d / 2; ++i) {
    const float a = x[2 * i], b = x[2 * i + 1], c = cs[2 * i], sn = cs[2 * i + 1];
    const float ac = a * c, bs = b * sn, as = a * sn, bc = b * c;
    x[2 * i] = ac - bs;
    x[2 * i + 1] = as + bc;
  }
}

// The same turn in double precision (the query side of attention).
static void rope_row_f64(double* x, int d, const float* cs) {
  for (int i = 0; i < d / 2; ++i) {
    const double a = x[2 * i], b = x[2 * i + 1], c = cs[2 * i], sn = cs[2 * i + 1];
    x[2 * i] = a * c - b * sn;
    x[2 * i + 1] = a * sn + b * c;
  }
}

// Paged placement (SAW-INT4 Summary: the quantizer writes straight into paged
// KV-cache layouts). Reading: pools are [page][kv_head][slot][d/2] bytes of
// codes and [page][kv_head][slot] pairs (s16, m16) of binary16 (scale first);
// K and V have separate pools; page = block_table[seq][pos / P], slot =
// pos % P.
// Error flags (OR-ed into *err): 1 = block-table entry outside [0, NP),
// 2 = position outside the table (pos < 0 or pos / P >= bt_stride),
// 4 = sequence index outside [0, num_seqs), 8 = sequence length invalid.
// ---------------------------------------------------------------------------

enum { ORC_ERR_PAGE = 1, ORC_ERR_POS = 2, ORC_ERR_SEQ = 4, ORC_ERR_LEN = 8 };

// With a RoPE table (rope != NULL, rows [rope_max_pos][d]), every key row is
// turned by the row of its position before the rotation; a token whose
// position has no row in the table is skipped with flag 2.
void orc_quantize_append(int d, int H, int P, int NP, int rot_kind, int rot_block,
                         const float* quat, int T, const uint16_t* k, const uint16_t* v,
                         int64_t tok_stride, const int32_t* token_seq,
                         const int32_t* token_pos, int num_seqs,
                         const int32_t* block_table, int bt_stride, uint8_t* k_codes,
                         void* k_params, uint8_t* v_codes, void* v_params,
                         const float* rope, int rope_max_pos, int fmt, const float* levels,
                         int32_t* err) {
  // Tokens are independent (each writes only its own slot), so they are
  // spread over threads; the arithmetic of every row is unchanged.
  int32_t flags = 0;
#pragma omp parallel for schedule(static) reduction(| : flags)
  for (int t = 0; t < T; ++t) {
    std::vector<float> row(d);
    const int seq = token_seq[t];
    if (seq < 0) continue;
    if (seq >= num_seqs) { flags |= ORC_ERR_SEQ; continue; }
    const int pos = token_pos[t];
    if (pos < 0 || pos / P >= bt_stride) { flags |= ORC_ERR_POS; continue; }
    if (rope != nullptr && pos >= rope_max_pos) { flags |= ORC_ERR_POS; continue; }
    const int page = block_table[(int64_t)seq * bt_stride + pos / P];
    if (page < 0 || page >= NP) { flags |= ORC_ERR_PAGE; continue; }
    const int slot = pos % P;
    for (int kv = 0; kv < 2; ++kv) {
      const uint16_t* src = kv == 0 ? k : v;
      uint8_t* codes = kv == 0 ? k_codes : v_codes;
      uint8_t* params = static_cast<uint8_t*>(kv == 0 ? k_params : v_params);
      for (int h = 0; h < H; ++h) {
        const uint16_t* x = src + (int64_t)t * tok_stride + (int64_t)h * d;
        for (int i = 0; i < d; ++i) row[i] = orc_half_to_float(x[i]);
        if (kv == 0 && rope != nullptr) orc_rope_row_f32(row.data(), d, rope + (int64_t)pos * d);
        orc_rotate_f32(row.data(), d, rot_kind, rot_block, quat);
        const int64_t r = ((int64_t)page * H + h) * P + slot;
        uint8_t* prow = params + r * params_row_bytes(fmt, d);
        uint8_t* crow = codes + r * code_row_bytes(fmt, d);
        if (fmt == ORC_FMT_MXFP4) {
          orc_mxfp4_quantize_row(row.data(), d, crow, prow);
        } else {
          uint16_t s16, m16;
          if (fmt == ORC_FMT_LUT4)
            orc_quantize_row_lut(row.data(), d, levels, crow, &s16, &m16);
          else
            orc_quantize_row_bits(row.data(), d, code_bits(fmt), crow, &s16, &m16);
          std::memcpy(prow, &s16, 2);
          std::memcpy(prow + 2, &m16, 2);
        }
      }
    }
  }
  *err |= flags;
}

// ---------------------------------------------------------------------------
// Inverse rotation in double precision, used after attention and by the
// dense export. Hadamard: R is symmetric and R R = I for the exact
// orthonormal R, so R^-1 = R (computed with the exact 1/sqrt(b)).
// Quaternion: T(v) = qL v conj(qR) is inverted by
// v = qL^-1 w conj(qR)^-1 = (conj(qL)/|qL|^2) w (qR/|qR|^2).
// ---------------------------------------------------------------------------

static void hamilton_f64(const double* a, const double* b, double* o) {
  o[0] = a[0] * b[0] - a[1] * b[1] - a[2] * b[2] - a[3] * b[3];
  o[1] = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];
  o[2] = a[0] * b[2] - a[1] * b[3] + a[2] * b[0] + a[3] * b[1];
  o[3] = a[0] * b[3] + a[1] * b[2] - a[2] * b[1] + a[3] * b[0];
}

void orc_rotate_f64(double* x, int d, int kind, int b, const float* quat) {
  if (kind == ORC_ROT_QUAT_MAT) {
    // the binary32 matrix M the cache was written with, applied exactly
    for (int j = 0; j < d / 4; ++j) {
      float M[16];
      orc_quat_matrix_f32(quat + j * 8, M);
      double y[4];
      for (int r = 0; r < 4; ++r) {
        y[r] = 0.0;
        for (int c = 0; c < 4; ++c) y[r] += (double)M[4 * r + c] * x[4 * j + c];
      }
      for (int r = 0; r < 4; ++r) x[4 * j + r] = y[r];
    }
  } else if (kind == ORC_ROT_HADAMARD_SIGNED) {
    for (int i = 0; i < d; ++i) x[i] *= (double)quat[i];
    orc_rotate_f64(x, d, ORC_ROT_HADAMARD, b, quat);
  } else if (kind == ORC_ROT_QUAT_FAST) {
    for (int j = 0; j < d / 4; ++j) {
      const double qL[4] = {quat[8 * j], quat[8 * j + 1], quat[8 * j + 2], quat[8 * j + 3]};
      double t[4];
      hamilton_f64(qL, x + 4 * j, t);
      for (int i = 0; i < 4; ++i) x[4 * j + i] = t[i];
    }
  } else if (kind == ORC_ROT_HADAMARD) {
    const double cb = 1.0 / std::sqrt((double)b);
    std::vector<double> y(b);
    for (int t = 0; t < d; t += b) {
      for (int i = 0; i < b; ++i) {
        double acc = 0.0;
        for (int j = 0; j < b; ++j)
          acc += (__builtin_popcount(i & j) & 1) ? -x[t + j] : x[t + j];
        y[i] = acc * cb;
      }
      for (int i = 0; i < b; ++i) x[t + i] = y[i];
    }
  } else if (kind == ORC_ROT_QUAT) {
    for (int j = 0; j < d / 4; ++j) {
      const double qL[4] = {quat[8 * j], quat[8 * j + 1], quat[8 * j + 2], quat[8 * j + 3]};
      const double qR[4] = {quat[8 * j + 4], -(double)quat[8 * j + 5], -(double)quat[8 * j + 6],
                            -(double)quat[8 * j + 7]};
      double t[4];
      hamilton_f64(qL, x + 4 * j, t);
      hamilton_f64(t, qR, x + 4 * j);
    }
  }
}

void orc_unrotate_f64(double* x, int d, int kind, int b, const float* quat) {
  if (kind == ORC_ROT_QUAT_MAT) {
    // reading: the inverse of the (orthogonal up to binary32 rounding)
    // matrix is taken as its transpose
    for (int j = 0; j < d / 4; ++j) {
      float M[16];
      orc_quat_matrix_f32(quat + j * 8, M);
      double y[4];
      for (int c = 0; c < 4; ++c) {
        y[c] = 0.0;
        for (int r = 0; r < 4; ++r) y[c] += (double)M[4 * r + c] * x[4 * j + r];
      }
      for (int c = 0; c < 4; ++c) x[4 * j + c] = y[c];
    }
  } else if (kind == ORC_ROT_HADAMARD) {
    orc_rotate_f64(x, d, kind, b, quat);  // R^-1 = R
  } else if (kind == ORC_ROT_HADAMARD_SIGNED) {
    // R = H S with S the sign diagonal: R^-1 = S^-1 H^-1 = S H
    orc_rotate_f64(x, d, ORC_ROT_HADAMARD, b, quat);
    for (int i = 0; i < d; ++i) x[i] *= (double)quat[i];
  } else if (kind == ORC_ROT_QUAT_FAST) {
    for (int j = 0; j < d / 4; ++j) {
      const double L[4] = {quat[8 * j], quat[8 * j + 1], quat[8 * j + 2], quat[8 * j + 3]};
      const double nL = L[0] * L[0] + L[1] * L[1] + L[2] * L[2] + L[3] * L[3];
      const double Linv[4] = {L[0] / nL, -L[1] / nL, -L[2] / nL, -L[3] / nL};
      double t[4];
      hamilton_f64(Linv, x + 4 * j, t);
      for (int i = 0; i < 4; ++i) x[4 * j + i] = t[i];
    }
  } else if (kind == ORC_ROT_QUAT) {
    for (int j = 0; j < d / 4; ++j) {
      const double L[4] = {quat[8 * j], quat[8 * j + 1], quat[8 * j + 2], quat[8 * j + 3]};
      const double R[4] = {quat[8 * j + 4], quat[8 * j + 5], quat[8 * j + 6], quat[8 * j + 7]};
      const double nL = L[0] * L[0] + L[1] * L[1] + L[2] * L[2] + L[3] * L[3];
      const double nR = R[0] * R[0] + R[1] * R[1] + R[2] * R[2] + R[3] * R[3];
      const double Linv[4] = {L[0] / nL, -L[1] / nL, -L[2] / nL, -L[3] / nL};
      const double Rinv[4] = {R[0] / nR, R[1] / nR, R[2] / nR, R[3] / nR};  // (conj qR)^-1
      double t[4];
      hamilton_f64(Linv, x + 4 * j, t);
      hamilton_f64(t, Rinv, x + 4 * j);
    }
  }
}

// Dequantized value of one stored element: c * s16 + m16 (exact in double).
static inline double deq(int c, uint16_t s16, uint16_t m16) {
  return (double)c * orc_half_to_double(s16) + orc_half_to_double(m16);
}

// Dense export of cached tokens: out[s][j][h][:] for j < seq_lens[s]
// (rows at or past seq_lens[s] are left untouched). Values are computed in
// double, optionally un-rotated, then rounded once to binary32 (out_fp32) or
// to binary16 with round-to-nearest-even.
void orc_dequantize_pages(int d, int H, int P, int NP, int rot_kind, int rot_block,
                          const float* quat, int S, const int32_t* seq_lens,
                          int max_seq_len, const int32_t* block_table, int bt_stride,
                          const uint8_t* codes, const void* params, int unrotate,
                          int out_fp32, void* out, int fmt, const float* levels,
                          int32_t* err) {
  int32_t flags = 0;
  std::vector<double> x(d);
  const uint8_t* pb = static_cast<const uint8_t*>(params);
  for (int s = 0; s < S; ++s) {
    int L = seq_lens[s];
    if (L < 0 || L > max_seq_len || (L + P - 1) / P > bt_stride) { flags |= ORC_ERR_LEN; continue; }
    for (int j = 0; j < L; ++j) {
      const int page = block_table[(int64_t)s * bt_stride + j / P];
      if (page < 0 || page >= NP) { flags |= ORC_ERR_PAGE; continue; }
      for (int h = 0; h < H; ++h) {
        const int64_t r = ((int64_t)page * H + h) * P + j % P;
        deq_row(fmt, levels, codes + r * code_row_bytes(fmt, d), pb + r * params_row_bytes(fmt, d),
                d, x.data());
        if (unrotate) orc_unrotate_f64(x.data(), d, rot_kind, rot_block, quat);
        const int64_t o = (((int64_t)s * max_seq_len + j) * H + h) * d;
        if (out_fp32) {
          float* of = (float*)out;
          for (int i = 0; i < d; ++i) of[o + i] = (float)x[i];
        } else {
          uint16_t* oh = (uint16_t*)out;
          for (int i = 0; i < d; ++i) oh[o + i] = orc_double_to_half(x[i], ORC_RN);
        }
      }
    }
  }
  *err |= flags;
}


// ---------------------------------------------------------------------------
// Decode attention over the INT4 pages (SAW-INT4 Key takeaway: the rotated
// INT4 cache must serve fused attention). Everything is in double precision:
// for sequence s and query head g (KV head h = g / (Hq/H), contiguous
// grouping),
//   qhat = R q_g, z_j = sm_scale * (qhat . khat_j) for every cached j < L_s,
//   p = softmax(z) (maximum subtracted first), otilde = sum_j p_j vhat_j,
//   o = R^-1 otilde,
// where khat_j, vhat_j are the dequantized rotated rows. Because R is
// orthogonal, qhat . (R k) = q . k: the query is rotated by the same R that
// the keys were quantized behind. A page whose block-table entry is outside
// [0, NP) contributes no token and sets flag 1; an invalid length sets flag 8
// and gives a zero output; a sequence with no token gives a zero output.
// ---------------------------------------------------------------------------

// With a RoPE table the query is turned by the row of its own position,
// seq_len - 1 (the last cached token is the one being decoded), before the
// rotation; a length whose last position has no row sets flag 8 and gives a
// zero output.
void orc_paged_decode_attn(int d, int H, int P, int NP, int rot_kind, int rot_block,
                           const float* quat, int S, int Hq, const uint16_t* q,
                           const int32_t* seq_lens, int max_seq_len,
                           const int32_t* block_table, int bt_stride, double sm_scale,
                           const uint8_t* k_codes, const void* k_params,
                           const uint8_t* v_codes, const void* v_params,
                           const float* rope, int rope_max_pos, int fmt, const float* levels,
                           double* out,
                           int32_t* err) {
  const uint8_t* kpb = static_cast<const uint8_t*>(k_params);
  const uint8_t* vpb = static_cast<const uint8_t*>(v_params);
  const int PB = params_row_bytes(fmt, d), CB = code_row_bytes(fmt, d);
  const int G = Hq / H;
  int32_t flags = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : flags)
  for (int sg = 0; sg < S * Hq; ++sg) {
    const int s = sg / Hq, g = sg % Hq, h = g / G;
    double* o = out + (int64_t)sg * d;
    for (int i = 0; i < d; ++i) o[i] = 0.0;
    const int L = seq_lens[s];
    if (L < 0 || L > max_seq_len || (L + P - 1) / P > bt_stride) { flags |= ORC_ERR_LEN; continue; }
    if (rope != nullptr && L > rope_max_pos) { flags |= ORC_ERR_LEN; continue; }
    std::vector<double> qh(d), kh(d), vh(d), acc(d, 0.0);
    if (fmt == ORC_FMT_MXFP4) {
      // the query as the MX FP4 path takes it: turned and rotated in binary32
      // (the quantize path's arithmetic), then MX E4M3 values
      std::vector<float> qf(d);
      for (int i = 0; i < d; ++i) qf[i] = orc_half_to_float(q[(int64_t)sg * d + i]);
      if (rope != nullptr && L >= 1) orc_rope_row_f32(qf.data(), d, rope + (int64_t)(L - 1) * d);
      orc_rotate_f32(qf.data(), d, rot_kind, rot_block, quat);
      orc_mxfp8_row_values(qf.data(), d, qh.data());
    } else {
      for (int i = 0; i < d; ++i) qh[i] = orc_half_to_double(q[(int64_t)sg * d + i]);
      if (rope != nullptr && L >= 1) rope_row_f64(qh.data(), d, rope + (int64_t)(L - 1) * d);
      orc_rotate_f64(qh.data(), d, rot_kind, rot_block, quat);
    }
    std::vector<double> z;
    std::vector<int64_t> rows;
    z.reserve(L);
    rows.reserve(L);
    for (int j = 0; j < L; ++j) {
      const int page = block_table[(int64_t)s * bt_stride + j / P];
      if (page < 0 || page >= NP) { flags |= ORC_ERR_PAGE; continue; }
      const int64_t r = ((int64_t)page * H + h) * P + j % P;
      deq_row(fmt, levels, k_codes + r * CB, kpb + r * PB, d, kh.data());
      double dot = 0.0;
      for (int i = 0; i < d; ++i) dot += qh[i] * kh[i];
      z.push_back(sm_scale * dot);
      rows.push_back(r);
    }
    if (z.empty()) continue;
    const double zmax = *std::max_element(z.begin(), z.end());
    double denom = 0.0;
    for (size_t j = 0; j < z.size(); ++j) { z[j] = std::exp(z[j] - zmax); denom += z[j]; }
    for (size_t j = 0; j < z.size(); ++j) {
      const int64_t r = rows[j];
      deq_row(fmt, levels, v_codes + r * CB, vpb + r * PB, d, vh.data());
      const double p = z[j] / denom;
      for (int i = 0; i < d; ++i) acc[i] += p * vh[i];
    }
    orc_unrotate_f64(acc.data(), d, rot_kind, rot_block, quat);
    for (int i = 0; i < d; ++i) o[i] = acc[i];
  }
  *err |= flags;
}

// The same attention over an unquantized binary16 paged cache
// ([page][kv_head][slot][d]), without rotation: the full-precision baseline
// the INT4 cache is compared against.
void orc_paged_decode_attn_fp16(int d, int H, int P, int NP, int S, int Hq, const uint16_t* q,
                                const int32_t* seq_lens, int max_seq_len,
                                const int32_t* block_table, int bt_stride, double sm_scale,
                                const uint16_t* k16, const uint16_t* v16, double* out,
                                int32_t* err) {
  const int G = Hq / H;
  int32_t flags = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : flags)
  for (int sg = 0; sg < S * Hq; ++sg) {
    const int s = sg / Hq, g = sg % Hq, h = g / G;
    double* o = out + (int64_t)sg * d;
    for (int i = 0; i < d; ++i) o[i] = 0.0;
    const int L = seq_lens[s];
    if (L < 0 || L > max_seq_len || (L + P - 1) / P > bt_stride) { flags |= ORC_ERR_LEN; continue; }
    std::vector<double> qh(d), acc(d, 0.0);
    for (int i = 0; i < d; ++i) qh[i] = orc_half_to_double(q[(int64_t)sg * d + i]);
    std::vector<double> z;
    std::vector<int64_t> rows;
    for (int j = 0; j < L; ++j) {
      const int page = block_table[(int64_t)s * bt_stride + j / P];
      if (page < 0 || page >= NP) { flags |= ORC_ERR_PAGE; continue; }
      const int64_t r = ((int64_t)page * H + h) * P + j % P;
      double dot = 0.0;
      for (int i = 0; i < d; ++i) dot += qh[i] * orc_half_to_double(k16[r * d + i]);
      z.push_back(sm_scale * dot);
      rows.push_back(r);
    }
    if (z.empty()) continue;
    const double zmax = *std::max_element(z.begin(), z.end());
    double denom = 0.0;
    for (size_t j = 0; j < z.size(); ++j) { z[j] = std::exp(z[j] - zmax); denom += z[j]; }
    for (size_t j = 0; j < z.size(); ++j) {
      const double p = z[j] / denom;
      for (int i = 0; i < d; ++i) acc[i] += p * orc_half_to_double(v16[rows[j] * d + i]);
    }
    for (int i = 0; i < d; ++i) o[i] = acc[i];
  }
  *err |= flags;
}

// Number of threads the parallel loops above use (1 without OpenMP).
int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

// ---------------------------------------------------------------------------
// Row-array helpers for the Python wrapper (loops over the functions above).
// ---------------------------------------------------------------------------

void orc_float_to_half_array(const float* x, int64_t n, int mode, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_float_to_half(x[i], mode);
}

void orc_double_to_half_array(const double* x, int64_t n, int mode, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_double_to_half(x[i], mode);
}

void orc_half_to_double_array(const uint16_t* h, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_half_to_double(h[i]);
}

void orc_rotate_rows_f32(float* x, int64_t rows, int d, int kind, int b, const float* quat) {
  for (int64_t r = 0; r < rows; ++r) orc_rotate_f32(x + r * d, d, kind, b, quat);
}

void orc_rotate_rows_f64(double* x, int64_t rows, int d, int kind, int b, const float* quat) {
  for (int64_t r = 0; r < rows; ++r) orc_rotate_f64(x + r * d, d, kind, b, quat);
}

void orc_unrotate_rows_f64(double* x, int64_t rows, int d, int kind, int b, const float* quat) {
  for (int64_t r = 0; r < rows; ++r) orc_unrotate_f64(x + r * d, d, kind, b, quat);
}

void orc_quantize_rows_fmt(const float* y, int64_t rows, int d, int fmt, const float* levels,
                           uint8_t* codes, uint16_t* s16, uint16_t* m16) {
  const int cb = code_row_bytes(fmt, d);
  for (int64_t r = 0; r < rows; ++r) {
    if (fmt == ORC_FMT_LUT4)
      orc_quantize_row_lut(y + r * d, d, levels, codes + r * cb, s16 + r, m16 + r);
    else
      orc_quantize_row_bits(y + r * d, d, code_bits(fmt), codes + r * cb, s16 + r, m16 + r);
  }
}

void orc_unpack_codes_rows(const uint8_t* codes, int64_t rows, int d, int bits, int32_t* c) {
  std::vector<int> t(d);
  for (int64_t r = 0; r < rows; ++r) {
    orc_unpack_codes(codes + r * (d * bits / 8), d, bits, t.data());
    for (int i = 0; i < d; ++i) c[r * d + i] = t[i];
  }
}

void orc_quantize_rows(const float* y, int64_t rows, int d, uint8_t* codes, uint16_t* s16,
                       uint16_t* m16) {
  for (int64_t r = 0; r < rows; ++r)
    orc_quantize_row(y + r * d, d, codes + r * (d / 2), s16 + r, m16 + r);
}

}  // extern "C"
