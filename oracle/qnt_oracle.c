/*
 * qnt_oracle.c -- plain CPU oracle for round-to-nearest (RTN) group-wise 4-bit
 * weight quantization and the fused-dequant GEMV/GEMM that consumes it.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant generator with the CUDA library it checks.
 *
 * Sources (the pages give prose, no formulas; the arithmetic below is the
 * plainest reading, and each such reading is tagged [R#] below):
 *  - "Is (Selective) Round-To-Nearest Quantization All You Need?" (Kogan,
 *    arXiv 2505.15909), English abstract: data-free RTN weight quantization and
 *    selective higher precision (INT8 / FP16) for chosen modules.
 *  - "Revisiting Block-based Quantisation" (Zhang et al., arXiv 2310.05079),
 *    English abstract: a scaling factor shared across a block of packed numbers
 *    (here: a group of g consecutive weights along the input dimension K).
 *  - "The Power of Negative Zero: RaZeR" (Chen et al., arXiv 2501.04052),
 *    English abstract and method section: the FP4 negative-zero encoding is
 *    remapped to a predefined special value.
 *  - "AFPQ: Asymmetric Floating Point Quantization" (Zhang et al., arXiv
 *    2311.01792), English abstract: separate scales for positive and negative
 *    values.
 *
 * Precision: every scalar quantization step is one IEEE binary32 operation with
 * round-to-nearest-even (compiled with -ffp-contract=off, SSE math); fp16 and
 * bf16 roundings are written out here from the IEEE-754 definitions; every
 * GEMV/GEMM accumulation is binary64.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* format ids (same numbering as the public C ABI, restated here) */
enum { OF_INT4 = 1, OF_FP4 = 2, OF_AFPQ = 3, OF_RAZER = 4, OF_INT8 = 5, OF_FP16 = 6 };
/* status codes the oracle reports (same meaning as the library's) */
enum { OS_OK = 0, OS_NONFINITE = 6, OS_RANGE = 7 };

/* ------------------------------------------------------------------------- */
/* IEEE binary16 / bfloat16 conversions, written from the format definitions  */
/* ------------------------------------------------------------------------- */

/* Exact value of an fp16 bit pattern. */
double o_h2d(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 31) v = m ? NAN : INFINITY;
  else if (e == 0) v = ldexp((double)m, -24);           /* subnormal: m * 2^-24 */
  else v = ldexp((double)(1024 + m), e - 25);           /* (1 + m/1024) 2^(e-15) */
  return s ? -v : v;
}

/* Round a finite-or-not binary32 value to the nearest fp16, ties to even.
 * The value is decomposed as an exact binary64 number, divided by the fp16
 * spacing of its binade (a power of two, so exact), rounded with rint() in the
 * default nearest-even mode, then re-encoded. */
uint16_t o_f2h(float f) {
  double a = fabs((double)f);
  uint16_t sign = signbit(f) ? 0x8000 : 0;
  if (isnan(f)) return 0x7E00;                /* canonical quiet NaN */
  if (a >= 65520.0) return sign | 0x7C00;     /* beyond 65504 + half spacing: inf */
  int e;                                      /* binade exponent: 2^e <= a < 2^(e+1) */
  double spacing;
  if (a < ldexp(1.0, -14)) spacing = ldexp(1.0, -24);            /* subnormal spacing */
  else { frexp(a, &e); e -= 1; spacing = ldexp(1.0, e - 10); }
  double n = rint(a / spacing);               /* integer multiple of the spacing */
  double r = n * spacing;                     /* rounded magnitude, exactly representable */
  if (r == 0.0) return sign;
  if (r < ldexp(1.0, -14)) return sign | (uint16_t)(r / ldexp(1.0, -24));
  frexp(r, &e); e -= 1;                       /* re-derive binade: rounding may carry up */
  uint16_t m = (uint16_t)(r / ldexp(1.0, e - 10) - 1024.0);
  return sign | (uint16_t)((e + 15) << 10) | m;
}

/* Exact value of a bfloat16 bit pattern (upper half of a binary32). */
double o_bf2d(uint16_t b) {
  uint32_t u = (uint32_t)b << 16; float f; memcpy(&f, &u, 4); return (double)f;
}

/* Round binary32 to bfloat16, ties to even (bfloat16 = binary32 with 7 stored
 * mantissa bits; rounding happens at bit 16 of the binary32 pattern). */
uint16_t o_f2bf(float f) {
  if (isnan(f)) return 0x7FC0;
  double a = fabs((double)f);
  uint16_t sign = signbit(f) ? 0x8000 : 0;
  if (a == 0.0) return sign;
  if (isinf(f)) return sign | 0x7F80;
  int e;
  double spacing;
  if (a < ldexp(1.0, -126)) spacing = ldexp(1.0, -133);          /* subnormal spacing */
  else { frexp(a, &e); e -= 1; spacing = ldexp(1.0, e - 7); }
  double r = rint(a / spacing) * spacing;
  if (r >= ldexp(1.0, 128)) return sign | 0x7F80;
  float rf = (float)r;                        /* exact: r has <= 8 significant bits */
  uint32_t u; memcpy(&u, &rf, 4);
  return sign | (uint16_t)((u >> 16) & 0x7FFF);
}

/* ------------------------------------------------------------------------- */
/* The FP4 E2M1 data type (RaZeR page: sign-magnitude FP with +0 and -0)       */
/* ------------------------------------------------------------------------- */

/* Magnitudes of codes 0..7, bit 3 is the sign: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double o_e2m1(int code) {
  double m = E2M1_MAG[code & 7];
  return (code & 8) ? -m : m;
}

/* RaZeR special values by 2-bit selector [R8]: +5, -5, +8, -8. */
static const double RAZER_SV[4] = {5.0, -5.0, 8.0, -8.0};
double o_razer_sv(int sel) { return RAZER_SV[sel & 3]; }

/* Nearest E2M1 magnitude index for a value v >= 0, ties to the code whose
 * mantissa bit is 0 (IEEE round-to-nearest-even) [R5]; saturates at 6. */
static int e2m1_nearest_mag(double v) {
  int best = 0;
  double bd = fabs(v - E2M1_MAG[0]);
  for (int i = 1; i < 8; i++) {
    double d = fabs(v - E2M1_MAG[i]);
    if (d < bd || (d == bd && (i & 1) == 0)) { best = i; bd = d; }
  }
  return best;
}

/* fp16 scale from a binary32 quotient; a zero scale becomes 1.0 [R2].
 * Overflow to infinity is reported through *st. */
static uint16_t scale_h(float q, int* st) {
  uint16_t h = o_f2h(q);
  if ((h & 0x7FFF) == 0) h = 0x3C00;
  if ((h & 0x7C00) == 0x7C00 && *st == OS_OK) *st = OS_RANGE;
  return h;
}

static float fclampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* Round-to-nearest-even of a binary32 value (rintf in the default mode). */
static float rne(float v) { return rintf(v); }

static int all_finite(const float* w, int n) {
  for (int i = 0; i < n; i++) if (!isfinite(w[i])) return 0;
  return 1;
}

/* ------------------------------------------------------------------------- */
/* Group quantizers.  Each returns logical codes (one per element) and the     */
/* group's metadata.                                                           */
/* ------------------------------------------------------------------------- */

/* INT4 asymmetric, scale + 4-bit zero [R1-R4]:
 *   s = fp16((max - min) / 15), z = clamp(rint(-min / s), 0, 15),
 *   q = clamp(rint(w / s) + z, 0, 15), dequant (q - z) * s. */
static void q_int4(const float* w, int g, uint8_t* codes, uint16_t* s_out, uint8_t* z_out, int* st) {
  float mn = w[0], mx = w[0];
  for (int i = 1; i < g; i++) { if (w[i] < mn) mn = w[i]; if (w[i] > mx) mx = w[i]; }
  float range = mx - mn;
  uint16_t sh = scale_h(range / 15.0f, st);
  float S = (float)o_h2d(sh);
  float zf = fclampf(rne(-mn / S), 0.0f, 15.0f);
  int z = (int)zf;
  for (int i = 0; i < g; i++) {
    float r = fclampf(rne(w[i] / S), -64.0f, 64.0f);   /* wider clamp first: exact */
    int q = (int)r + z;
    codes[i] = (uint8_t)(q < 0 ? 0 : (q > 15 ? 15 : q));
  }
  *s_out = sh; *z_out = (uint8_t)z;
}

/* FP4 E2M1 code of w under scale S: sign bit | nearest magnitude; magnitude 0
 * always gets code 0, so 0b1000 is never produced [R6]. */
static uint8_t fp4_code(float w, float S) {
  float v = w / S;
  int m = e2m1_nearest_mag(fabs((double)v));
  if (m == 0) return 0;
  return (uint8_t)((v < 0.0f ? 8 : 0) | m);
}

/* Symmetric FP4: s = fp16(absmax / 6). */
static void q_fp4(const float* w, int g, uint8_t* codes, uint16_t* s_out, int* st) {
  float am = 0.0f;
  for (int i = 0; i < g; i++) { float a = fabsf(w[i]); if (a > am) am = a; }
  uint16_t sh = scale_h(am / 6.0f, st);
  float S = (float)o_h2d(sh);
  for (int i = 0; i < g; i++) codes[i] = fp4_code(w[i], S);
  *s_out = sh;
}

/* AFPQ: s+ = fp16(max(max,0)/6), s- = fp16(max(-min,0)/6) [R7]; positive
 * weights use s+, negative weights use s- with the sign bit set. */
static void q_afpq(const float* w, int g, uint8_t* codes, uint16_t* sp_out, uint16_t* sn_out, int* st) {
  float mn = w[0], mx = w[0];
  for (int i = 1; i < g; i++) { if (w[i] < mn) mn = w[i]; if (w[i] > mx) mx = w[i]; }
  float pos = mx > 0.0f ? mx : 0.0f;
  float neg = mn < 0.0f ? -mn : 0.0f;
  uint16_t sp = scale_h(pos / 6.0f, st), sn = scale_h(neg / 6.0f, st);
  float Sp = (float)o_h2d(sp), Sn = (float)o_h2d(sn);
  for (int i = 0; i < g; i++) {
    if (w[i] > 0.0f) codes[i] = fp4_code(w[i], Sp);
    else if (w[i] < 0.0f) codes[i] = fp4_code(w[i], Sn);
    else codes[i] = 0;
  }
  *sp_out = sp; *sn_out = sn;
}

/* RaZeR code of w for candidate special value sv under scale S: the grid is
 * the 15 regular FP4 values (codes 0..7, 9..15) plus sv at code 0b1000.
 * Nearest in v = w/S; a regular/regular tie goes to the even-mantissa code
 * [R5]; a tie between sv and a regular value goes to the regular value [R10]. */
static uint8_t razer_code(float w, float S, double sv) {
  double v = (double)(w / S);
  int best = -1; double bd = 0.0; int best_is_sv = 0;
  for (int c = 0; c < 16; c++) {
    double val = (c == 8) ? sv : o_e2m1(c);
    double d = fabs(v - val);
    int better;
    if (best < 0) better = 1;
    else if (d < bd) better = 1;
    else if (d > bd) better = 0;
    else if (c == 8) better = 0;                          /* sv loses ties */
    else if (best_is_sv) better = 1;
    else if (o_e2m1(c) == o_e2m1(best)) better = 0;       /* +0 (code 0) vs nothing else */
    else better = ((c & 1) == 0) && ((best & 1) != 0);   /* even mantissa wins */
    if (better) { best = c; bd = d; best_is_sv = (c == 8); }
  }
  return (uint8_t)best;
}

/* Sum of e[0..n) (n a power of two) in a balanced binary tree in index order:
 * (0+1), (2+3), ... then adjacent partial sums [R11]. */
static double tree_sum(double* t, int n) {
  for (int width = 1; width < n; width *= 2)
    for (int i = 0; i + width < n; i += 2 * width) t[i] = t[i] + t[i + width];
  return t[0];
}

/* RaZeR: for each selector c with special value sv_c, the scale is
 * fp16(absmax / max(6, |sv_c|)) [R9]; the codes are the RTN codes above; the
 * error is the binary64 sum of squared errors in tree order; the smallest
 * error wins, ties to the smallest selector [R12]. */
static void q_razer(const float* w, int g, uint8_t* codes, uint16_t* s_out, uint8_t* sel_out, int* st) {
  float am = 0.0f;
  for (int i = 0; i < g; i++) { float a = fabsf(w[i]); if (a > am) am = a; }
  double* t = (double*)malloc(sizeof(double) * (size_t)g);
  uint8_t* cc = (uint8_t*)malloc((size_t)g);
  double best_e = 0.0; int best = -1;
  uint16_t best_s = 0;
  for (int c = 0; c < 4; c++) {
    double sv = RAZER_SV[c];
    float denom = fabs(sv) > 6.0 ? (float)fabs(sv) : 6.0f;
    int st_c = OS_OK;
    uint16_t sh = scale_h(am / denom, &st_c);
    float S = (float)o_h2d(sh);
    for (int i = 0; i < g; i++) {
      cc[i] = razer_code(w[i], S, sv);
      double val = (cc[i] == 8) ? sv : o_e2m1(cc[i]);
      double dq = val * (double)S;             /* exact: <= 14 significant bits */
      double e = (double)w[i] - dq;
      t[i] = e * e;
    }
    double E = tree_sum(t, g);
    if (best < 0 || E < best_e) {
      best = c; best_e = E; best_s = sh;
      memcpy(codes, cc, (size_t)g);
      if (st_c != OS_OK && *st == OS_OK) *st = st_c;
    }
  }
  free(t); free(cc);
  *s_out = best_s; *sel_out = (uint8_t)best;
}

/* INT8 symmetric per output channel [R13]: s = fp16(absmax_row / 127),
 * q = clamp(rint(w / s), -127, 127). */
static void q_int8_row(const float* w, int k, int8_t* codes, uint16_t* s_out, int* st) {
  float am = 0.0f;
  for (int i = 0; i < k; i++) { float a = fabsf(w[i]); if (a > am) am = a; }
  uint16_t sh = scale_h(am / 127.0f, st);
  float S = (float)o_h2d(sh);
  for (int i = 0; i < k; i++) codes[i] = (int8_t)(int)fclampf(rne(w[i] / S), -127.0f, 127.0f);
  *s_out = sh;
}

/* ------------------------------------------------------------------------- */
/* Whole-matrix quantize to LOGICAL codes and metadata.                        */
/*   W: [N][K] binary32 row-major, groups of g consecutive weights along K.    */
/*   codes: [N][K] one byte per weight (FP16: two bytes, little-endian bits).  */
/*   s1: [N][G] fp16 bits (INT4/FP4/RaZeR scale, AFPQ s+; INT8: [N] row scale) */
/*   s2: [N][G] fp16 bits (AFPQ s-), z: [N][G] (INT4 zero, RaZeR selector).    */
/* Returns a status code.                                                      */
/* ------------------------------------------------------------------------- */
int o_quantize(int fmt, const float* W, int N, int K, int g,
               uint8_t* codes, uint16_t* s1, uint16_t* s2, uint8_t* z) {
  int status = OS_OK;
  for (long n = 0; n < N; n++)
    if (!all_finite(W + n * (long)K, K)) return OS_NONFINITE;
  if (fmt == OF_FP16) {
    uint16_t* out = (uint16_t*)codes;
    for (long i = 0; i < (long)N * K; i++) {
      out[i] = o_f2h(W[i]);
      if ((out[i] & 0x7C00) == 0x7C00) status = OS_RANGE;
    }
    return status;
  }
  if (fmt == OF_INT8) {
    int st = OS_OK;
    #pragma omp parallel for schedule(static) reduction(max:st)
    for (long n = 0; n < N; n++) {
      int st_n = OS_OK;
      q_int8_row(W + n * (long)K, K, (int8_t*)codes + n * (long)K, s1 + n, &st_n);
      if (st_n > st) st = st_n;
    }
    return st;
  }
  int G = K / g;
  int st = OS_OK;
  #pragma omp parallel for schedule(static) reduction(max:st)
  for (long n = 0; n < N; n++) {
    int st_n = OS_OK;
    for (int j = 0; j < G; j++) {
      const float* w = W + n * (long)K + (long)j * g;
      uint8_t* c = codes + n * (long)K + (long)j * g;
      long f = n * (long)G + j;
      switch (fmt) {
        case OF_INT4: q_int4(w, g, c, s1 + f, z + f, &st_n); break;
        case OF_FP4: q_fp4(w, g, c, s1 + f, &st_n); break;
        case OF_AFPQ: q_afpq(w, g, c, s1 + f, s2 + f, &st_n); break;
        case OF_RAZER: q_razer(w, g, c, s1 + f, z + f, &st_n); break;
        default: break;
      }
    }
    if (st_n > st) st = st_n;
  }
  return st;
}

/* Dequantized value of one logical code, exact in binary64. */
double o_dequant_one(int fmt, int code, uint16_t s1, uint16_t s2, int z) {
  switch (fmt) {
    case OF_INT4: return (double)(code - z) * o_h2d(s1);
    case OF_FP4: return o_e2m1(code) * o_h2d(s1);
    case OF_AFPQ: {
      double v = o_e2m1(code);
      return v > 0.0 ? v * o_h2d(s1) : v * o_h2d(s2);
    }
    case OF_RAZER: return (code == 8 ? RAZER_SV[z & 3] : o_e2m1(code)) * o_h2d(s1);
    case OF_INT8: return (double)(int8_t)code * o_h2d(s1);
    default: return 0.0;
  }
}

/* Dequantize a whole matrix of logical codes into binary64 [N][K]. */
void o_dequant(int fmt, const uint8_t* codes, const uint16_t* s1, const uint16_t* s2,
               const uint8_t* z, int N, int K, int g, double* out) {
  #pragma omp parallel for schedule(static)
  for (long n = 0; n < N; n++) {
    for (long k = 0; k < K; k++) {
      long i = n * (long)K + k;
      if (fmt == OF_FP16) { out[i] = o_h2d(((const uint16_t*)codes)[i]); continue; }
      if (fmt == OF_INT8) { out[i] = o_dequant_one(fmt, codes[i], s1[n], 0, 0); continue; }
      long f = n * (long)(K / g) + k / g;
      out[i] = o_dequant_one(fmt, codes[i], s1[f], s2 ? s2[f] : 0, z ? z[f] : 0);
    }
  }
}

/* ------------------------------------------------------------------------- */
/* Reference GEMV/GEMM in binary64:                                            */
/*   Y[m][n] = sum_k dq[n][k] * X[m][k],  A[m][n] = sum_k |dq[n][k] X[m][k]|   */
/* X is given as fp16 (xdt=0) or bf16 (xdt=1) bit patterns, [M][K] row-major.  */
/* Summation over k in increasing order.                                       */
/* ------------------------------------------------------------------------- */
void o_gemm(int fmt, const uint8_t* codes, const uint16_t* s1, const uint16_t* s2,
            const uint8_t* z, int N, int K, int g,
            const uint16_t* X, int xdt, int M, double* Y, double* A) {
  double* xd = (double*)malloc(sizeof(double) * (size_t)M * K);
  for (long i = 0; i < (long)M * K; i++) xd[i] = xdt ? o_bf2d(X[i]) : o_h2d(X[i]);
  #pragma omp parallel for schedule(static)
  for (long n = 0; n < N; n++) {
    double* dq = (double*)malloc(sizeof(double) * (size_t)K);
    for (long k = 0; k < K; k++) {
      long i = n * (long)K + k;
      if (fmt == OF_FP16) dq[k] = o_h2d(((const uint16_t*)codes)[i]);
      else if (fmt == OF_INT8) dq[k] = o_dequant_one(fmt, codes[i], s1[n], 0, 0);
      else {
        long f = n * (long)(K / g) + k / g;
        dq[k] = o_dequant_one(fmt, codes[i], s1[f], s2 ? s2[f] : 0, z ? z[f] : 0);
      }
    }
    for (int m = 0; m < M; m++) {
      double acc = 0.0, aacc = 0.0;
      const double* x = xd + (long)m * K;
      for (long k = 0; k < K; k++) { double p = dq[k] * x[k]; acc += p; aacc += fabs(p); }
      Y[(long)m * N + n] = acc;
      A[(long)m * N + n] = aacc;
    }
    free(dq);
  }
  free(xd);
}

/* ------------------------------------------------------------------------- */
/* Packed layout (the library's documented storage format, restated from its */
/* text; this is the independent unpacker/packer used by the tests).           */
/*                                                                            */
/* 4-bit formats: rows are stored in groups of eight (row group R = n/8; the  */
/* codes buffer holds ceil(N/8)*8 rows, padding rows unspecified).  Row group */
/* R occupies 4K bytes starting at R*4K.  Within it, block b (weights         */
/* 128b..128b+127 of each of the eight rows) occupies 512 bytes at 512b; row  */
/* i = n%8 of the group sits at 64i inside the block as four 16-byte chunks,  */
/* and chunk c (weights 128b+32c..128b+32c+31 of the row) is stored at chunk  */
/* position c XOR ((i/2) % 4), i.e. at byte 64i + 16*(c ^ ((i/2) % 4)).       */
/* The 16 bytes of a chunk are four little-endian 32-bit words; nibble p      */
/* (bits 4p..4p+3) of word j holds chunk weight                               */
/*   INT4:             16*(p%2) + 4j + 2*((p/2)%2) + p/4                      */
/*   FP4, AFPQ, RaZeR: 8j + p                                                 */
/* INT8: codes row-major, one signed byte per weight.  FP16: row-major fp16.  */
/*                                                                            */
/* Metadata (byte offsets within the metadata buffer), G = K/g, P = N*G:      */
/*   INT4:  fp16 scale[P] at 0; zero nibbles at Z0 = round_up(2P, 256):        */
/*          group f -> byte Z0 + f/2, low nibble if f even else high nibble;   */
/*          plane length round_up(ceil(P/2), 16) bytes.                        */
/*   FP4:   fp16 scale[P] at 0.                                                */
/*   AFPQ:  32-bit word[P] at 0: low half fp16 s+, high half fp16 s-.          */
/*   RaZeR: fp16 scale[P] at 0; selectors at Z0 = round_up(2P, 256):           */
/*          group f -> byte Z0 + f/4, bits 2*(f%4)..2*(f%4)+1;                 */
/*          plane length round_up(ceil(P/4), 16) bytes.                        */
/*   Every metadata buffer length is a multiple of 16 bytes.                  */
/*   INT8:  fp16 scale[N] at 0.                                                */
/*   FP16:  no metadata.                                                       */
/* ------------------------------------------------------------------------- */

/* Byte offset within the packed codes and nibble index (0 low, 1 high) of
 * weight (n, k) for a 4-bit format: invert the chunk-weight formula above. */
static void nib_pos(int fmt, long n, long k, int K, long* byte, int* hi) {
  long R = n / 8, i = n % 8;            /* row group, row within the group */
  long b = k / 128, c = (k % 128) / 32; /* block, chunk within the row's block */
  long e = k % 32;                      /* weight within the chunk */
  long j;
  int p;
  if (fmt == OF_INT4) {
    long h = e / 16, r = e % 16;        /* h = p%2; r = 4j + 2*((p/2)%2) + p/4 */
    j = r / 4;
    p = (int)(h + 2 * ((r % 4) / 2) + 4 * (r % 2));
  } else {
    j = e / 8;
    p = (int)(e % 8);
  }
  *byte = R * 4L * K + 512 * b + 64 * i + 16 * (c ^ ((i / 2) % 4)) + 4 * j + p / 2;
  *hi = p & 1;
}

long o_codes_bytes(int fmt, long N, long K) {
  if (fmt == OF_INT8) return N * K;
  if (fmt == OF_FP16) return 2 * N * K;
  return (N + 7) / 8 * 8 * K / 2;   /* 4-bit: whole row groups of eight */
}

static long round_up(long v, long a) { return (v + a - 1) / a * a; }

long o_meta_bytes(int fmt, long N, long K, long g) {
  long P = (fmt == OF_INT8 || fmt == OF_FP16) ? N : N * (K / g);
  switch (fmt) {
    case OF_INT4: return round_up(2 * P, 256) + round_up((P + 1) / 2, 16);
    case OF_FP4: return round_up(2 * P, 16);
    case OF_AFPQ: return round_up(4 * P, 16);
    case OF_RAZER: return round_up(2 * P, 256) + round_up((P + 3) / 4, 16);
    case OF_INT8: return round_up(2 * N, 16);
    default: return 0;
  }
}

/* logical -> packed */
void o_pack(int fmt, int N, int K, int g, const uint8_t* codes, const uint16_t* s1,
            const uint16_t* s2, const uint8_t* z, uint8_t* pc, uint8_t* pm) {
  long P = (fmt == OF_INT8 || fmt == OF_FP16) ? N : (long)N * (K / g);
  memset(pc, 0, (size_t)o_codes_bytes(fmt, N, K));
  memset(pm, 0, (size_t)o_meta_bytes(fmt, N, K, g));
  if (fmt == OF_INT8 || fmt == OF_FP16) {
    memcpy(pc, codes, (size_t)o_codes_bytes(fmt, N, K));
    if (fmt == OF_INT8) memcpy(pm, s1, 2 * (size_t)N);
    return;
  }
  for (long n = 0; n < N; n++)
    for (long k = 0; k < K; k++) {
      long b; int hi;
      nib_pos(fmt, n, k, K, &b, &hi);
      uint8_t c = codes[n * (long)K + k] & 15;
      pc[b] |= hi ? (uint8_t)(c << 4) : c;
    }
  long Z0 = round_up(2 * P, 256);
  for (long f = 0; f < P; f++) {
    if (fmt == OF_AFPQ) {
      pm[4 * f] = s1[f] & 255; pm[4 * f + 1] = s1[f] >> 8;
      pm[4 * f + 2] = s2[f] & 255; pm[4 * f + 3] = s2[f] >> 8;
      continue;
    }
    pm[2 * f] = s1[f] & 255; pm[2 * f + 1] = s1[f] >> 8;
    if (fmt == OF_INT4) pm[Z0 + f / 2] |= (uint8_t)((z[f] & 15) << (4 * (f & 1)));
    if (fmt == OF_RAZER) pm[Z0 + f / 4] |= (uint8_t)((z[f] & 3) << (2 * (f & 3)));
  }
}

/* packed -> logical */
void o_unpack(int fmt, int N, int K, int g, const uint8_t* pc, const uint8_t* pm,
              uint8_t* codes, uint16_t* s1, uint16_t* s2, uint8_t* z) {
  long P = (fmt == OF_INT8 || fmt == OF_FP16) ? N : (long)N * (K / g);
  if (fmt == OF_INT8 || fmt == OF_FP16) {
    memcpy(codes, pc, (size_t)o_codes_bytes(fmt, N, K));
    if (fmt == OF_INT8) for (long n = 0; n < N; n++) s1[n] = (uint16_t)(pm[2 * n] | (pm[2 * n + 1] << 8));
    return;
  }
  for (long n = 0; n < N; n++)
    for (long k = 0; k < K; k++) {
      long b; int hi;
      nib_pos(fmt, n, k, K, &b, &hi);
      codes[n * (long)K + k] = hi ? (pc[b] >> 4) : (pc[b] & 15);
    }
  long Z0 = round_up(2 * P, 256);
  for (long f = 0; f < P; f++) {
    if (fmt == OF_AFPQ) {
      s1[f] = (uint16_t)(pm[4 * f] | (pm[4 * f + 1] << 8));
      s2[f] = (uint16_t)(pm[4 * f + 2] | (pm[4 * f + 3] << 8));
      continue;
    }
    s1[f] = (uint16_t)(pm[2 * f] | (pm[2 * f + 1] << 8));
    if (fmt == OF_INT4) z[f] = (pm[Z0 + f / 2] >> (4 * (f & 1))) & 15;
    if (fmt == OF_RAZER) z[f] = (pm[Z0 + f / 4] >> (2 * (f & 3))) & 3;
  }
}

/* Vectorized conversion helpers for the tests. */
void o_f2h_array(const float* in, uint16_t* out, long n) { for (long i = 0; i < n; i++) out[i] = o_f2h(in[i]); }
void o_f2bf_array(const float* in, uint16_t* out, long n) { for (long i = 0; i < n; i++) out[i] = o_f2bf(in[i]); }
void o_h2d_array(const uint16_t* in, double* out, long n) { for (long i = 0; i < n; i++) out[i] = o_h2d(in[i]); }

/* Per-group quantizers exposed for brute-force tests on tiny groups. */
int o_quantize_group(int fmt, const float* w, int g, uint8_t* codes,
                     uint16_t* s1, uint16_t* s2, uint8_t* z) {
  int st = OS_OK;
  if (!all_finite(w, g)) return OS_NONFINITE;
  switch (fmt) {
    case OF_INT4: q_int4(w, g, codes, s1, z, &st); break;
    case OF_FP4: q_fp4(w, g, codes, s1, &st); break;
    case OF_AFPQ: q_afpq(w, g, codes, s1, s2, &st); break;
    case OF_RAZER: q_razer(w, g, codes, s1, z, &st); break;
    default: return -1;
  }
  return st;
}

/* Number of OpenMP threads the oracle's parallel loops use (1 without OpenMP). */
int o_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
