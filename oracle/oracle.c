/*
 * oracle.c -- plain, slow CPU oracle for int4 KV-cache quantization and
 * decode attention over the packed int4 cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or constant with the CUDA path and includes nothing
 * from it.
 *
 * Sources (web pages on the method; cited by title and section):
 *  [OTM]    "Open-TQ-Metal: Fused Compressed-Domain Attention for Long-Context
 *           LLM Inference on Apple Silicon" (arXiv 2604.16957v1), abstract:
 *           the KV cache is quantized to int4 as it is produced and attention
 *           is computed directly on the compressed representation, with no
 *           intermediate dequantized matrix; attn_scale is 1/sqrt(d) (Llama)
 *           or 1.0 (Gemma 4).
 *  [OTM-F]  zingnex forum summary of Open-TQ-Metal, sections "on-the-fly
 *           quantization", "compressed-domain attention", "eliminating
 *           intermediate matrices", "numerical stability".
 *  [AdapTQ] zingnex post on AdapTQ, section "Fast Hadamard Rotation (HAR)":
 *           an in-place O(d log d) Hadamard rotation before quantization
 *           spreads outliers.
 *  [SRFT]   agents-report.net post "SRFT + int4 KV-cache on Apple Silicon",
 *           section on the core method: sign-randomized rotation (the
 *           sign-randomized Hadamard is reported equivalent in quality), then
 *           per-group abs-max, symmetric int4, nibble packing.
 *
 * Readings where the pages are silent (all listed in the design notes):
 *  - rotation R = (1/sqrt d) * H_d * diag(sigma), H_d Sylvester-ordered,
 *    H[i][j] = (-1)^popcount(i & j); sigma in {+1,-1}^d; inverse is R^T.
 *  - rotated vector computed in fp64 with the explicit d x d matrix and
 *    rounded once to fp32.
 *  - groups of 32 consecutive rotated coordinates; scale s = fl32(amax / 7)
 *    (fp32 IEEE division); codes c = clamp(rne(fl32(y / s)), -7, 7) with
 *    round-half-to-even of the fp32 quotient; an all-zero group has s = 0 and
 *    codes 0.
 *  - attention output = exact softmax attention over the dequantized values
 *    s*c in the rotated basis, mapped back with R^T, all in fp64.
 *  - codebook variant ([AdapTQ], sections "unified SIMD pipeline",
 *    "precomputed lookup tables", "performance and quality": 2-, 3- and 4-bit
 *    indices into a Max-Lloyd codebook with +-3 sigma clipping; int2 is the
 *    future work of [OTM-F]): per group of 32 rotated coordinates a scale
 *    sigma = fl32(sqrt(S / 32)), S = sum of y^2 in fp64; u = fl32(y / sigma)
 *    clipped to [-3, 3]; index = number of thresholds t_i < u, where
 *    t_i = fl32(fl32(C_i + C_{i+1}) * 0.5) for the fp32 levels C_0 < ... <
 *    C_{L-1}, L = 2^bits; the value is sigma * C[index].  Indices are packed
 *    little-endian: index j of group g occupies bits bits*j .. bits*j+bits-1
 *    of the group's 4*bits bytes, groups in order.  The Gaussian Max-Lloyd
 *    codebook is the fixed point of "thresholds at midpoints, levels at the
 *    cell means of N(0,1)".
 *  - uniform low-bit variant ([OTM-F], future work: int2; read as the int4
 *    quantizer at fewer bits): with m = 2^(bits-1) - 1, per group of 32
 *    rotated coordinates s = fl32(amax / m) (fp32 IEEE division; s = amax at
 *    two bits), c = clamp(rne(fl32(y / s)), -m, m), stored as the index c + m
 *    in the codebook layout; the value is s * c.  The cache is a codebook
 *    cache whose levels are the integers C[u] = u - m (u < 2^bits; the top
 *    index is never written).
 *  - SRFT variant ([SRFT], core method: a sign-randomized Fourier transform
 *    instead of the Hadamard one, usable at widths that are not powers of
 *    two, followed by a per-coordinate scale lambda): the transform is the
 *    orthonormal discrete Hartley transform F[k][j] = cas(2 pi k j / d) /
 *    sqrt(d), cas = cos + sin (real, symmetric, F F = I).  The stored vector
 *    is y = fl32(lambda (.) F (sigma (.) x)); K and V have their own lambda.
 *    Scores use q_r = F (sigma (.) q) / lambda_K, so q_r . y_k = q . k; the
 *    output is sigma (.) F (o_r / lambda_V).
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GROUP 32

/* ------------------------------------------------------------------ */
/* inputs                                                               */
/* ------------------------------------------------------------------ */

/* bf16 -> fp32 is exact: the 16 bits are the high half of the fp32 word. */
static float bf16_bits_to_float(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* element `idx` of an fp32 (dtype 0) or bf16 (dtype 1) array, as fp32 */
static float load_input(const void* base, int dtype, int64_t idx) {
  if (dtype == 0) return ((const float*)base)[idx];
  return bf16_bits_to_float(((const uint16_t*)base)[idx]);
}

/* ------------------------------------------------------------------ */
/* rotation ([AdapTQ] HAR; [SRFT] sign-randomized rotation)             */
/* ------------------------------------------------------------------ */

static int popcount_u32(uint32_t x) {
  int n = 0;
  while (x) { n += (int)(x & 1u); x >>= 1; }
  return n;
}

/* Sylvester-ordered Walsh-Hadamard entry H_d[i][j] = (-1)^popcount(i&j). */
int oracle_hadamard_entry(int i, int j) {
  return (popcount_u32((uint32_t)(i & j)) & 1) ? -1 : 1;
}

/* R[i*d + j] = H[i][j] * sigma[j] / sqrt(d); identity when signs == NULL. */
int oracle_rotation_matrix(int d, const int8_t* signs, double* R) {
  if (d <= 0 || (d & (d - 1)) != 0 || !R) return -1;
  double inv = 1.0 / sqrt((double)d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) {
      if (!signs) R[(int64_t)i * d + j] = (i == j) ? 1.0 : 0.0;
      else R[(int64_t)i * d + j] = inv * (double)oracle_hadamard_entry(i, j) * (double)signs[j];
    }
  return 0;
}

/* y = fl32(R x): fp64 matrix-vector product, rounded once to fp32. */
void oracle_rotate_vector(int d, const double* R, const float* x, float* y) {
  for (int i = 0; i < d; ++i) {
    double acc = 0.0;
    for (int j = 0; j < d; ++j) acc += R[(int64_t)i * d + j] * (double)x[j];
    y[i] = (float)acc;
  }
}

/* ------------------------------------------------------------------ */
/* SRFT rotation ([SRFT] core method: sign-randomized Fourier transform, */
/* any width, then a per-coordinate scale lambda)                        */
/* ------------------------------------------------------------------ */

/* Orthonormal discrete Hartley transform entry F_d[k][j] = cas(2 pi k j / d) / sqrt(d);
   the product k j is reduced mod d first so the angle is computed exactly. */
double oracle_dht_entry(int d, int k, int j) {
  int64_t t = ((int64_t)k * (int64_t)j) % d;
  double th = 2.0 * acos(-1.0) * (double)t / (double)d;
  return (cos(th) + sin(th)) / sqrt((double)d);
}

/* Store map A[k*d + j] = lambda[k] * F_d[k][j] * sigma[j] (y = A x); lambda NULL = ones,
   signs NULL = ones.  Any d >= 1. */
int oracle_srft_matrix(int d, const int8_t* signs, const float* lambda, double* A) {
  if (d <= 0 || !A) return -1;
  for (int k = 0; k < d; ++k)
    for (int j = 0; j < d; ++j) {
      double v = oracle_dht_entry(d, k, j);
      if (signs) v *= (double)signs[j];
      if (lambda) v *= (double)lambda[k];
      A[(int64_t)k * d + j] = v;
    }
  return 0;
}

/* Query map Q[k*d + j] = F_d[k][j] * sigma[j] / lambda_k[k] (q_r = Q q) and output map
   O[j*d + k] = sigma[j] * F_d[j][k] / lambda_v[k] (o = O o_r). */
static void srft_query_output_maps(int d, const int8_t* signs, const float* lambda_k,
                                   const float* lambda_v, double* Q, double* O) {
  for (int k = 0; k < d; ++k)
    for (int j = 0; j < d; ++j) {
      double f = oracle_dht_entry(d, k, j);
      double sj = signs ? (double)signs[j] : 1.0;
      Q[(int64_t)k * d + j] = f * sj / (lambda_k ? (double)lambda_k[k] : 1.0);
      /* F is symmetric: F[j][k] = F[k][j] */
      O[(int64_t)j * d + k] = sj * f / (lambda_v ? (double)lambda_v[k] : 1.0);
    }
}

/* ------------------------------------------------------------------ */
/* quantization ([SRFT] per-group abs-max, symmetric int4)              */
/* ------------------------------------------------------------------ */

/* codes[d] in [-7,7], scales[d/32]; y already rotated (or not). */
void oracle_quantize_vector(int d, const float* y, int8_t* codes, float* scales) {
  int ng = d / ORACLE_GROUP;
  for (int g = 0; g < ng; ++g) {
    const float* yg = y + g * ORACLE_GROUP;
    float amax = 0.0f;
    for (int i = 0; i < ORACLE_GROUP; ++i) {
      float a = fabsf(yg[i]);
      if (a > amax) amax = a;
    }
    volatile float seven = 7.0f;          /* keep the division in fp32 IEEE */
    float s = amax / seven;
    scales[g] = s;
    for (int i = 0; i < ORACLE_GROUP; ++i) {
      int c = 0;
      if (amax > 0.0f) {
        volatile float quot = yg[i] / s;  /* fp32 quotient, rounded once */
        float r = nearbyintf(quot);       /* round half to even (default mode) */
        if (r > 7.0f) r = 7.0f;
        if (r < -7.0f) r = -7.0f;
        c = (int)r;
      }
      codes[g * ORACLE_GROUP + i] = (int8_t)c;
    }
  }
}

/* ------------------------------------------------------------------ */
/* nibble packing ([SRFT] "nibble pack"; byte order is this library's)  */
/* ------------------------------------------------------------------ */
/*
 * Packed row of one vector: d/2 bytes.  Coordinate i (rotated basis) with
 * group g = i / 32 and in-group index j = i % 32 lives in
 *     byte  = (j / 4) * (2 * ng) + 2 * g + (j % 4) / 2,      ng = d / 32
 *     nibble = j % 2          (0 = bits 0..3, 1 = bits 4..7)
 * as a 4-bit two's-complement code.  I.e. the row is 8 sub-blocks; sub-block
 * r holds in-group coordinates 4r..4r+3 of every group, two bytes per group.
 */
int64_t oracle_packed_byte_index(int d, int i) {
  int ng = d / ORACLE_GROUP;
  int g = i / ORACLE_GROUP, j = i % ORACLE_GROUP;
  return (int64_t)(j / 4) * (2 * ng) + 2 * g + (j % 4) / 2;
}

void oracle_pack_vector(int d, const int8_t* codes, uint8_t* packed) {
  memset(packed, 0, (size_t)d / 2);
  for (int i = 0; i < d; ++i) {
    int64_t b = oracle_packed_byte_index(d, i);
    uint8_t nib = (uint8_t)(codes[i] & 0x0F);
    int shift = ((i % ORACLE_GROUP) % 2) ? 4 : 0;
    packed[b] = (uint8_t)(packed[b] | (nib << shift));
  }
}

void oracle_unpack_vector(int d, const uint8_t* packed, int8_t* codes) {
  for (int i = 0; i < d; ++i) {
    int64_t b = oracle_packed_byte_index(d, i);
    int shift = ((i % ORACLE_GROUP) % 2) ? 4 : 0;
    int nib = (packed[b] >> shift) & 0x0F;
    codes[i] = (int8_t)(nib >= 8 ? nib - 16 : nib);
  }
}

/* ------------------------------------------------------------------ */
/* quantize-append ([OTM-F] on-the-fly quantization)                    */
/* ------------------------------------------------------------------ */
/*
 * k, v: [B][Hkv][n_new][d] fp32 (dtype 0) or bf16 (dtype 1).
 * Token n of (b, h) goes to cache row pos[b] + n of that (b, h) slot.
 * caches: packed [B][Hkv][capacity][d/2], scales [B][Hkv][capacity][d/32].
 */
/* The store maps Ak, Av (d x d, y = fl32(A x)) or NULL for y = x. */
static int quantize_append_maps(const void* k, const void* v, int in_dtype, int B, int Hkv,
                                int n_new, int d, const int32_t* pos, const double* Ak,
                                const double* Av, uint8_t* k_packed, float* k_scales,
                                uint8_t* v_packed, float* v_scales, int64_t capacity,
                                int nthreads) {
  int ng = d / ORACLE_GROUP;
  int64_t nvec = (int64_t)B * Hkv * n_new;
#ifdef _OPENMP
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
#endif
  for (int64_t idx = 0; idx < nvec; ++idx) {
    float x[512], y[512];
    int8_t codes[512];
    int64_t b = idx / ((int64_t)Hkv * n_new);
    int64_t h = (idx / n_new) % Hkv;
    int64_t n = idx % n_new;
    int64_t row = ((int64_t)b * Hkv + h) * capacity + pos[b] + n;
    for (int kv = 0; kv < 2; ++kv) {
      const void* src = kv ? v : k;
      const double* A = kv ? Av : Ak;
      for (int i = 0; i < d; ++i) x[i] = load_input(src, in_dtype, idx * d + i);
      if (A) oracle_rotate_vector(d, A, x, y);
      else memcpy(y, x, sizeof(float) * (size_t)d);
      float* sc = (kv ? v_scales : k_scales) + row * ng;
      uint8_t* pk = (kv ? v_packed : k_packed) + row * (d / 2);
      oracle_quantize_vector(d, y, codes, sc);
      oracle_pack_vector(d, codes, pk);
    }
  }
  return 0;
}

static int check_append(int B, int n_new, int d, const int32_t* pos, int64_t capacity) {
  if (d % ORACLE_GROUP != 0 || d > 512) return -1;
  for (int b = 0; b < B; ++b)
    if (pos[b] < 0 || (int64_t)pos[b] + n_new > capacity) return -1;
  return 0;
}

/* Hadamard rotation (signs) or none (signs == NULL). */
int oracle_quantize_append(const void* k, const void* v, int in_dtype, int B, int Hkv,
                           int n_new, int d, const int32_t* pos, const int8_t* signs,
                           uint8_t* k_packed, float* k_scales, uint8_t* v_packed,
                           float* v_scales, int64_t capacity, int nthreads) {
  if ((d & (d - 1)) != 0 || check_append(B, n_new, d, pos, capacity) != 0) return -1;
  double* R = NULL;
  if (signs) {
    R = (double*)malloc(sizeof(double) * (size_t)d * d);
    if (!R) return -2;
    oracle_rotation_matrix(d, signs, R);
  }
  int rc = quantize_append_maps(k, v, in_dtype, B, Hkv, n_new, d, pos, R, R, k_packed, k_scales,
                                v_packed, v_scales, capacity, nthreads);
  free(R);
  return rc;
}

/* SRFT rotation: y = fl32(lambda (.) F (sigma (.) x)), lambda_k for K, lambda_v for V. */
int oracle_quantize_append_srft(const void* k, const void* v, int in_dtype, int B, int Hkv,
                                int n_new, int d, const int32_t* pos, const int8_t* signs,
                                const float* lambda_k, const float* lambda_v, uint8_t* k_packed,
                                float* k_scales, uint8_t* v_packed, float* v_scales,
                                int64_t capacity, int nthreads) {
  if (check_append(B, n_new, d, pos, capacity) != 0) return -1;
  double* Ak = (double*)malloc(sizeof(double) * (size_t)d * d);
  double* Av = (double*)malloc(sizeof(double) * (size_t)d * d);
  int rc = -2;
  if (Ak && Av) {
    oracle_srft_matrix(d, signs, lambda_k, Ak);
    oracle_srft_matrix(d, signs, lambda_v, Av);
    rc = quantize_append_maps(k, v, in_dtype, B, Hkv, n_new, d, pos, Ak, Av, k_packed, k_scales,
                              v_packed, v_scales, capacity, nthreads);
  }
  free(Ak);
  free(Av);
  return rc;
}

/* ------------------------------------------------------------------ */
/* decode attention over the packed cache ([OTM] sdpa_int4)             */
/* ------------------------------------------------------------------ */
/*
 * q: [B][Hq][d] fp32/bf16, one query token per sequence.  Query head hq uses
 * KV head hq / (Hq/Hkv).  Sequence b attends cache rows 0..ctx_lens[b]-1.
 * out: [B][Hq][d] fp64, in the unrotated basis.
 *   q_r = R q;  S_t = attn_scale * sum_i q_r[i] * s_k[t][g(i)] * c_k[t][i]
 *   p = softmax(S);  o_r[i] = sum_t p_t * s_v[t][g(i)] * c_v[t][i];  o = R^T o_r
 */
/* Q: query map (q_r = Q q), O: output map (o = O o_r), both d x d. */
static int sdpa_int4_decode_maps(const void* q, int q_dtype, int B, int Hq, int Hkv, int d,
                                 const uint8_t* k_packed, const float* k_scales,
                                 const uint8_t* v_packed, const float* v_scales, int64_t capacity,
                                 const int32_t* ctx_lens, const double* Q, const double* O,
                                 double attn_scale, double* out, int nthreads) {
  int G = Hq / Hkv, ng = d / ORACLE_GROUP;
  int64_t nrows = (int64_t)B * Hq;
  int fail = 0;
#ifdef _OPENMP
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
#endif
  for (int64_t bh = 0; bh < nrows; ++bh) {
    int64_t b = bh / Hq, hq = bh % Hq, hk = hq / G;
    int64_t T = ctx_lens[b];
    double qv[512], qr[512], orot[512];
    int8_t codes[512];
    double* S = (double*)malloc(sizeof(double) * (size_t)T);
    if (!S) { fail = 1; continue; }
    for (int i = 0; i < d; ++i) qv[i] = (double)load_input(q, q_dtype, bh * d + i);
    for (int i = 0; i < d; ++i) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += Q[(int64_t)i * d + j] * qv[j];
      qr[i] = acc;
    }
    int64_t base = ((int64_t)b * Hkv + hk) * capacity;
    double smax = -INFINITY;
    for (int64_t t = 0; t < T; ++t) {
      oracle_unpack_vector(d, k_packed + (base + t) * (d / 2), codes);
      const float* sk = k_scales + (base + t) * ng;
      double dot = 0.0;
      for (int i = 0; i < d; ++i) dot += qr[i] * ((double)sk[i / ORACLE_GROUP] * (double)codes[i]);
      S[t] = attn_scale * dot;
      if (S[t] > smax) smax = S[t];
    }
    double Z = 0.0;
    for (int64_t t = 0; t < T; ++t) { S[t] = exp(S[t] - smax); Z += S[t]; }
    for (int i = 0; i < d; ++i) orot[i] = 0.0;
    for (int64_t t = 0; t < T; ++t) {
      oracle_unpack_vector(d, v_packed + (base + t) * (d / 2), codes);
      const float* sv = v_scales + (base + t) * ng;
      double p = S[t] / Z;
      for (int i = 0; i < d; ++i) orot[i] += p * ((double)sv[i / ORACLE_GROUP] * (double)codes[i]);
    }
    for (int j = 0; j < d; ++j) {   /* o = O o_r */
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += O[(int64_t)j * d + i] * orot[i];
      out[bh * d + j] = acc;
    }
    free(S);
  }
  return fail ? -2 : 0;
}

static int check_decode(int B, int Hq, int Hkv, int d, const int32_t* ctx_lens, int64_t capacity) {
  if (Hkv <= 0 || Hq % Hkv != 0 || d % ORACLE_GROUP != 0 || d > 512) return -1;
  for (int b = 0; b < B; ++b)
    if (ctx_lens[b] < 1 || ctx_lens[b] > capacity) return -1;
  return 0;
}

/* Hadamard rotation (signs; q_r = R q, o = R^T o_r) or none (signs == NULL). */
int oracle_sdpa_int4_decode(const void* q, int q_dtype, int B, int Hq, int Hkv, int d,
                            const uint8_t* k_packed, const float* k_scales,
                            const uint8_t* v_packed, const float* v_scales, int64_t capacity,
                            const int32_t* ctx_lens, const int8_t* signs, double attn_scale,
                            double* out, int nthreads) {
  if ((d & (d - 1)) != 0 || check_decode(B, Hq, Hkv, d, ctx_lens, capacity) != 0) return -1;
  double* R = (double*)malloc(sizeof(double) * (size_t)d * d);
  double* RT = (double*)malloc(sizeof(double) * (size_t)d * d);
  int rc = -2;
  if (R && RT) {
    oracle_rotation_matrix(d, signs, R);
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < d; ++j) RT[(int64_t)j * d + i] = R[(int64_t)i * d + j];
    rc = sdpa_int4_decode_maps(q, q_dtype, B, Hq, Hkv, d, k_packed, k_scales, v_packed, v_scales,
                               capacity, ctx_lens, R, RT, attn_scale, out, nthreads);
  }
  free(R);
  free(RT);
  return rc;
}

/* SRFT rotation: q_r = F (sigma (.) q) / lambda_k, o = sigma (.) F (o_r / lambda_v). */
int oracle_sdpa_int4_decode_srft(const void* q, int q_dtype, int B, int Hq, int Hkv, int d,
                                 const uint8_t* k_packed, const float* k_scales,
                                 const uint8_t* v_packed, const float* v_scales, int64_t capacity,
                                 const int32_t* ctx_lens, const int8_t* signs,
                                 const float* lambda_k, const float* lambda_v, double attn_scale,
                                 double* out, int nthreads) {
  if (check_decode(B, Hq, Hkv, d, ctx_lens, capacity) != 0) return -1;
  double* Q = (double*)malloc(sizeof(double) * (size_t)d * d);
  double* O = (double*)malloc(sizeof(double) * (size_t)d * d);
  int rc = -2;
  if (Q && O) {
    srft_query_output_maps(d, signs, lambda_k, lambda_v, Q, O);
    rc = sdpa_int4_decode_maps(q, q_dtype, B, Hq, Hkv, d, k_packed, k_scales, v_packed, v_scales,
                               capacity, ctx_lens, Q, O, attn_scale, out, nthreads);
  }
  free(Q);
  free(O);
  return rc;
}

/* ------------------------------------------------------------------ */
/* codebook variant ([AdapTQ] Max-Lloyd codebook, 2/3/4-bit indices)   */
/* ------------------------------------------------------------------ */

static double std_normal_pdf(double x) { return exp(-0.5 * x * x) / sqrt(2.0 * acos(-1.0)); }
static double std_normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Gaussian Max-Lloyd codebook of 2^bits levels (fp64, increasing): iterate
   thresholds = midpoints of adjacent levels, levels = means of N(0,1) over
   their cells, E[X | a < X < b] = (pdf(a) - pdf(b)) / (cdf(b) - cdf(a)). */
int oracle_lloyd_max_gaussian(int bits, double* levels) {
  if (bits < 1 || bits > 8 || !levels) return -1;
  int L = 1 << bits;
  for (int i = 0; i < L; ++i) levels[i] = -3.0 + 6.0 * (i + 0.5) / L;  /* start: uniform on [-3, 3] */
  for (int it = 0; it < 100000; ++it) {
    double change = 0.0;
    for (int i = 0; i < L; ++i) {
      double a = (i == 0) ? -INFINITY : 0.5 * (levels[i - 1] + levels[i]);
      double b = (i == L - 1) ? INFINITY : 0.5 * (levels[i] + levels[i + 1]);
      double pa = isinf(a) ? 0.0 : std_normal_pdf(a), pb = isinf(b) ? 0.0 : std_normal_pdf(b);
      double ca = isinf(a) ? 0.0 : std_normal_cdf(a), cb = isinf(b) ? 1.0 : std_normal_cdf(b);
      double m = (pa - pb) / (cb - ca);
      change = fmax(change, fabs(m - levels[i]));
      levels[i] = m;
    }
    if (change < 1e-15) break;
  }
  return 0;
}

/* thresholds t_i = fl32(fl32(C_i + C_{i+1}) * 0.5), i < L - 1 */
static void cb_thresholds(int L, const float* C, float* t) {
  for (int i = 0; i + 1 < L; ++i) {
    volatile float sum = C[i] + C[i + 1];
    t[i] = sum * 0.5f;
  }
}

/* indices[d], scales[d/32] of an already-rotated vector y */
void oracle_cb_quantize_vector(int d, const float* y, int bits, const float* C, uint8_t* idx,
                               float* scales) {
  int L = 1 << bits, ng = d / ORACLE_GROUP;
  float t[255];
  cb_thresholds(L, C, t);
  for (int g = 0; g < ng; ++g) {
    const float* yg = y + g * ORACLE_GROUP;
    double S = 0.0;
    for (int j = 0; j < ORACLE_GROUP; ++j) S += (double)yg[j] * (double)yg[j];
    float sigma = (float)sqrt(S / (double)ORACLE_GROUP);
    scales[g] = sigma;
    for (int j = 0; j < ORACLE_GROUP; ++j) {
      float u = 0.0f;
      if (sigma > 0.0f) {
        volatile float quot = yg[j] / sigma;  /* fp32 quotient, rounded once */
        u = quot;
      }
      if (u > 3.0f) u = 3.0f;
      if (u < -3.0f) u = -3.0f;
      int k = 0;
      for (int i = 0; i + 1 < L; ++i)
        if (u > t[i]) ++k;
      idx[g * ORACLE_GROUP + j] = (uint8_t)k;
    }
  }
}

/* row bytes d * bits / 8: index j of group g at bits bits*j.. of the group's bytes */
void oracle_cb_pack_vector(int d, int bits, const uint8_t* idx, uint8_t* packed) {
  int gbytes = 4 * bits;
  memset(packed, 0, (size_t)d * bits / 8);
  for (int i = 0; i < d; ++i) {
    int g = i / ORACLE_GROUP, j = i % ORACLE_GROUP;
    for (int k = 0; k < bits; ++k) {
      int bit = bits * j + k;
      if ((idx[i] >> k) & 1) packed[g * gbytes + bit / 8] |= (uint8_t)(1u << (bit % 8));
    }
  }
}

void oracle_cb_unpack_vector(int d, int bits, const uint8_t* packed, uint8_t* idx) {
  int gbytes = 4 * bits;
  for (int i = 0; i < d; ++i) {
    int g = i / ORACLE_GROUP, j = i % ORACLE_GROUP, v = 0;
    for (int k = 0; k < bits; ++k) {
      int bit = bits * j + k;
      v |= ((packed[g * gbytes + bit / 8] >> (bit % 8)) & 1) << k;
    }
    idx[i] = (uint8_t)v;
  }
}

/* Hadamard rotation (signs) or none, then the codebook quantizer; cache rows of
   d * bits / 8 bytes and d / 32 scales. */
int oracle_quantize_append_cb(const void* k, const void* v, int in_dtype, int B, int Hkv,
                              int n_new, int d, const int32_t* pos, const int8_t* signs, int bits,
                              const float* C, uint8_t* k_packed, float* k_scales,
                              uint8_t* v_packed, float* v_scales, int64_t capacity, int nthreads) {
  if ((d & (d - 1)) != 0 || check_append(B, n_new, d, pos, capacity) != 0) return -1;
  if (bits < 2 || bits > 4) return -1;
  for (int i = 0; i + 1 < (1 << bits); ++i)
    if (!(C[i] < C[i + 1])) return -1;
  double* R = NULL;
  if (signs) {
    R = (double*)malloc(sizeof(double) * (size_t)d * d);
    if (!R) return -2;
    oracle_rotation_matrix(d, signs, R);
  }
  int ng = d / ORACLE_GROUP, rowb = d * bits / 8;
  int64_t nvec = (int64_t)B * Hkv * n_new;
#ifdef _OPENMP
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
#endif
  for (int64_t idx = 0; idx < nvec; ++idx) {
    float x[512], y[512];
    uint8_t ci[512];
    int64_t b = idx / ((int64_t)Hkv * n_new);
    int64_t h = (idx / n_new) % Hkv;
    int64_t n = idx % n_new;
    int64_t row = ((int64_t)b * Hkv + h) * capacity + pos[b] + n;
    for (int kv = 0; kv < 2; ++kv) {
      const void* src = kv ? v : k;
      for (int i = 0; i < d; ++i) x[i] = load_input(src, in_dtype, idx * d + i);
      if (R) oracle_rotate_vector(d, R, x, y);
      else memcpy(y, x, sizeof(float) * (size_t)d);
      oracle_cb_quantize_vector(d, y, bits, C, ci, (kv ? v_scales : k_scales) + row * ng);
      oracle_cb_pack_vector(d, bits, ci, (kv ? v_packed : k_packed) + row * rowb);
    }
  }
  free(R);
  return 0;
}

/* ------------------------------------------------------------------ */
/* uniform low-bit variant ([OTM-F] future work: int2)                  */
/* ------------------------------------------------------------------ */

/* levels[u] = u - m, m = 2^(bits-1) - 1, u < 2^bits: the decode-side table */
int oracle_uniform_levels(int bits, float* levels) {
  if (bits < 2 || bits > 4) return -1;
  int m = (1 << (bits - 1)) - 1;
  for (int u = 0; u < (1 << bits); ++u) levels[u] = (float)(u - m);
  return 0;
}

/* indices[d] (c + m), scales[d/32] of an already-rotated vector y */
void oracle_uniform_quantize_vector(int d, const float* y, int bits, uint8_t* idx, float* scales) {
  int ng = d / ORACLE_GROUP, m = (1 << (bits - 1)) - 1;
  for (int g = 0; g < ng; ++g) {
    const float* yg = y + g * ORACLE_GROUP;
    float amax = 0.0f;
    for (int j = 0; j < ORACLE_GROUP; ++j) {
      float a = fabsf(yg[j]);
      if (a > amax) amax = a;
    }
    volatile float top = (float)m;        /* keep the division in fp32 IEEE */
    float s = amax / top;
    scales[g] = s;
    for (int j = 0; j < ORACLE_GROUP; ++j) {
      int c = 0;
      if (amax > 0.0f) {
        volatile float uq = yg[j] / s;    /* fp32 quotient, rounded once */
        float rq = nearbyintf(uq);        /* round half to even (default mode) */
        if (rq > (float)m) rq = (float)m;
        if (rq < (float)-m) rq = (float)-m;
        c = (int)rq;
      }
      idx[g * ORACLE_GROUP + j] = (uint8_t)(c + m);
    }
  }
}

/* Hadamard rotation (signs) or none, then the uniform quantizer; cache rows of
   d * bits / 8 bytes (codebook layout) and d / 32 scales. */
int oracle_quantize_append_uniform(const void* k, const void* v, int in_dtype, int B, int Hkv,
                                   int n_new, int d, const int32_t* pos, const int8_t* signs,
                                   int bits, uint8_t* k_packed, float* k_scales,
                                   uint8_t* v_packed, float* v_scales, int64_t capacity,
                                   int nthreads) {
  if ((d & (d - 1)) != 0 || check_append(B, n_new, d, pos, capacity) != 0) return -1;
  if (bits < 2 || bits > 4) return -1;
  double* R = NULL;
  if (signs) {
    R = (double*)malloc(sizeof(double) * (size_t)d * d);
    if (!R) return -2;
    oracle_rotation_matrix(d, signs, R);
  }
  int ng = d / ORACLE_GROUP, rowb = d * bits / 8;
  int64_t nvec = (int64_t)B * Hkv * n_new;
#ifdef _OPENMP
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
#endif
  for (int64_t idx = 0; idx < nvec; ++idx) {
    float x[512], y[512];
    uint8_t ci[512];
    int64_t b = idx / ((int64_t)Hkv * n_new);
    int64_t h = (idx / n_new) % Hkv;
    int64_t n = idx % n_new;
    int64_t row = ((int64_t)b * Hkv + h) * capacity + pos[b] + n;
    for (int kv = 0; kv < 2; ++kv) {
      const void* src = kv ? v : k;
      for (int i = 0; i < d; ++i) x[i] = load_input(src, in_dtype, idx * d + i);
      if (R) oracle_rotate_vector(d, R, x, y);
      else memcpy(y, x, sizeof(float) * (size_t)d);
      oracle_uniform_quantize_vector(d, y, bits, ci, (kv ? v_scales : k_scales) + row * ng);
      oracle_cb_pack_vector(d, bits, ci, (kv ? v_packed : k_packed) + row * rowb);
    }
  }
  free(R);
  return 0;
}

/* attention over a codebook cache: k_hat = sigma_k * C[index], v_hat likewise,
   q_r = R q, o = R^T o_r (R = identity without signs); fp64 */
int oracle_sdpa_cb_decode(const void* q, int q_dtype, int B, int Hq, int Hkv, int d, int bits,
                          const float* C, const uint8_t* k_packed, const float* k_scales,
                          const uint8_t* v_packed, const float* v_scales, int64_t capacity,
                          const int32_t* ctx_lens, const int8_t* signs, double attn_scale,
                          double* out, int nthreads) {
  if ((d & (d - 1)) != 0 || check_decode(B, Hq, Hkv, d, ctx_lens, capacity) != 0) return -1;
  if (bits < 2 || bits > 4) return -1;
  double* R = (double*)malloc(sizeof(double) * (size_t)d * d);
  if (!R) return -2;
  oracle_rotation_matrix(d, signs, R);
  int G = Hq / Hkv, ng = d / ORACLE_GROUP, rowb = d * bits / 8;
  int64_t nrows = (int64_t)B * Hq;
  int fail = 0;
#ifdef _OPENMP
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
#endif
  for (int64_t bh = 0; bh < nrows; ++bh) {
    int64_t b = bh / Hq, hq = bh % Hq, hk = hq / G;
    int64_t T = ctx_lens[b];
    double qv[512], qr[512], orot[512];
    uint8_t ci[512];
    double* S = (double*)malloc(sizeof(double) * (size_t)T);
    if (!S) { fail = 1; continue; }
    for (int i = 0; i < d; ++i) qv[i] = (double)load_input(q, q_dtype, bh * d + i);
    for (int i = 0; i < d; ++i) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += R[(int64_t)i * d + j] * qv[j];
      qr[i] = acc;
    }
    int64_t base = ((int64_t)b * Hkv + hk) * capacity;
    double smax = -INFINITY;
    for (int64_t t = 0; t < T; ++t) {
      oracle_cb_unpack_vector(d, bits, k_packed + (base + t) * rowb, ci);
      const float* sk = k_scales + (base + t) * ng;
      double dot = 0.0;
      for (int i = 0; i < d; ++i) dot += qr[i] * ((double)sk[i / ORACLE_GROUP] * (double)C[ci[i]]);
      S[t] = attn_scale * dot;
      if (S[t] > smax) smax = S[t];
    }
    double Z = 0.0;
    for (int64_t t = 0; t < T; ++t) { S[t] = exp(S[t] - smax); Z += S[t]; }
    for (int i = 0; i < d; ++i) orot[i] = 0.0;
    for (int64_t t = 0; t < T; ++t) {
      oracle_cb_unpack_vector(d, bits, v_packed + (base + t) * rowb, ci);
      const float* sv = v_scales + (base + t) * ng;
      double p = S[t] / Z;
      for (int i = 0; i < d; ++i) orot[i] += p * ((double)sv[i / ORACLE_GROUP] * (double)C[ci[i]]);
    }
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += R[(int64_t)i * d + j] * orot[i];
      out[bh * d + j] = acc;
    }
    free(S);
  }
  free(R);
  return fail ? -2 : 0;
}

/* ------------------------------------------------------------------ */
/* unquantized attention, for the fidelity report only                  */
/* ------------------------------------------------------------------ */
/*
 * k, v: [B][Hkv][capacity][d] fp32/bf16 (the original vectors, unrotated).
 * out: [B][Hq][d] fp64 = softmax(attn_scale q k^T) v, in fp64.
 */
int oracle_exact_attention(const void* q, int q_dtype, const void* k, const void* v,
                           int kv_dtype, int B, int Hq, int Hkv, int d, int64_t capacity,
                           const int32_t* ctx_lens, double attn_scale, double* out,
                           int nthreads) {
  if (Hkv <= 0 || Hq % Hkv != 0) return -1;
  int G = Hq / Hkv;
  int64_t nrows = (int64_t)B * Hq;
  int fail = 0;
#ifdef _OPENMP
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
#endif
  for (int64_t bh = 0; bh < nrows; ++bh) {
    int64_t b = bh / Hq, hq = bh % Hq, hk = hq / G;
    int64_t T = ctx_lens[b];
    double* S = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!S) { fail = 1; continue; }
    int64_t base = ((int64_t)b * Hkv + hk) * capacity;
    double smax = -INFINITY;
    for (int64_t t = 0; t < T; ++t) {
      double dot = 0.0;
      for (int i = 0; i < d; ++i)
        dot += (double)load_input(q, q_dtype, bh * d + i) *
               (double)load_input(k, kv_dtype, (base + t) * d + i);
      S[t] = attn_scale * dot;
      if (S[t] > smax) smax = S[t];
    }
    double Z = 0.0;
    for (int64_t t = 0; t < T; ++t) { S[t] = exp(S[t] - smax); Z += S[t]; }
    for (int i = 0; i < d; ++i) {
      double acc = 0.0;
      for (int64_t t = 0; t < T; ++t) acc += S[t] * (double)load_input(v, kv_dtype, (base + t) * d + i);
      out[bh * d + i] = acc / Z;
    }
    free(S);
  }
  return fail ? -2 : 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
