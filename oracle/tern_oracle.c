/*
 * tern_oracle.c -- plain CPU reference for the packed-ternary linear path.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the bench's CPU-baseline leg may load
 * or run this code. The product path (the CUDA library) never calls it, and this file shares no
 * code, header, table or constant generator with it.
 *
 * Everything here is the plain definition written out: nested loops, fp64 sums for bf16
 * activations, int64 sums for int8 activations, no blocking and no reordering beyond the
 * definition. Rows may be split across threads (each output is computed by one thread, start to
 * finish), which changes nothing in the arithmetic.
 *
 * What is computed. Sources are three of the pages about the Neutrino-1 ternary models, cited by
 * page and section heading:
 *   [R] the PyTorchKR review "Fermion Research, 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군
 *       3종 공개" (discuss.pytorch.kr/t/11456);
 *   [A] the aiatolah.com article "Neutrino-1 8B: modelo ternario de 3,88 GB roda em GPU e laptop";
 *   [O] the origotech.dev explainer "더 적은 비트로 계산하기" (lowbit).
 *   - the linear-layer contraction y_j = sum_i w_ij x_i ([R] "학습 중에 포맷이 있어야 하는 이유",
 *     displayed equation), with w in {-1, 0, +1} times a per-row scale;
 *   - ternary weights mean add / skip / subtract, no multiplies ([O] Figure I caption);
 *   - weights packed at rest and decoded inside the matrix kernels ([A] second paragraph and
 *     "Formato unico, tres portas");
 *   - the transport form of the ternary lane expands bit-exactly into the container ([R] "3진
 *     계열이라는 이름의 실체"; [A] "Formato unico"); the pages do not give its coder, so this
 *     library uses fixed-rate base 3, five trits per byte;
 *   - int8 activations (the 0.6B C runtime) and bf16 activations (the CLI default), fp32 output
 *     ([R] "토큰 동일성의 경계: 그리디, float32, 그리고 두 개의 근접 동점");
 *   - the int8 output head with greedy argmax ([R] "3진 계열이라는 이름의 실체": embeddings and
 *     head stay int8; [R] "토큰 동일성의 경계": near ties between implementations); the lowest
 *     index wins an exact tie;
 *   - the steps on either side of the linears in a Qwen3 block ([R] "세 모델과 하나의 컨테이너",
 *     model table: RMSNorm, SwiGLU): RMSNorm y = x / sqrt(mean(x^2) + eps) * gain, and
 *     SwiGLU h = silu(gate) * up with silu(z) = z / (1 + e^-z); both computed in fp64 from fp32
 *     inputs and rounded once to bf16, the activation type of the next linear;
 *   - the acceptance rule of speculative decoding ([R] "검증된 추측 디코딩: 속도만 바꾸고 답은
 *     바꾸지 않는다"): the target scores the k drafted positions in one pass and keeps the longest
 *     prefix of drafts that equal its own greedy choices, then adds its own next token.
 *
 * Packed layout (this library's own definition; the pages' FV5 planes are only partly described):
 *   row n of an N x K matrix (K % 128 == 0) occupies K/16 uint32 words starting at word n*K/16;
 *   words [0, K/32) are the nonzero-mask plane, words [K/32, K/16) the sign plane;
 *   trit k is in word k/32 of each plane; with j = k % 32 its mask bit is at position
 *   p(j) = 16*(j%2) + j/16 + 2*((j%16)/2) and its sign bit at position (p(j) + 1) % 32;
 *   mask bit = (t != 0), sign bit = (t == -1), so the sign bit is 0 wherever the mask bit is 0.
 * Transport layout: row n occupies ceil(K/5) bytes; byte j holds trits 5j..5j+4 as
 *   b = d0 + 3 d1 + 9 d2 + 27 d3 + 81 d4 with d_i = t_{5j+i} + 1; trits past K are t = 0 (d = 1)
 *   when encoding and are ignored when decoding; a byte above 242 is an error.
 *
 * Parity pins: every function here is checked against something other than itself in the CPU
 * test-suite (numpy brute force, closed forms, exhaustive small cases, hand-worked fixtures).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ----------------------------------------------------------------------------------------- */
/* number formats                                                                              */

/* IEEE binary16 -> double, from the format definition (sign, 5-bit exponent, 10-bit fraction). */
double orc_half_to_double(uint16_t h) {
  const int sign = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0) v = ldexp((double)m, -24);            /* subnormal: m * 2^-24            */
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp(1024.0 + (double)m, e - 25);       /* (1 + m/1024) * 2^(e-15)         */
  return sign ? -v : v;
}

/* bfloat16 -> float: the upper half of an IEEE binary32. */
float orc_bf16_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* double -> bfloat16, round to nearest, ties to even, in one step from the format definition
 * (sign, 8-bit exponent with bias 127, 7 fraction bits; subnormals are multiples of 2^-133). */
uint16_t orc_round_bf16(double v) {
  if (isnan(v)) return 0x7FC0;
  const uint16_t sign = signbit(v) ? 0x8000 : 0;
  const double a = fabs(v);
  if (a == 0.0) return sign;
  if (isinf(a)) return sign | 0x7F80;
  int ex;
  frexp(a, &ex);                        /* 2^(ex-1) <= a < 2^ex */
  int e = ex - 1;                       /* unbiased exponent of a */
  if (e < -126) e = -126;               /* subnormal range: the quantum stays 2^-133 */
  const double q = ldexp(1.0, e - 7);   /* spacing of bf16 values with this exponent */
  const double r = rint(a / q);         /* a / q is exact (power of two); rint: ties to even */
  /* r * q is the rounded magnitude; r = 256 carries into the next exponent, and a subnormal
   * that rounds up to 2^-126 (r = 128 at e = -126) lands on the smallest normal: in both cases the
   * encoding below, exponent field + fraction, gives the right bits. */
  uint32_t bits;
  if (r >= 128.0) bits = (uint32_t)(e + 127) * 128u + (uint32_t)(r - 128.0);
  else bits = (uint32_t)r;              /* subnormal (e == -126): fraction field = r */
  if (bits >= 0x7F80u) return sign | 0x7F80;   /* overflow to infinity */
  return sign | (uint16_t)bits;
}

/* ----------------------------------------------------------------------------------------- */
/* packed layout                                                                               */

static int mask_bit(int k) { const int j = k % 32; return 16 * (j % 2) + j / 16 + 2 * ((j % 16) / 2); }
static int sign_bit(int k) { return (mask_bit(k) + 1) % 32; }

int64_t orc_packed_words(int32_t N, int32_t K) { return (int64_t)N * (K / 16); }

/* Dense trits (int8, N x K, row-major) -> planes. Returns -1 on success, else the flat index of
 * the first trit outside {-1, 0, +1} (planes then hold an unspecified partial result). */
int64_t orc_pack(const int8_t* trits, int32_t N, int32_t K, uint32_t* planes) {
  const int kw = K / 32;
  memset(planes, 0, sizeof(uint32_t) * (size_t)orc_packed_words(N, K));
  for (int n = 0; n < N; ++n) {
    uint32_t* mask = planes + (size_t)n * (K / 16);
    uint32_t* sign = mask + kw;
    for (int k = 0; k < K; ++k) {
      const int8_t t = trits[(size_t)n * K + k];
      if (t != -1 && t != 0 && t != 1) return (int64_t)n * K + k;
      if (t != 0) mask[k / 32] |= 1u << mask_bit(k);
      if (t == -1) sign[k / 32] |= 1u << sign_bit(k);
    }
  }
  return -1;
}

/* One row of planes -> dense trits. A sign bit without its mask bit reads as 0 (never produced by
 * orc_pack). */
void orc_unpack_row(const uint32_t* planes, int32_t K, int32_t n, int8_t* out) {
  const uint32_t* mask = planes + (size_t)n * (K / 16);
  const uint32_t* sign = mask + K / 32;
  for (int k = 0; k < K; ++k) {
    const int m = (mask[k / 32] >> mask_bit(k)) & 1, s = (sign[k / 32] >> sign_bit(k)) & 1;
    out[k] = (int8_t)(m ? (s ? -1 : 1) : 0);
  }
}

void orc_unpack(const uint32_t* planes, int32_t N, int32_t K, int8_t* trits) {
  for (int n = 0; n < N; ++n) orc_unpack_row(planes, K, n, trits + (size_t)n * K);
}

/* Per-row occupancy: counts[3n+0] = zeros, [3n+1] = +1s, [3n+2] = -1s. */
void orc_occupancy(const uint32_t* planes, int32_t N, int32_t K, int64_t* counts) {
  int8_t* row = (int8_t*)malloc((size_t)K);
  for (int n = 0; n < N; ++n) {
    orc_unpack_row(planes, K, n, row);
    int64_t z = 0, p = 0, q = 0;
    for (int k = 0; k < K; ++k) { if (row[k] == 0) ++z; else if (row[k] == 1) ++p; else ++q; }
    counts[3 * n] = z; counts[3 * n + 1] = p; counts[3 * n + 2] = q;
  }
  free(row);
}

/* ----------------------------------------------------------------------------------------- */
/* base-3 transport                                                                            */

int32_t orc_base3_row_bytes(int32_t K) { return (K + 4) / 5; }

/* Returns -1 on success, else the flat index of the first trit outside {-1, 0, +1}. */
int64_t orc_base3_encode(const int8_t* trits, int32_t N, int32_t K, uint8_t* bytes) {
  const int nb = orc_base3_row_bytes(K);
  for (int n = 0; n < N; ++n) {
    for (int j = 0; j < nb; ++j) {
      int b = 0, w = 1;
      for (int i = 0; i < 5; ++i) {
        const int k = 5 * j + i;
        int d = 1;                                   /* padding past K: t = 0 */
        if (k < K) {
          const int8_t t = trits[(size_t)n * K + k];
          if (t != -1 && t != 0 && t != 1) return (int64_t)n * K + k;
          d = t + 1;
        }
        b += d * w;
        w *= 3;
      }
      bytes[(size_t)n * nb + j] = (uint8_t)b;
    }
  }
  return -1;
}

/* Returns -1 on success, else the flat index of the first byte above 242. */
int64_t orc_base3_decode(const uint8_t* bytes, int32_t N, int32_t K, int8_t* trits) {
  const int nb = orc_base3_row_bytes(K);
  for (int n = 0; n < N; ++n) {
    for (int j = 0; j < nb; ++j) {
      int b = bytes[(size_t)n * nb + j];
      if (b > 242) return (int64_t)n * nb + j;
      for (int i = 0; i < 5; ++i) {
        const int d = b % 3;
        b /= 3;
        const int k = 5 * j + i;
        if (k < K) trits[(size_t)n * K + k] = (int8_t)(d - 1);
      }
    }
  }
  return -1;
}

/* ----------------------------------------------------------------------------------------- */
/* threads: outputs split into contiguous ranges, one thread per range                         */

typedef void (*range_fn)(void* ctx, int64_t begin, int64_t end);
typedef struct { range_fn fn; void* ctx; int64_t b, e; } range_job;

static void* run_range(void* p) {
  range_job* j = (range_job*)p;
  j->fn(j->ctx, j->b, j->e);
  return NULL;
}

static void parallel_for(int64_t n, int nthreads, range_fn fn, void* ctx) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((int64_t)nthreads > n) nthreads = n > 0 ? (int)n : 1;
  if (nthreads == 1) { fn(ctx, 0, n); return; }
  pthread_t th[256];
  range_job jobs[256];
  for (int i = 0; i < nthreads; ++i) {
    jobs[i].fn = fn; jobs[i].ctx = ctx;
    jobs[i].b = n * i / nthreads; jobs[i].e = n * (i + 1) / nthreads;
    pthread_create(&th[i], NULL, run_range, &jobs[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
}

/* ----------------------------------------------------------------------------------------- */
/* bf16 activations: Y[m][n] = scale[n] * sum_k t[n][k] * X[m][k], all in fp64                  */

typedef struct {
  const uint32_t* planes; const uint16_t* scale; int32_t N, K, M; const uint16_t* X; double* Y;
} gemm_bf16_ctx;

static void gemm_bf16_rows(void* p, int64_t b, int64_t e) {
  gemm_bf16_ctx* c = (gemm_bf16_ctx*)p;
  int8_t* t = (int8_t*)malloc((size_t)c->K);
  for (int64_t n = b; n < e; ++n) {
    orc_unpack_row(c->planes, c->K, (int32_t)n, t);
    const double s = orc_half_to_double(c->scale[n]);
    for (int m = 0; m < c->M; ++m) {
      const uint16_t* x = c->X + (size_t)m * c->K;
      double acc = 0.0;
      for (int k = 0; k < c->K; ++k)
        if (t[k] != 0) acc += (double)t[k] * (double)orc_bf16_to_float(x[k]);   /* add / skip / subtract */
      c->Y[(size_t)m * c->N + n] = s * acc;
    }
  }
  free(t);
}

void orc_gemm_bf16(const uint32_t* planes, const uint16_t* scale, int32_t N, int32_t K, int32_t M,
                   const uint16_t* X, double* Y, int32_t nthreads) {
  gemm_bf16_ctx c = {planes, scale, N, K, M, X, Y};
  parallel_for(N, nthreads, gemm_bf16_rows, &c);
}

/* ----------------------------------------------------------------------------------------- */
/* int8 activations: per-token absmax quantisation, int64 accumulation, fp32 epilogue           */

/* s_x = absmax/127 (fp32 division); q = clamp(rint(x / s_x), -127, 127) with fp32 division and
 * round-half-to-even; an all-zero row gives s_x = 0 and q = 0. Finite inputs. */
void orc_quantize_act(const uint16_t* X, int32_t M, int32_t K, int8_t* Q, float* SX) {
  for (int m = 0; m < M; ++m) {
    const uint16_t* x = X + (size_t)m * K;
    float amax = 0.0f;
    for (int k = 0; k < K; ++k) {
      const float v = fabsf(orc_bf16_to_float(x[k]));
      if (v > amax) amax = v;
    }
    const float s = amax / 127.0f;
    SX[m] = s;
    for (int k = 0; k < K; ++k) {
      float r = 0.0f;
      if (s != 0.0f) {
        const float xs = orc_bf16_to_float(x[k]) / s;
        r = rintf(xs);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
      }
      Q[(size_t)m * K + k] = (int8_t)r;
    }
  }
}

typedef struct {
  const uint32_t* planes; const uint16_t* scale; int32_t N, K, M; const int8_t* Q; const float* SX;
  int64_t* ACC; float* Y;
} gemm_i8_ctx;

static void gemm_i8_rows(void* p, int64_t b, int64_t e) {
  gemm_i8_ctx* c = (gemm_i8_ctx*)p;
  int8_t* t = (int8_t*)malloc((size_t)c->K);
  for (int64_t n = b; n < e; ++n) {
    orc_unpack_row(c->planes, c->K, (int32_t)n, t);
    const float sw = (float)orc_half_to_double(c->scale[n]);          /* exact */
    for (int m = 0; m < c->M; ++m) {
      const int8_t* q = c->Q + (size_t)m * c->K;
      int64_t acc = 0;
      for (int k = 0; k < c->K; ++k)
        if (t[k] == 1) acc += q[k]; else if (t[k] == -1) acc -= q[k];
      if (c->ACC) c->ACC[(size_t)m * c->N + n] = acc;
      float y = (float)acc;            /* round to nearest */
      y = y * c->SX[m];                /* fp32 multiply #1 */
      y = y * sw;                      /* fp32 multiply #2 */
      c->Y[(size_t)m * c->N + n] = y;
    }
  }
  free(t);
}

void orc_gemm_i8(const uint32_t* planes, const uint16_t* scale, int32_t N, int32_t K, int32_t M,
                 const int8_t* Q, const float* SX, int64_t* ACC, float* Y, int32_t nthreads) {
  gemm_i8_ctx c = {planes, scale, N, K, M, Q, SX, ACC, Y};
  parallel_for(N, nthreads, gemm_i8_rows, &c);
}

/* ----------------------------------------------------------------------------------------- */
/* int8 output head with greedy argmax                                                         */

typedef struct {
  const int8_t* W; const uint16_t* SH; int32_t V, K, M; const uint16_t* X; double* L;
} head_bf16_ctx;

static void head_bf16_rows(void* p, int64_t b, int64_t e) {
  head_bf16_ctx* c = (head_bf16_ctx*)p;
  for (int64_t v = b; v < e; ++v) {
    const int8_t* w = c->W + (size_t)v * c->K;
    const double s = orc_half_to_double(c->SH[v]);
    for (int m = 0; m < c->M; ++m) {
      const uint16_t* x = c->X + (size_t)m * c->K;
      double acc = 0.0;
      for (int k = 0; k < c->K; ++k) acc += (double)w[k] * (double)orc_bf16_to_float(x[k]);
      c->L[(size_t)m * c->V + v] = s * acc;
    }
  }
}

/* logits[m][v] = s_h[v] * sum_k W[v][k] x[m][k] (fp64); argmax over v, lowest index on ties. */
void orc_head_bf16(const int8_t* W, const uint16_t* SH, int32_t V, int32_t K, int32_t M,
                   const uint16_t* X, double* LOGITS, int32_t* ARGMAX, double* MAXV, int32_t nthreads) {
  double* L = LOGITS ? LOGITS : (double*)malloc(sizeof(double) * (size_t)M * V);
  head_bf16_ctx c = {W, SH, V, K, M, X, L};
  parallel_for(V, nthreads, head_bf16_rows, &c);
  for (int m = 0; m < M; ++m) {
    int32_t best = 0;
    for (int32_t v = 1; v < V; ++v)
      if (L[(size_t)m * V + v] > L[(size_t)m * V + best]) best = v;
    ARGMAX[m] = best;
    MAXV[m] = L[(size_t)m * V + best];
  }
  if (!LOGITS) free(L);
}

typedef struct {
  const int8_t* W; const uint16_t* SH; int32_t V, K, M; const int8_t* Q; const float* SX; float* L;
} head_i8_ctx;

static void head_i8_rows(void* p, int64_t b, int64_t e) {
  head_i8_ctx* c = (head_i8_ctx*)p;
  for (int64_t v = b; v < e; ++v) {
    const int8_t* w = c->W + (size_t)v * c->K;
    const float sh = (float)orc_half_to_double(c->SH[v]);
    for (int m = 0; m < c->M; ++m) {
      const int8_t* q = c->Q + (size_t)m * c->K;
      int64_t acc = 0;
      for (int k = 0; k < c->K; ++k) acc += (int64_t)w[k] * q[k];
      float y = (float)acc;
      y = y * c->SX[m];
      y = y * sh;
      c->L[(size_t)m * c->V + v] = y;
    }
  }
}

void orc_head_i8(const int8_t* W, const uint16_t* SH, int32_t V, int32_t K, int32_t M,
                 const int8_t* Q, const float* SX, float* LOGITS, int32_t* ARGMAX, float* MAXV,
                 int32_t nthreads) {
  float* L = LOGITS ? LOGITS : (float*)malloc(sizeof(float) * (size_t)M * V);
  head_i8_ctx c = {W, SH, V, K, M, Q, SX, L};
  parallel_for(V, nthreads, head_i8_rows, &c);
  for (int m = 0; m < M; ++m) {
    int32_t best = 0;
    for (int32_t v = 1; v < V; ++v)
      if (L[(size_t)m * V + v] > L[(size_t)m * V + best]) best = v;
    ARGMAX[m] = best;
    MAXV[m] = L[(size_t)m * V + best];
  }
  if (!LOGITS) free(L);
}

/* ----------------------------------------------------------------------------------------- */
/* the steps on either side of the linears                                                     */

/* RMSNorm of each fp32 row x[m][0..K): r = 1 / sqrt(sum_k x_k^2 / K + eps) in fp64, then
 * out_k = bf16((x_k * r) * gain_k), the products in fp64 and one rounding to bf16. */
void orc_rmsnorm(const float* X, int32_t M, int32_t K, const uint16_t* gain_bf16, double eps, uint16_t* OUT) {
  for (int m = 0; m < M; ++m) {
    const float* x = X + (size_t)m * K;
    double ss = 0.0;
    for (int k = 0; k < K; ++k) ss += (double)x[k] * (double)x[k];
    const double r = 1.0 / sqrt(ss / (double)K + eps);
    for (int k = 0; k < K; ++k)
      OUT[(size_t)m * K + k] = orc_round_bf16(((double)x[k] * r) * (double)orc_bf16_to_float(gain_bf16[k]));
  }
}

/* SwiGLU of each row of a gate|up output GU[m][0..2K) (gate at k, up at K + k):
 * out_k = bf16(silu(g_k) * u_k), silu(z) = z / (1 + exp(-z)), all in fp64. */
void orc_swiglu(const float* GU, int32_t M, int32_t K, uint16_t* OUT) {
  for (int m = 0; m < M; ++m) {
    const float* g = GU + (size_t)m * 2 * K;
    const float* u = g + K;
    for (int k = 0; k < K; ++k) {
      const double z = (double)g[k];
      const double silu = z / (1.0 + exp(-z));
      OUT[(size_t)m * K + k] = orc_round_bf16(silu * (double)u[k]);
    }
  }
}

/* ----------------------------------------------------------------------------------------- */
/* speculative-verify acceptance                                                               */

/* The verify pass scores positions 0..k: argmax[j] is the target's greedy token after position
 * j, and draft[j] the drafted token for position j + 1. The accepted count n is the length of the
 * longest prefix with draft[j] == argmax[j]; the target then supplies argmax[n], so a round
 * yields n + 1 tokens. */
void orc_verify_accept(const int32_t* argmax, const int32_t* draft, int32_t k, int32_t* n_accept,
                       int32_t* next_token) {
  int32_t n = 0;
  while (n < k && draft[n] == argmax[n]) ++n;
  *n_accept = n;
  *next_token = argmax[n];
}

/* ----------------------------------------------------------------------------------------- */
/* order-0 entropy-coded transport (rANS)                                                      */
/*
 * The pages code the ternary lane for transport to within a hair of its order-0 coding bound
 * ([R] "3진 계열이라는 이름의 실체": the 0.6B container shrinks to within 0.007% of that bound)
 * but do not name the coder. This library's coder is byte-wise range asymmetric numeral systems
 * (rANS; J. Duda, "Asymmetric numeral systems: entropy coding combining speed of Huffman coding
 * with compression rate of arithmetic coding", 2013): one static frequency table per tensor and
 * one independent stream per row, so that rows decode in parallel.
 *   - Symbols: s = 0 for t = 0, 1 for t = +1, 2 for t = -1. Frequencies f_s >= 1 with
 *     f_0 + f_1 + f_2 = 4096 (12-bit precision); cum = (0, f_0, f_0 + f_1).
 *   - State x in [L, 256 L), L = 2^23. A row is encoded from its last trit to its first, starting
 *     from x = L: before each symbol, while x >= 2^19 * f_s, the low byte of x is emitted and x
 *     shifted right by 8; then x = (x / f_s) * 4096 + x % f_s + cum_s. The final x is emitted low
 *     byte first. The row's stream is all emitted bytes in reverse order (so it starts with x,
 *     most significant byte first).
 *   - Decoding reads a row's stream forward: x = its first four bytes (big-endian); per trit,
 *     slot = x % 4096, s = the symbol whose [cum_s, cum_s + f_s) holds slot,
 *     x = f_s * (x / 4096) + slot - cum_s, then while x < L: x = 256 x + next byte. A valid stream
 *     ends with x = L and every byte read.
 *   - Frequencies of a tensor: counts c_s over all its trits, f_s = max(1, floor(4096 c_s / total)),
 *     and 4096 - sum f added to the symbol with the largest count (the lowest s on ties).
 */

#define ORC_RANS_L (1u << 23)

void orc_rans_freqs(const int8_t* trits, int64_t n, uint16_t* freq) {
  int64_t c[3] = {0, 0, 0};
  for (int64_t i = 0; i < n; ++i) c[trits[i] == 0 ? 0 : (trits[i] == 1 ? 1 : 2)]++;
  int64_t f[3], sum = 0;
  int best = 0;
  for (int s = 0; s < 3; ++s) {
    f[s] = c[s] * 4096 / n;
    if (f[s] < 1) f[s] = 1;
    sum += f[s];
    if (c[s] > c[best]) best = s;
  }
  f[best] += 4096 - sum;
  for (int s = 0; s < 3; ++s) freq[s] = (uint16_t)f[s];
}

/* Encodes N rows of K trits; row n's stream ends at byte row_end[n] of out (rows back to back).
 * Returns the payload bytes, or -1 if cap is too small or a value is not a trit. */
int64_t orc_rans_encode(const int8_t* trits, int32_t N, int32_t K, const uint16_t* freq, uint32_t* row_end,
                        uint8_t* out, int64_t cap) {
  const uint32_t cum[3] = {0u, freq[0], (uint32_t)freq[0] + freq[1]};
  uint8_t* tmp = (uint8_t*)malloc((size_t)2 * K + 8);
  int64_t pos = 0;
  for (int32_t n = 0; n < N; ++n) {
    const int8_t* t = trits + (size_t)n * K;
    uint32_t x = ORC_RANS_L;
    int64_t e = 0;                                   /* bytes emitted, in emission order */
    for (int32_t k = K - 1; k >= 0; --k) {
      if (t[k] < -1 || t[k] > 1) { free(tmp); return -1; }
      const int s = t[k] == 0 ? 0 : (t[k] == 1 ? 1 : 2);
      const uint32_t f = freq[s];
      const uint64_t x_max = (uint64_t)(1u << 19) * f;
      while ((uint64_t)x >= x_max) { tmp[e++] = (uint8_t)(x & 255u); x >>= 8; }
      x = (x / f) * 4096u + x % f + cum[s];
    }
    for (int b = 0; b < 4; ++b) { tmp[e++] = (uint8_t)(x & 255u); x >>= 8; }
    if (pos + e > cap) { free(tmp); return -1; }
    for (int64_t i = 0; i < e; ++i) out[pos + i] = tmp[e - 1 - i];   /* reversed */
    pos += e;
    row_end[n] = (uint32_t)pos;
  }
  free(tmp);
  return pos;
}

/* Decodes the rows back into trits; returns 0, or -1 if any row's stream is not a valid one
 * (frequencies not summing to 4096, a read past the row's end, or a row not ending at x = L
 * with all its bytes read). */
int32_t orc_rans_decode(const uint8_t* payload, const uint32_t* row_end, int32_t N, int32_t K, const uint16_t* freq,
                        int8_t* trits) {
  if (freq[0] < 1 || freq[1] < 1 || freq[2] < 1 || (uint32_t)freq[0] + freq[1] + freq[2] != 4096u) return -1;
  const uint32_t cum[3] = {0u, freq[0], (uint32_t)freq[0] + freq[1]};
  int32_t status = 0;
  for (int32_t n = 0; n < N; ++n) {
    const uint32_t start = n ? row_end[n - 1] : 0u, end = row_end[n];
    int8_t* t = trits + (size_t)n * K;
    if (end < start || end - start < 4) { status = -1; memset(t, 0, (size_t)K); continue; }
    uint32_t p = start;
    uint32_t x = ((uint32_t)payload[p] << 24) | ((uint32_t)payload[p + 1] << 16) | ((uint32_t)payload[p + 2] << 8) |
                 payload[p + 3];
    p += 4;
    int ok = 1;
    for (int32_t k = 0; k < K; ++k) {
      const uint32_t slot = x & 4095u;
      const int s = slot < cum[1] ? 0 : (slot < cum[2] ? 1 : 2);
      t[k] = (int8_t)(s == 0 ? 0 : (s == 1 ? 1 : -1));
      x = freq[s] * (x >> 12) + slot - cum[s];
      while (x < ORC_RANS_L) {
        if (p >= end) { ok = 0; break; }
        x = (x << 8) | payload[p++];
      }
      if (!ok) break;
    }
    if (!ok || x != ORC_RANS_L || p != end) status = -1;
  }
  return status;
}

/* ----------------------------------------------------------------------------------------- */
/* five-valued blocks (FV5-style) and the block-scaled int8 head (FV5B-style)                  */
/*
 * The pages' shipped formats ([R] "FV5와 FV5B: llama.cpp 포크가 공개한 블록 구조", table): FV5
 * stores 256 weights per block as three 32-byte bitplanes plus fp32 s_lo and s_hi (3.25 bits per
 * weight), read as sign and zero plus two magnitude steps -- five states; FV5B stores 256 int8
 * weights per block with one fp32 scale. The pages do not give the plane semantics; this
 * library's reading:
 *   - a five-valued code c in {-2, -1, 0, +1, +2}; block b = weights 256b .. 256b + 255 of a row;
 *     weight w = 0 (c = 0), sign(c) * s_lo[b] (|c| = 1), sign(c) * s_hi[b] (|c| = 2);
 *   - planes of a row: mask (c != 0), sign (c < 0), magnitude (|c| = 2), each K/32 words with the
 *     ternary layout's bit order (mask and magnitude bit of in-word trit j at p(j), sign bit at
 *     (p(j) + 1) % 32); inside each group of 16 words (512 trits) of a plane, logical word
 *     w = 4e + t is stored at position 4t + e; row n = [mask | sign | magnitude], 3K/32 words;
 *   - scales: fp32 [N][K/256][2] = (s_lo, s_hi) per row and block; FV5B head: fp32 [V][K/256];
 *   - K is a multiple of 512 (whole groups of 16 words).
 * Products: bf16 mode in fp64 (the plain definition). int8 mode: per block the exact integer sums
 * A_lo, A_hi of sign * q over the block's |c| = 1 and |c| = 2 weights, then
 * y = fp32(s_x * sum_b (s_lo[b] A_lo[b] + s_hi[b] A_hi[b])), the sum in fp64 in block order, one
 * rounding to fp32.
 */

static int fv5_storage_word(int w) {          /* logical word w of a row plane -> stored word */
  const int g = w / 16, i = w % 16;
  return 16 * g + 4 * (i % 4) + i / 4;
}

int64_t orc_fv5_pack(const int8_t* codes, int32_t N, int32_t K, uint32_t* planes) {
  const int KW = K / 32;
  int64_t bad = 0;
  if (K % 512) return -1;
  memset(planes, 0, sizeof(uint32_t) * (size_t)N * 3 * KW);
  for (int32_t n = 0; n < N; ++n) {
    uint32_t* row = planes + (size_t)n * 3 * KW;
    for (int32_t k = 0; k < K; ++k) {
      const int c = codes[(size_t)n * K + k];
      if (c < -2 || c > 2) { ++bad; continue; }
      const int w = fv5_storage_word(k / 32);
      if (c != 0) row[w] |= 1u << mask_bit(k);
      if (c < 0) row[KW + w] |= 1u << sign_bit(k);
      if (c == 2 || c == -2) row[2 * KW + w] |= 1u << mask_bit(k);
    }
  }
  return bad;
}

void orc_fv5_unpack(const uint32_t* planes, int32_t N, int32_t K, int8_t* codes) {
  const int KW = K / 32;
  for (int32_t n = 0; n < N; ++n) {
    const uint32_t* row = planes + (size_t)n * 3 * KW;
    for (int32_t k = 0; k < K; ++k) {
      const int w = fv5_storage_word(k / 32);
      const int m = (row[w] >> mask_bit(k)) & 1, s = (row[KW + w] >> sign_bit(k)) & 1;
      const int g = (row[2 * KW + w] >> mask_bit(k)) & 1;
      codes[(size_t)n * K + k] = (int8_t)(m ? (s ? -1 : 1) * (g ? 2 : 1) : 0);
    }
  }
}

typedef struct {
  const uint32_t* planes; const float* scales; int32_t N, K, M; const uint16_t* X; double* Y;
} fv5_bf16_ctx;

static void fv5_bf16_rows(void* p, int64_t b, int64_t e) {
  fv5_bf16_ctx* c = (fv5_bf16_ctx*)p;
  int8_t* code = (int8_t*)malloc((size_t)c->K);
  for (int64_t n = b; n < e; ++n) {
    orc_fv5_unpack(c->planes + (size_t)n * 3 * (c->K / 32), 1, c->K, code);
    const float* sc = c->scales + (size_t)n * (c->K / 256) * 2;
    for (int m = 0; m < c->M; ++m) {
      const uint16_t* x = c->X + (size_t)m * c->K;
      double acc = 0.0;
      for (int k = 0; k < c->K; ++k) {
        const int cc = code[k];
        if (!cc) continue;
        const double w = (cc > 0 ? 1.0 : -1.0) * (double)sc[2 * (k / 256) + (cc == 2 || cc == -2)];
        acc += w * (double)orc_bf16_to_float(x[k]);
      }
      c->Y[(size_t)m * c->N + n] = acc;
    }
  }
  free(code);
}

void orc_fv5_gemm_bf16(const uint32_t* planes, const float* scales, int32_t N, int32_t K, int32_t M,
                       const uint16_t* X, double* Y, int32_t nthreads) {
  fv5_bf16_ctx c = {planes, scales, N, K, M, X, Y};
  parallel_for(N, nthreads, fv5_bf16_rows, &c);
}

typedef struct {
  const uint32_t* planes; const float* scales; int32_t N, K, M; const int8_t* Q; const float* SX; float* Y;
} fv5_i8_ctx;

static void fv5_i8_rows(void* p, int64_t b, int64_t e) {
  fv5_i8_ctx* c = (fv5_i8_ctx*)p;
  int8_t* code = (int8_t*)malloc((size_t)c->K);
  for (int64_t n = b; n < e; ++n) {
    orc_fv5_unpack(c->planes + (size_t)n * 3 * (c->K / 32), 1, c->K, code);
    const float* sc = c->scales + (size_t)n * (c->K / 256) * 2;
    for (int m = 0; m < c->M; ++m) {
      const int8_t* q = c->Q + (size_t)m * c->K;
      double tot = 0.0;
      for (int blk = 0; blk < c->K / 256; ++blk) {
        int64_t lo = 0, hi = 0;
        for (int k = 256 * blk; k < 256 * blk + 256; ++k) {
          const int cc = code[k];
          if (cc == 1) lo += q[k]; else if (cc == -1) lo -= q[k];
          else if (cc == 2) hi += q[k]; else if (cc == -2) hi -= q[k];
        }
        tot += (double)sc[2 * blk] * (double)lo + (double)sc[2 * blk + 1] * (double)hi;
      }
      c->Y[(size_t)m * c->N + n] = (float)((double)c->SX[m] * tot);
    }
  }
  free(code);
}

void orc_fv5_gemm_i8(const uint32_t* planes, const float* scales, int32_t N, int32_t K, int32_t M,
                     const int8_t* Q, const float* SX, float* Y, int32_t nthreads) {
  fv5_i8_ctx c = {planes, scales, N, K, M, Q, SX, Y};
  parallel_for(N, nthreads, fv5_i8_rows, &c);
}

/* FV5B-style head: logits[m][v] = sum_b s[v][b] * sum_{k in b} W[v][k] x[m][k]; argmax, lowest
 * index on exact ties. bf16 mode in fp64; int8 mode fp32(s_x * sum_b s_b A_b), fp64 sum in order. */
void orc_fv5b_head(const int8_t* W, const float* S, int32_t V, int32_t K, int32_t M, const uint16_t* X,
                   const int8_t* Q, const float* SX, double* LOGITS, int32_t* ARGMAX) {
  const int nb = K / 256;
  for (int m = 0; m < M; ++m) {
    for (int32_t v = 0; v < V; ++v) {
      const int8_t* w = W + (size_t)v * K;
      double tot = 0.0;
      for (int blk = 0; blk < nb; ++blk) {
        if (Q) {
          int64_t a = 0;
          for (int k = 256 * blk; k < 256 * blk + 256; ++k) a += (int64_t)w[k] * Q[(size_t)m * K + k];
          tot += (double)S[(size_t)v * nb + blk] * (double)a;
        } else {
          double a = 0.0;
          for (int k = 256 * blk; k < 256 * blk + 256; ++k)
            a += (double)w[k] * (double)orc_bf16_to_float(X[(size_t)m * K + k]);
          tot += (double)S[(size_t)v * nb + blk] * a;
        }
      }
      LOGITS[(size_t)m * V + v] = Q ? (double)(float)((double)SX[m] * tot) : tot;
    }
    int32_t best = 0;
    for (int32_t v = 1; v < V; ++v)
      if (LOGITS[(size_t)m * V + v] > LOGITS[(size_t)m * V + best]) best = v;
    ARGMAX[m] = best;
  }
}
