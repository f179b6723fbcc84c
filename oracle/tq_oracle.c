/*
 * tq_oracle.c -- plain CPU oracle for the W4A4 + low-rank linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct
 * definition the CUDA path is checked against.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
 * code, header, table or helper with the CUDA library, and the CUDA library
 * never calls it.
 *
 * Everything is fp64 (codes and accumulators are integers), loops are plain,
 * and there is no blocking, fusion or reordering beyond the definitions:
 *
 *   Xh   = X H                      rotation, CoQuant Eq. (3)
 *   s_x  = max_k |Xh[m,k]| / 7      symmetric scale, CoQuant Eq. (1) with
 *   q_x  = RoundClip(Xh / s_x)      N = 4 (2^(N-1)-1 = 7); TwinQuant notes,
 *                                   section 02 ("Integer quantization formula")
 *   Rh^T = R^T H, s_w, q_w          per-output-channel weights, same quantizer
 *                                   (CoQuant, experimental protocol:
 *                                   "per-channel symmetric ... for weights")
 *   acc  = sum_k q_x q_w            INT32 accumulation (TwinQuant notes,
 *                                   section 04.C, Figure 4)
 *   XL1  = X L1,  lr = bf16(XL1) L2 low-rank branch (TwinQuant notes,
 *                                   section 02.A, the U V term)
 *   Y    = s_x s_w acc + lr         single shared epilogue (TwinQuant notes,
 *                                   section 04.C; TwinQuant abstract)
 *
 * Readings where the pages are silent: H is the Sylvester Hadamard in natural
 * order normalised by 1/sqrt(b) with no random signs; "round to nearest" is
 * round-half-to-even; an all-zero row gets s = 0 and all codes 0; XL1 is
 * rounded to bf16 (round-to-nearest-even) before the up-projection.
 *
 * Parallelism: OpenMP over independent rows only (each output row is computed
 * by one thread with the same loop order as the serial code).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

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

static int popcount_u32(uint32_t v) {
  int c = 0;
  while (v) { c += (int)(v & 1u); v >>= 1; }
  return c;
}

/* Entry (i, j) of the normalised Sylvester Hadamard matrix of order b
 * (b a power of two): (-1)^{popcount(i & j)} / sqrt(b).  Its rows are
 * orthonormal, so it is an orthogonal U in the sense of CoQuant Eq. (3). */
double orc_hadamard_entry(int b, int i, int j) {
  double sgn = (popcount_u32((uint32_t)(i & j)) & 1) ? -1.0 : 1.0;
  return sgn / sqrt((double)b);
}

/* out = in * diag(H_b, ..., H_b) for each row of a [rows][K] matrix, K % b == 0.
 * Applied to X this is the online rotation X H; applied to the rows of R^T it
 * is (H^T R)^T, the offline rotation of the residual (CoQuant Eq. (3)). */
void orc_rotate(const double* in, long rows, long K, int b, double* out) {
  long nblk = K / b;
#pragma omp parallel for schedule(static)
  for (long m = 0; m < rows; ++m) {
    const double* x = in + m * K;
    double* y = out + m * K;
    for (long blk = 0; blk < nblk; ++blk) {
      for (int j = 0; j < b; ++j) {
        double acc = 0.0;
        for (int i = 0; i < b; ++i)
          acc += x[blk * b + i] * orc_hadamard_entry(b, i, j);
        y[blk * b + j] = acc;
      }
    }
  }
}

/* Asymmetric per-row quantizer of CoQuant Eq. (1) with a real zero-point
 * chosen from the row's range (the protocol's per-token asymmetric
 * activations): z = min(v), s = (max(v) - min(v)) / qmax,
 * q = RoundClip((v - z) / s) in [0, qmax], so that Q(v) = q s + z.
 * Round-to-nearest is half-to-even.  A constant row gets s = 0, all codes 0
 * and Q(v) = z exactly.  If t_out is not NULL it receives (v - z) / s. */
void orc_quantize_asym(const double* v, long rows, long K, int qmax,
                       uint8_t* q, double* s, double* z, double* t_out) {
#pragma omp parallel for schedule(static)
  for (long m = 0; m < rows; ++m) {
    const double* x = v + m * K;
    double lo = x[0], hi = x[0];
    for (long k = 1; k < K; ++k) {
      if (x[k] < lo) lo = x[k];
      if (x[k] > hi) hi = x[k];
    }
    z[m] = lo;
    if (hi == lo) {
      s[m] = 0.0;
      for (long k = 0; k < K; ++k) {
        q[m * K + k] = 0;
        if (t_out) t_out[m * K + k] = 0.0;
      }
      continue;
    }
    double scale = (hi - lo) / (double)qmax;
    s[m] = scale;
    for (long k = 0; k < K; ++k) {
      double t = (x[k] - lo) / scale;
      double r = nearbyint(t);
      if (r > qmax) r = qmax;
      if (r < 0) r = 0;
      q[m * K + k] = (uint8_t)r;
      if (t_out) t_out[m * K + k] = t;
    }
  }
}

/* Symmetric per-row quantizer of CoQuant Eq. (1) with zero-point 0:
 *   s = max|v| / qmax,  q = RoundClip(v / s) in [-qmax, qmax].
 * Round-to-nearest is half-to-even (nearbyint in the default rounding mode).
 * An all-zero row gets s = 0 and all codes 0.  If t_out is not NULL it
 * receives the unrounded value v / s that decided each code. */
void orc_quantize_sym(const double* v, long rows, long K, int qmax,
                      int8_t* q, double* s, double* t_out) {
#pragma omp parallel for schedule(static)
  for (long m = 0; m < rows; ++m) {
    const double* x = v + m * K;
    double amax = 0.0;
    for (long k = 0; k < K; ++k) {
      double a = fabs(x[k]);
      if (a > amax) amax = a;
    }
    if (amax == 0.0) {
      s[m] = 0.0;
      for (long k = 0; k < K; ++k) {
        q[m * K + k] = 0;
        if (t_out) t_out[m * K + k] = 0.0;
      }
      continue;
    }
    double scale = amax / (double)qmax;
    s[m] = scale;
    for (long k = 0; k < K; ++k) {
      double t = x[k] / scale;
      double r = nearbyint(t);
      if (r > qmax) r = qmax;
      if (r < -qmax) r = -qmax;
      q[m * K + k] = (int8_t)r;
      if (t_out) t_out[m * K + k] = t;
    }
  }
}

/* Packed int4 storage of a [rows][K] code matrix (K % 32 == 0) as
 * [rows][K/2] bytes: within every group of 32 consecutive codes
 * (16 bytes), byte i holds code i in its low nibble and code i+16 in its high
 * nibble, each as a 4-bit two's complement number. */
void orc_pack_int4(const int8_t* q, long rows, long K, uint8_t* out) {
  for (long m = 0; m < rows; ++m) {
    for (long g = 0; g < K / 32; ++g) {
      for (int i = 0; i < 16; ++i) {
        int lo = q[m * K + g * 32 + i];
        int hi = q[m * K + g * 32 + 16 + i];
        out[m * (K / 2) + g * 16 + i] =
            (uint8_t)(((unsigned)lo & 0xFu) | (((unsigned)hi & 0xFu) << 4));
      }
    }
  }
}

void orc_unpack_int4(const uint8_t* in, long rows, long K, int8_t* q) {
  for (long m = 0; m < rows; ++m) {
    for (long g = 0; g < K / 32; ++g) {
      for (int i = 0; i < 16; ++i) {
        unsigned byte = in[m * (K / 2) + g * 16 + i];
        int lo = (int)(byte & 0xFu);
        int hi = (int)((byte >> 4) & 0xFu);
        if (lo >= 8) lo -= 16;
        if (hi >= 8) hi -= 16;
        q[m * K + g * 32 + i] = (int8_t)lo;
        q[m * K + g * 32 + 16 + i] = (int8_t)hi;
      }
    }
  }
}

/* acc[m][n] = sum_k qa[m][k] * qb[n][k] in int64 (both operands K-contiguous).
 * Returns the number of entries whose magnitude exceeds 49*K or does not fit
 * in a signed 32-bit integer (the INT32 accumulator of TwinQuant, Figure 4). */
long orc_int_gemm(const int8_t* qa, const int8_t* qb, long M, long N, long K,
                  int64_t* acc) {
  long bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad)
  for (long m = 0; m < M; ++m) {
    for (long n = 0; n < N; ++n) {
      int64_t a = 0;
      for (long k = 0; k < K; ++k)
        a += (int64_t)qa[m * K + k] * (int64_t)qb[n * K + k];
      acc[m * N + n] = a;
      if (a > 49 * K || a < -49 * K || a > INT32_MAX || a < INT32_MIN) ++bad;
    }
  }
  return bad;
}

/* Round an fp64 value to the nearest bfloat16 (8 significant bits, 8-bit
 * exponent), ties to even, returned as fp64. */
double orc_round_bf16(double x) {
  if (x == 0.0 || isnan(x) || isinf(x)) return x;
  int e;
  (void)frexp(x, &e);                   /* x = m 2^e, 0.5 <= |m| < 1 */
  int qexp = e - 8;                     /* quantum of an 8-bit significand */
  if (qexp < -133) qexp = -133;         /* bf16 subnormal spacing 2^-133 */
  double t = ldexp(x, -qexp);
  double r = nearbyint(t);
  double y = ldexp(r, qexp);
  const double max_bf16 = ldexp(255.0, 120); /* (2 - 2^-7) 2^127 */
  if (y > max_bf16) return INFINITY;
  if (y < -max_bf16) return -INFINITY;
  return y;
}

/* Low-rank branch of the SVDQuant-style split (TwinQuant notes, 02.A):
 *   XL1[m][j] = sum_k X[m][k] L1t[j][k]
 *   lr[m][n]  = sum_j rnd(XL1[m][j]) L2t[n][j]
 * with rnd = bf16 round-to-nearest-even if round_mid, else identity. */
void orc_lowrank(const double* X, const double* L1t, const double* L2t,
                 long M, long N, long K, long r, int round_mid,
                 double* XL1, double* lr) {
#pragma omp parallel for schedule(static)
  for (long m = 0; m < M; ++m) {
    for (long j = 0; j < r; ++j) {
      double a = 0.0;
      for (long k = 0; k < K; ++k) a += X[m * K + k] * L1t[j * K + k];
      XL1[m * r + j] = a;
    }
    for (long n = 0; n < N; ++n) {
      double a = 0.0;
      for (long j = 0; j < r; ++j) {
        double u = round_mid ? orc_round_bf16(XL1[m * r + j]) : XL1[m * r + j];
        a += u * L2t[n * r + j];
      }
      lr[m * N + n] = a;
    }
  }
}

/* Shared epilogue: Y[m][n] = s_x[m] s_w[n] acc[m][n] + lr[m][n] (lr may be
 * NULL for rank 0). */
void orc_epilogue(const double* s_x, const double* s_w, const int64_t* acc,
                  const double* lr, long M, long N, double* Y) {
#pragma omp parallel for schedule(static)
  for (long m = 0; m < M; ++m)
    for (long n = 0; n < N; ++n)
      Y[m * N + n] = s_x[m] * s_w[n] * (double)acc[m * N + n] +
                     (lr ? lr[m * N + n] : 0.0);
}
