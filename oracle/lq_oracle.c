/*
 * lq_oracle.c -- plain, slow, fp64 CPU oracle for the LiftQuant decode operator.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may build, load or call this file. The library under
 * fractional_bit_weight_b200/ never does, and shares no code, header, table or
 * constant with it.
 *
 * What it computes (sources are the pages on LiftQuant):
 *   - "LiftQuant: Continuous Bit-Width LLM Quantization via Dimensional Lifting
 *     and Projection" (paper translation, bittide.aicompass.dev), sec. 3.1:
 *     every length-d weight block is w ~= M * w_q with w_q in {+1,-1}^D and
 *     w_i = sum_j M_ij (w_q)_j; M is the d x D mapping matrix.
 *   - same paper, sec. 3 (intro) and sec. 2: the bit-width is D/d and the
 *     fused decode operator is o = diag(s) W (M T a).
 *   - "Paper Review: LiftQuant" (romaanj.github.io), "Method": decode is
 *     diag(s) * W_q * (T* a) with T* the lift fused with the whitening T,
 *     and T is Hadamard-initialised orthogonal mixing plus scalings.
 *
 * Readings taken where the pages are silent (each is listed in the design notes):
 *   - T acts on contiguous blocks of Bh inputs: xt = H_Bh (sigma . c . x) / sqrt(Bh),
 *     H in Sylvester (natural) order, H[i][j] = (-1)^popcount(i & j);
 *     Bh = 0 means T is the identity.
 *   - K is zero-padded up to G*d (G = ceil(K/d)) after T.
 *   - Bitstream LQ_FORMAT_V1: row n, block g, lifted coordinate j is bit
 *     q = g*D + j of the row; bit q lives in byte q/8 at bit position q%8
 *     (LSB first); a set bit means w_q = -1; each row is zero-padded to a
 *     multiple of 16 bytes.
 *
 * Everything below is written as the plain definition: explicit dense H, an
 * explicit weight row W[n][.] = blockwise M * b, and an fp64 dot product.
 * Threads (OpenMP) split output rows only; each row is computed by one thread
 * in a fixed order, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- sizes */

/* Number of length-d blocks in a row of K inputs (K zero-padded to G*d). */
static int64_t orc_groups(int32_t K, int32_t d) { return ((int64_t)K + d - 1) / d; }

static int orc_valid_code(int32_t K, int32_t d, int32_t D) {
  return K >= 1 && d >= 1 && D >= d && D <= 32;
}

/* Lifted length of a row = number of stored bits = G*D. */
int64_t orc_lifted_bits(int32_t K, int32_t d, int32_t D) {
  if (!orc_valid_code(K, d, D)) return -1;
  return orc_groups(K, d) * D;
}

/* Bytes per stored row: ceil(G*D / 8) rounded up to a multiple of 16. */
int64_t orc_row_bytes(int32_t K, int32_t d, int32_t D) {
  int64_t bits = orc_lifted_bits(K, d, D);
  if (bits < 0) return -1;
  int64_t bytes = (bits + 7) / 8;
  return (bytes + 15) / 16 * 16;
}

/* ---------------------------------------------------------------- packing */

/* b: [N][G*D] int8 entries in {+1,-1}; out: [N][row_bytes] bytes.
 * Returns 0, or -1 if an entry of b is not +1/-1 or the sizes are invalid. */
int orc_pack(const int8_t* b, int64_t N, int32_t K, int32_t d, int32_t D, uint8_t* out) {
  int64_t bits = orc_lifted_bits(K, d, D);
  int64_t rb = orc_row_bytes(K, d, D);
  if (bits < 0 || N < 0) return -1;
  memset(out, 0, (size_t)(N * rb));
  for (int64_t n = 0; n < N; ++n) {
    const int8_t* br = b + n * bits;
    uint8_t* orow = out + n * rb;
    for (int64_t q = 0; q < bits; ++q) {
      if (br[q] == -1) {
        orow[q / 8] |= (uint8_t)(1u << (q % 8));
      } else if (br[q] != 1) {
        return -1;
      }
    }
  }
  return 0;
}

/* Inverse of orc_pack. Padding bits are ignored. */
int orc_unpack(const uint8_t* packed, int64_t N, int32_t K, int32_t d, int32_t D, int8_t* b) {
  int64_t bits = orc_lifted_bits(K, d, D);
  int64_t rb = orc_row_bytes(K, d, D);
  if (bits < 0 || N < 0) return -1;
  for (int64_t n = 0; n < N; ++n) {
    const uint8_t* prow = packed + n * rb;
    for (int64_t q = 0; q < bits; ++q) {
      int bit = (prow[q / 8] >> (q % 8)) & 1;
      b[n * bits + q] = bit ? (int8_t)-1 : (int8_t)1;
    }
  }
  return 0;
}

/* ---------------------------------------------------------------- whitening */

static int orc_parity(uint32_t v) {
  int p = 0;
  while (v) {
    p ^= (int)(v & 1u);
    v >>= 1;
  }
  return p;
}

/* Entry (i, j) of the Sylvester-ordered Hadamard matrix. */
static double orc_hadamard_entry(int32_t i, int32_t j) {
  return orc_parity((uint32_t)(i & j)) ? -1.0 : 1.0;
}

static int orc_is_pow2(int32_t v) { return v > 0 && (v & (v - 1)) == 0; }

/* xt[t][k] = T(x[t])[k] for batch rows of K inputs.
 * sign: [K] entries +1/-1 or NULL (all +1); chan_scale: [K] or NULL (all 1).
 * block = 0: T is the identity (sign and chan_scale unused).
 * Returns 0, or -1 on invalid sizes. Dense O(K * block) per row, on purpose. */
int orc_whiten(const double* x, int64_t batch, int32_t K, const int8_t* sign,
               const double* chan_scale, int32_t block, double* xt) {
  if (K < 1 || batch < 0) return -1;
  if (block == 0) {
    memcpy(xt, x, (size_t)(batch * K) * sizeof(double));
    return 0;
  }
  if (!orc_is_pow2(block) || K % block != 0) return -1;
  const double norm = 1.0 / sqrt((double)block);
  double* u = (double*)malloc((size_t)block * sizeof(double));
  if (!u) return -1;
  for (int64_t t = 0; t < batch; ++t) {
    const double* xr = x + t * K;
    double* yr = xt + t * K;
    for (int32_t b0 = 0; b0 < K; b0 += block) {
      for (int32_t j = 0; j < block; ++j) {
        double v = xr[b0 + j];
        if (chan_scale) v *= chan_scale[b0 + j];
        if (sign) v *= (double)sign[b0 + j];
        u[j] = v;
      }
      for (int32_t i = 0; i < block; ++i) {
        double acc = 0.0;
        for (int32_t j = 0; j < block; ++j) acc += orc_hadamard_entry(i, j) * u[j];
        yr[b0 + i] = acc * norm;
      }
    }
  }
  free(u);
  return 0;
}

/* ---------------------------------------------------------------- lift */

/* z[t][g*D + j] = sum_i M[i][j] * xt[t][g*d + i], with xt zero beyond K.
 * This is the lifted activation (M^T applied per block), computed after T.
 * M: [d][D] row-major. z: [batch][G*D]. */
int orc_lift(const double* x, int64_t batch, int32_t K, const int8_t* sign,
             const double* chan_scale, int32_t block, const double* M, int32_t d, int32_t D,
             double* z) {
  if (!orc_valid_code(K, d, D) || batch < 0) return -1;
  const int64_t G = orc_groups(K, d);
  double* xt = (double*)malloc((size_t)(batch * K) * sizeof(double));
  if (!xt) return -1;
  if (orc_whiten(x, batch, K, sign, chan_scale, block, xt) != 0) {
    free(xt);
    return -1;
  }
  for (int64_t t = 0; t < batch; ++t) {
    for (int64_t g = 0; g < G; ++g) {
      for (int32_t j = 0; j < D; ++j) {
        double acc = 0.0;
        for (int32_t i = 0; i < d; ++i) {
          int64_t k = g * d + i;
          double v = (k < K) ? xt[t * K + k] : 0.0;
          acc += M[i * D + j] * v;
        }
        z[t * G * D + g * D + j] = acc;
      }
    }
  }
  free(xt);
  return 0;
}

/* ---------------------------------------------------------------- forward */

/* y[t][n] = s[n] * sum_{k<K} W[n][k] * T(x[t])[k], with W[n][g*d+i] = sum_j M[i][j] b[n][g][j]
 * and b unpacked from the LQ_FORMAT_V1 rows in `packed` ([nrows][row_bytes]).
 * s: [nrows]. y: [batch][nrows]. nthreads <= 0 means one thread.
 * This forms each weight row explicitly, the plain definition of the operator. */
int orc_forward(const double* x, int64_t batch, int32_t K, int64_t nrows, int32_t d, int32_t D,
                const uint8_t* packed, const double* M, const double* s, const int8_t* sign,
                const double* chan_scale, int32_t block, double* y, int nthreads) {
  if (!orc_valid_code(K, d, D) || batch < 0 || nrows < 0) return -1;
  const int64_t G = orc_groups(K, d);
  const int64_t bits = G * D;
  const int64_t rb = orc_row_bytes(K, d, D);
  double* xt = (double*)malloc((size_t)(batch * K + 1) * sizeof(double));
  if (!xt) return -1;
  if (orc_whiten(x, batch, K, sign, chan_scale, block, xt) != 0) {
    free(xt);
    return -1;
  }
  int failed = 0;
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel num_threads(nthreads)
  {
    int8_t* br = (int8_t*)malloc((size_t)bits);
    double* w = (double*)malloc((size_t)(G * d) * sizeof(double));
    if (!br || !w) {
#pragma omp atomic write
      failed = 1;
    }
#pragma omp for schedule(static)
    for (int64_t n = 0; n < nrows; ++n) {
      if (!br || !w) continue;
      orc_unpack(packed + n * rb, 1, K, d, D, br);
      for (int64_t g = 0; g < G; ++g) {
        for (int32_t i = 0; i < d; ++i) {
          double acc = 0.0;
          for (int32_t j = 0; j < D; ++j) acc += M[i * D + j] * (double)br[g * D + j];
          w[g * d + i] = acc;
        }
      }
      for (int64_t t = 0; t < batch; ++t) {
        double acc = 0.0;
        for (int32_t k = 0; k < K; ++k) acc += w[k] * xt[t * K + k];
        y[t * nrows + n] = s[n] * acc;
      }
    }
    free(br);
    free(w);
  }
  free(xt);
  return failed ? -1 : 0;
}

/* Same operator in the lifted form: y[t][n] = s[n] * sum_q b[n][q] * z[t][q], with z from
 * orc_lift. Used to check the identity b^T (M^T x) = (M b)^T x against orc_forward. */
int orc_forward_lifted(const double* x, int64_t batch, int32_t K, int64_t nrows, int32_t d,
                       int32_t D, const uint8_t* packed, const double* M, const double* s,
                       const int8_t* sign, const double* chan_scale, int32_t block, double* y,
                       int nthreads) {
  if (!orc_valid_code(K, d, D) || batch < 0 || nrows < 0) return -1;
  const int64_t bits = orc_lifted_bits(K, d, D);
  const int64_t rb = orc_row_bytes(K, d, D);
  double* z = (double*)malloc((size_t)(batch * bits + 1) * sizeof(double));
  if (!z) return -1;
  if (orc_lift(x, batch, K, sign, chan_scale, block, M, d, D, z) != 0) {
    free(z);
    return -1;
  }
  int failed = 0;
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel num_threads(nthreads)
  {
    int8_t* br = (int8_t*)malloc((size_t)bits);
    if (!br) {
#pragma omp atomic write
      failed = 1;
    }
#pragma omp for schedule(static)
    for (int64_t n = 0; n < nrows; ++n) {
      if (!br) continue;
      orc_unpack(packed + n * rb, 1, K, d, D, br);
      for (int64_t t = 0; t < batch; ++t) {
        double acc = 0.0;
        for (int64_t q = 0; q < bits; ++q) acc += (double)br[q] * z[t * bits + q];
        y[t * nrows + n] = s[n] * acc;
      }
    }
    free(br);
  }
  free(z);
  return failed ? -1 : 0;
}

/* ---------------------------------------------------------------- encoder */

/* Nearest codeword by exhaustive search, the inner minimisation of Eq. (1) of the paper:
 * argmin over b in {+1,-1}^D of || w - M b ||^2, w in R^d.
 * Codeword c has b_j = -1 exactly when bit j of c is set; ties keep the smallest c.
 * b_out: [D]. Returns the codeword index c, or -1 if D > 24 or sizes are invalid. */
int64_t orc_encode_bruteforce(const double* w, const double* M, int32_t d, int32_t D,
                              int8_t* b_out) {
  if (d < 1 || D < 1 || D > 24) return -1;
  int64_t best = -1;
  double best_dist = 0.0;
  for (int64_t c = 0; c < ((int64_t)1 << D); ++c) {
    double dist = 0.0;
    for (int32_t i = 0; i < d; ++i) {
      double r = w[i];
      for (int32_t j = 0; j < D; ++j) r -= M[i * D + j] * (((c >> j) & 1) ? -1.0 : 1.0);
      dist += r * r;
    }
    if (best < 0 || dist < best_dist) {
      best = c;
      best_dist = dist;
    }
  }
  for (int32_t j = 0; j < D; ++j) b_out[j] = ((best >> j) & 1) ? (int8_t)-1 : (int8_t)1;
  return best;
}

/* Squared distance || w - M b ||^2 of the block w (length d) to the codeword b (length D). */
static double orc_block_dist(const double* w, const double* M, int32_t d, int32_t D,
                             const int8_t* b) {
  double dist = 0.0;
  for (int32_t i = 0; i < d; ++i) {
    double r = w[i];
    for (int32_t j = 0; j < D; ++j) r -= M[i * D + j] * (double)b[j];
    dist += r * r;
  }
  return dist;
}

/* Seeded search, the review's "pseudo-inverse initialisation" that cuts the 2^D search of
 * Eq. (1) to 2^(D-d) (romaanj.github.io review, "Method"; the cap D - d <= 20 is in its
 * "Limitations"). Reading (the pages give no more): the first d coordinates are solved, the
 * other D - d are enumerated. For every f in [0, 2^(D-d)), b_{d+k} = -1 exactly when bit k of
 * f is set; r = w - sum_{j>=d} M[:,j] b_j; u solves M_S u = r with M_S = M[:, 0..d) (Gaussian
 * elimination with partial pivoting); b_i = +1 when u_i >= 0, else -1 (i < d). The candidate
 * with the smallest || w - M b ||^2 wins, ties keeping the smallest f. Writes b_out [D] and the
 * distance; returns f, or -1 for invalid sizes or a singular M_S. */
int64_t orc_encode_seeded(const double* w, const double* M, int32_t d, int32_t D, int8_t* b_out,
                          double* dist_out) {
  if (d < 1 || D < d || D > 32 || D - d > 24) return -1;
  const int32_t F = D - d;
  double* A = (double*)malloc(sizeof(double) * (size_t)d * (size_t)(d + 1));
  int8_t* b = (int8_t*)malloc((size_t)D);
  if (!A || !b) {
    free(A);
    free(b);
    return -1;
  }
  int64_t best = -1;
  double best_dist = 0.0;
  int singular = 0;
  for (int64_t f = 0; f < ((int64_t)1 << F) && !singular; ++f) {
    for (int32_t k = 0; k < F; ++k) b[d + k] = ((f >> k) & 1) ? (int8_t)-1 : (int8_t)1;
    /* augmented system [M_S | r] */
    for (int32_t i = 0; i < d; ++i) {
      double r = w[i];
      for (int32_t k = 0; k < F; ++k) r -= M[i * D + d + k] * (double)b[d + k];
      for (int32_t c = 0; c < d; ++c) A[i * (d + 1) + c] = M[i * D + c];
      A[i * (d + 1) + d] = r;
    }
    for (int32_t c = 0; c < d; ++c) {               /* forward elimination */
      int32_t piv = c;
      for (int32_t i = c + 1; i < d; ++i)
        if (fabs(A[i * (d + 1) + c]) > fabs(A[piv * (d + 1) + c])) piv = i;
      if (A[piv * (d + 1) + c] == 0.0) {
        singular = 1;
        break;
      }
      if (piv != c)
        for (int32_t k = 0; k <= d; ++k) {
          const double t = A[c * (d + 1) + k];
          A[c * (d + 1) + k] = A[piv * (d + 1) + k];
          A[piv * (d + 1) + k] = t;
        }
      for (int32_t i = c + 1; i < d; ++i) {
        const double m = A[i * (d + 1) + c] / A[c * (d + 1) + c];
        for (int32_t k = c; k <= d; ++k) A[i * (d + 1) + k] -= m * A[c * (d + 1) + k];
      }
    }
    if (singular) break;
    for (int32_t c = d - 1; c >= 0; --c) {          /* back substitution: u into column d */
      double u = A[c * (d + 1) + d];
      for (int32_t k = c + 1; k < d; ++k) u -= A[c * (d + 1) + k] * A[k * (d + 1) + d];
      u /= A[c * (d + 1) + c];
      A[c * (d + 1) + d] = u;
      b[c] = u >= 0.0 ? (int8_t)1 : (int8_t)-1;
    }
    const double dist = orc_block_dist(w, M, d, D, b);
    if (dist < best_dist || best < 0) {
      best = f;
      best_dist = dist;
      memcpy(b_out, b, (size_t)D);
    }
  }
  free(A);
  free(b);
  if (singular) return -1;
  if (dist_out) *dist_out = best_dist;
  return best;
}

/* Encodes a weight matrix w [N][K] block by block (K zero-padded to G*d): b [N][G][D] in
 * {+1,-1} and err [N][G] = || w_block - M b ||^2. mode 0: exhaustive search over all 2^D
 * codewords; mode 1: the seeded search above. Blocks are independent; threads split rows.
 * Returns 0, or -1 if a block was rejected. */
int orc_encode_rows(const double* w, int64_t N, int32_t K, const double* M, int32_t d, int32_t D,
                    int32_t mode, int8_t* b, double* err, int nthreads) {
  if (N < 0 || K < 1 || d < 1 || D < d || D > 32 || (mode != 0 && mode != 1)) return -1;
  if (mode == 0 && D > 24) return -1;
  const int64_t G = orc_groups(K, d);
  int failed = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static) reduction(| : failed)
#endif
  for (int64_t n = 0; n < N; ++n) {
    double blk[64];
    for (int64_t g = 0; g < G; ++g) {
      for (int32_t i = 0; i < d; ++i) {
        const int64_t k = g * d + i;
        blk[i] = k < K ? w[n * K + k] : 0.0;
      }
      int8_t* bo = b + (n * G + g) * D;
      double dist = 0.0;
      int64_t r;
      if (mode == 0) {
        r = orc_encode_bruteforce(blk, M, d, D, bo);
        if (r >= 0) dist = orc_block_dist(blk, M, d, D, bo);
      } else {
        r = orc_encode_seeded(blk, M, d, D, bo, &dist);
      }
      if (r < 0) failed = 1;
      if (err) err[n * G + g] = dist;
    }
  }
  (void)nthreads;
  return failed ? -1 : 0;
}

/* The least-squares step of the codebook fit (review "Method": M is fitted offline to a
 * standard Gaussian; paper sec. 3.1, Eq. (1)): with the codes b_s of the samples w_s [S][d]
 * fixed, M [d][D] becomes M = (sum_s w_s b_s^T)(sum_s b_s b_s^T)^-1, the point where the
 * straight-through gradient -2 sum_s (w_s - M b_s) b_s^T vanishes. Sums run in sample order in
 * fp64; the D x D system is solved by elimination with partial pivoting. Returns 0, or -1 for
 * invalid sizes or a singular sum b b^T (M is then left unchanged). */
int orc_codebook_refit(const double* w, int64_t S, const int8_t* b, double* M, int32_t d,
                       int32_t D) {
  if (S < 1 || d < 1 || D < d || D > 32) return -1;
  double* A = (double*)calloc((size_t)d * (size_t)D, sizeof(double));
  double* C = (double*)calloc((size_t)D * (size_t)(D + d), sizeof(double));
  if (!A || !C) {
    free(A);
    free(C);
    return -1;
  }
  int rc = 0;
  /* sums in sample order: A = sum w b^T [d][D]; the system C^T X = A^T with C = sum b b^T,
   * stored augmented as [D][D + d] */
  for (int64_t n = 0; n < S; ++n) {
    const int8_t* bn = b + n * D;
    for (int32_t i = 0; i < d; ++i)
      for (int32_t j = 0; j < D; ++j) A[i * D + j] += w[n * d + i] * (double)bn[j];
    for (int32_t j = 0; j < D; ++j)
      for (int32_t k = 0; k < D; ++k) C[j * (D + d) + k] += (double)bn[j] * (double)bn[k];
  }
  for (int32_t j = 0; j < D; ++j)
    for (int32_t i = 0; i < d; ++i) C[j * (D + d) + D + i] = A[i * D + j];
  /* C is symmetric: solve C X = A^T (X = M^T) by elimination with partial pivoting */
  const int32_t W = D + d;
  for (int32_t c = 0; c < D && rc == 0; ++c) {
    int32_t piv = c;
    for (int32_t r = c + 1; r < D; ++r)
      if (fabs(C[r * W + c]) > fabs(C[piv * W + c])) piv = r;
    if (fabs(C[piv * W + c]) < 1e-12 * (double)S) {
      rc = -1;
      break;
    }
    if (piv != c)
      for (int32_t k = 0; k < W; ++k) {
        const double t = C[c * W + k];
        C[c * W + k] = C[piv * W + k];
        C[piv * W + k] = t;
      }
    for (int32_t r = c + 1; r < D; ++r) {
      const double m = C[r * W + c] / C[c * W + c];
      for (int32_t k = c; k < W; ++k) C[r * W + k] -= m * C[c * W + k];
    }
  }
  if (rc == 0) {
    for (int32_t i = 0; i < d; ++i)
      for (int32_t c = D - 1; c >= 0; --c) {
        double x = C[c * W + D + i];
        for (int32_t k = c + 1; k < D; ++k) x -= C[c * W + k] * C[k * W + D + i];
        x /= C[c * W + c];
        C[c * W + D + i] = x;            /* X[c][i] = M[i][c] */
      }
    for (int32_t i = 0; i < d; ++i)
      for (int32_t c = 0; c < D; ++c) M[i * D + c] = C[c * W + D + i];
  }
  free(A);
  free(C);
  return rc;
}

/* One round of the codebook optimisation: M is fitted offline to a standard Gaussian (review
 * "Method"; paper sec. 3.1, Eq. (1), whose text is cut before the gradient path through the
 * encoder). Reading: alternating minimisation of the mean of ||w - M b(w)||^2 over samples
 * w_s [S][d]: (1) every sample takes its nearest codeword under the current M (mode 0
 * exhaustive, 1 seeded); (2) with the codes fixed, M becomes the least-squares fit
 * (orc_codebook_refit). M [d][D] is updated in place; b_out [S][D] (optional) receives the
 * codes of step (1). Returns the mean squared error per weight of step (1), or -1 for invalid
 * input or a singular sum b b^T (M is then left unchanged). */
double orc_codebook_round(const double* w, int64_t S, double* M, int32_t d, int32_t D,
                          int32_t mode, int8_t* b_out, int nthreads) {
  if (S < 1 || d < 1 || D < d || D > 24 || (mode != 0 && mode != 1)) return -1.0;
  int8_t* b = b_out ? b_out : (int8_t*)malloc((size_t)S * (size_t)D);
  double* err = (double*)malloc(sizeof(double) * (size_t)S);
  if (!b || !err) {
    if (!b_out) free(b);
    free(err);
    return -1.0;
  }
  int failed = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static) reduction(| : failed)
#endif
  for (int64_t n = 0; n < S; ++n) {
    int8_t* bn = b + n * D;
    const int64_t r = mode == 0 ? orc_encode_bruteforce(w + n * d, M, d, D, bn)
                                : orc_encode_seeded(w + n * d, M, d, D, bn, NULL);
    if (r < 0) failed = 1;
    err[n] = r < 0 ? 0.0 : orc_block_dist(w + n * d, M, d, D, bn);
  }
  (void)nthreads;
  double mse = -1.0;
  if (!failed) {
    double tot = 0.0;
    for (int64_t n = 0; n < S; ++n) tot += err[n];
    mse = tot / ((double)S * d);
    if (orc_codebook_refit(w, S, b, M, d, D) != 0) mse = -1.0;
  }
  if (!b_out) free(b);
  free(err);
  return mse;
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
