// lq_codebook.cu -- one round of the offline codebook fit on the GPU.
//
// The review's "Method" fits the projection M offline to a standard Gaussian; the paper's
// sec. 3.1, Eq. (1) writes the objective M* = argmin E ||w - M b*(w)||^2 with b*(w) the
// nearest codeword (its text stops before the gradient path through the encoder). Reading: one
// round of alternating minimisation over samples w_s [S][d]:
//   (1) b_s = nearest codeword of w_s under M (the lq_encode search, exact or seeded);
//   (2) with the codes fixed, M = (sum_s w_s b_s^T)(sum_s b_s b_s^T)^-1, the least-squares fit,
//       where the straight-through gradient -2 sum_s (w_s - M b_s) b_s^T vanishes.
// Kernels: the encoder (lq_encode.cu); cb_sums_kernel, one CTA per contiguous range of samples,
// which stages the range's samples and codes in shared memory and accumulates A = sum w b^T in
// fp64 and C = sum b b^T exactly in int64 (one thread per entry, samples in order); and
// cb_solve_kernel, one CTA, which adds the CTA partials in CTA order, solves C M^T = A^T by
// Gaussian elimination with partial pivoting in fp64 and writes M (fp32) and the mean squared
// error of step (1). Every sum has a fixed order: the result does not depend on timing.
#include "lq_device.cuh"

namespace lq {
namespace cb {

constexpr int kThreads = 512;
constexpr int kTile = 256;      // samples staged per pass
constexpr int kMaxD = 32;

// partials of one CTA: A [d][D] (fp64), C [D][D] (int64), sum of err (fp64)
__global__ void __launch_bounds__(kThreads)
    cb_sums_kernel(const float* __restrict__ w, int64_t S, const int8_t* __restrict__ b,
                   const float* __restrict__ err, int d, int D, int64_t per_cta,
                   double* __restrict__ pA, long long* __restrict__ pC, double* __restrict__ pE) {
  __shared__ float sw[kTile * 16];
  __shared__ int8_t sb[kTile * kMaxD];
  __shared__ double sred[kThreads / 32];
  const int tid = threadIdx.x;
  const int64_t s0 = (int64_t)blockIdx.x * per_cta;
  const int64_t s1 = min(S, s0 + per_cta);
  const int nA = d * D, nC = D * D;
  double acc_a[2] = {0.0, 0.0};
  long long acc_c[2] = {0, 0};
  double e = 0.0;
  for (int64_t t0 = s0; t0 < s1; t0 += kTile) {
    const int nt = (int)min((int64_t)kTile, s1 - t0);
    __syncthreads();
    for (int i = tid; i < nt * d; i += kThreads) sw[i] = w[t0 * d + i];
    for (int i = tid; i < nt * D; i += kThreads) sb[i] = b[t0 * D + i];
    for (int i = tid; i < nt; i += kThreads) e += (double)err[t0 + i];
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int ea = tid + r * kThreads;
      if (ea < nA) {
        const int i = ea / D, j = ea - i * D;
        double a = acc_a[r];
        for (int s = 0; s < nt; ++s) a += (double)sw[s * d + i] * (double)sb[s * D + j];
        acc_a[r] = a;
      }
      if (ea < nC) {
        const int j = ea / D, k = ea - j * D;
        long long c = acc_c[r];
        for (int s = 0; s < nt; ++s) c += (int)sb[s * D + j] * (int)sb[s * D + k];
        acc_c[r] = c;
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int ea = tid + r * kThreads;
    if (ea < nA) pA[(int64_t)blockIdx.x * nA + ea] = acc_a[r];
    if (ea < nC) pC[(int64_t)blockIdx.x * nC + ea] = acc_c[r];
  }
  // the error sum: per thread in sample order, then over threads in thread order
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
  if ((tid & 31) == 0) sred[tid >> 5] = e;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int i = 0; i < kThreads / 32; ++i) t += sred[i];
    pE[blockIdx.x] = t;
  }
}

// One CTA: partials summed in CTA order, then the D x D solve; M is left unchanged (and mse
// set to -1) when sum b b^T is singular.
__global__ void __launch_bounds__(kThreads)
    cb_solve_kernel(const double* __restrict__ pA, const long long* __restrict__ pC,
                    const double* __restrict__ pE, int nparts, int64_t S, int d, int D,
                    float* __restrict__ M, double* __restrict__ mse_out) {
  __shared__ double aug[kMaxD][kMaxD + 17];   // [D][D + d]: C | A^T
  __shared__ int s_piv;
  __shared__ int s_bad;
  const int tid = threadIdx.x;
  const int Wd = D + d;
  for (int ea = tid; ea < D * D; ea += kThreads) {
    long long c = 0;
    for (int p = 0; p < nparts; ++p) c += pC[(int64_t)p * D * D + ea];
    aug[ea / D][ea % D] = (double)c;
  }
  for (int ea = tid; ea < d * D; ea += kThreads) {
    double a = 0.0;
    for (int p = 0; p < nparts; ++p) a += pA[(int64_t)p * d * D + ea];
    const int i = ea / D, j = ea - i * D;
    aug[j][D + i] = a;
  }
  if (tid == 0) {
    s_bad = 0;
    double e = 0.0;
    for (int p = 0; p < nparts; ++p) e += pE[p];
    if (mse_out) *mse_out = e / ((double)S * d);
  }
  __syncthreads();
  for (int c = 0; c < D; ++c) {
    if (tid == 0) {
      int piv = c;
      for (int r = c + 1; r < D; ++r)
        if (fabs(aug[r][c]) > fabs(aug[piv][c])) piv = r;
      s_piv = piv;
      if (fabs(aug[piv][c]) < 1e-12 * (double)S) s_bad = 1;
    }
    __syncthreads();
    if (s_bad) break;
    const int piv = s_piv;
    if (piv != c)
      for (int k = tid; k < Wd; k += kThreads) {
        const double t = aug[c][k];
        aug[c][k] = aug[piv][k];
        aug[piv][k] = t;
      }
    __syncthreads();
    // rows below c: r = c + 1 + tid / Wd, column k = tid % Wd (k >= c)
    for (int e = tid; e < (D - c - 1) * Wd; e += kThreads) {
      const int r = c + 1 + e / Wd, k = e % Wd;
      if (k > c) aug[r][k] -= aug[r][c] / aug[c][c] * aug[c][k];
    }
    __syncthreads();
    for (int r = c + 1 + tid; r < D; r += kThreads) aug[r][c] = 0.0;
    __syncthreads();
  }
  if (s_bad) {
    if (tid == 0 && mse_out) *mse_out = -1.0;
    return;
  }
  // back substitution, one thread per right-hand side i: X[c][i] = M[i][c]
  if (tid < d) {
    const int i = tid;
    for (int c = D - 1; c >= 0; --c) {
      double x = aug[c][D + i];
      for (int k = c + 1; k < D; ++k) x -= aug[c][k] * aug[k][D + i];
      x /= aug[c][c];
      aug[c][D + i] = x;
    }
  }
  __syncthreads();
  for (int ea = tid; ea < d * D; ea += kThreads) {
    const int i = ea / D, c = ea - i * D;
    M[ea] = (float)aug[c][D + i];
  }
}

}  // namespace cb

size_t codebook_partials(int64_t S) {
  return (size_t)std::max<int64_t>(1, std::min<int64_t>(4 * 148, (S + 1023) / 1024));
}

cudaError_t launch_codebook_round(const float* w, int64_t S, float* M, int32_t d, int32_t D,
                                  int32_t mode, int8_t* b, float* err, double* pA, long long* pC,
                                  double* pE, double* mse, cudaStream_t st) {
  cudaError_t e = launch_encode(w, S, d, M, d, D, mode, b, err, st);
  if (e != cudaSuccess) return e;
  const int64_t parts = (int64_t)codebook_partials(S);
  const int64_t per = (S + parts - 1) / parts;
  const int nparts = (int)((S + per - 1) / per);
  cb::cb_sums_kernel<<<nparts, cb::kThreads, 0, st>>>(w, S, b, err, d, D, per, pA, pC, pE);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cb::cb_solve_kernel<<<1, cb::kThreads, 0, st>>>(pA, pC, pE, nparts, S, d, D, M, mse);
  return cudaGetLastError();
}

}  // namespace lq
