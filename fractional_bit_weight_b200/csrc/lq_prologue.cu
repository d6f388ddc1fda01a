// lq_prologue.cu -- the whitening T and the lift z = blockdiag(M^T) T(x).
//
// T (romaanj.github.io review, "Method": Hadamard-initialised orthogonal mixing plus
// scalings): on each contiguous block of Bh inputs, xt = H_Bh (sign . chan_scale . x) / sqrt(Bh)
// with H in Sylvester order. It is computed here as an in-place fast Walsh-Hadamard
// transform (log2 Bh butterfly stages) in shared memory.
// Lift (paper sec. 3 intro: o = diag(s) W (M T a); review: T* = lift o T):
// z[g*D + j] = sum_{i<d} M[i][j] xt[g*d + i], xt zero beyond K.
#include "lq_device.cuh"

namespace lq {

// One CTA per (Hadamard block, token).
__global__ void whiten_kernel(const void* __restrict__ x, int xdt, int K, Whiten T,
                              float* __restrict__ xt) {
  extern __shared__ float sm[];
  const int t = blockIdx.y;
  const int64_t row = (int64_t)t * K;
  if (T.block == 0) {
    // identity: one CTA per 1024-input chunk
    const int k0 = blockIdx.x * 1024;
    for (int i = threadIdx.x; i < 1024 && k0 + i < K; i += blockDim.x)
      xt[row + k0 + i] = load_as_f32(x, xdt, row + k0 + i);
    return;
  }
  whiten_blocks_smem(x, xdt, row, K, T, blockIdx.x, 1, sm);
  const int k0 = blockIdx.x * T.block;
  for (int i = threadIdx.x; i < T.block; i += blockDim.x) xt[row + k0 + i] = sm[i];
}

// One CTA per (chunk of gpc blocks of d inputs, token). Writes z fp32 [batch][G*D].
__global__ void lift_f32_kernel(const void* __restrict__ x, int xdt, int K, Whiten T,
                                const float* __restrict__ M, int d, int D, int G, int gpc,
                                float* __restrict__ z, uint32_t* __restrict__ zero_ptr,
                                int zero_words) {
  extern __shared__ float sm[];
  float* sM = sm;                  // [d][D], at most LQ_MAX_D * LQ_MAX_D floats
  float* sx = sm + LQ_MAX_D * LQ_MAX_D;
  const int t = blockIdx.y;
  const int64_t row = (int64_t)t * K;
  if (zero_ptr && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < zero_words; i += blockDim.x) zero_ptr[i] = 0u;
  for (int i = threadIdx.x; i < d * D; i += blockDim.x) sM[i] = M[i];
  const int g0 = blockIdx.x * gpc;
  const int g1 = min(G, g0 + gpc);
  const int k0 = g0 * d;
  const int k1 = min(g1 * d, K);
  int base;
  if (T.block > 0) {
    const int b0 = k0 / T.block;
    const int b1 = (k1 + T.block - 1) / T.block;
    base = b0 * T.block;
    whiten_blocks_smem(x, xdt, row, K, T, b0, b1 - b0, sx);  // ends with a barrier
  } else {
    base = k0;
    for (int i = threadIdx.x; i < k1 - k0; i += blockDim.x)
      sx[i] = load_as_f32(x, xdt, row + k0 + i);
    __syncthreads();
  }
  const int ne = (g1 - g0) * D;
  float* zrow = z + (int64_t)t * G * D;
  for (int e = threadIdx.x; e < ne; e += blockDim.x) {
    const int gl = e / D;
    const int j = e - gl * D;
    const int g = g0 + gl;
    float acc = 0.f;
    for (int i = 0; i < d; ++i) {
      const int k = g * d + i;
      const float v = (k < K) ? sx[k - base] : 0.f;
      acc = fmaf(sM[i * D + j], v, acc);
    }
    zrow[(int64_t)g * D + j] = acc;
  }
}

cudaError_t ensure_smem(const void* func, size_t bytes, int* cache_per_device) {
  if (bytes == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache_per_device[dev] >= (int)bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) cache_per_device[dev] = (int)bytes;
  return e;
}

cudaError_t launch_whiten(const void* x, int xdt, int32_t batch, int32_t K, Whiten T,
                          float* xt, cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  if (T.block == 0) {
    dim3 grid((K + 1023) / 1024, batch);
    whiten_kernel<<<grid, 256, 0, st>>>(x, xdt, K, T, xt);
  } else {
    dim3 grid(K / T.block, batch);
    const int threads = T.block >= 512 ? 512 : (T.block >= 64 ? T.block / 2 : 32);
    whiten_kernel<<<grid, threads, T.block * sizeof(float), st>>>(x, xdt, K, T, xt);
  }
  return cudaGetLastError();
}

cudaError_t launch_lift_f32(const void* x, int xdt, int32_t batch, int32_t K, Whiten T,
                            const float* M, int32_t d, int32_t D, float* z, uint32_t* zero_ptr,
                            int32_t zero_words, cudaStream_t st) {
  const int G = (K + d - 1) / d;
  const int gpc = d >= 1024 ? 1 : 1024 / d;   // about 1024 inputs per CTA
  const int span = gpc * d;
  int sx_floats;
  if (T.block > 0)
    sx_floats = ((span - 1) / T.block + 2) * T.block;
  else
    sx_floats = span;
  const size_t smem = (size_t)(LQ_MAX_D * LQ_MAX_D + sx_floats) * sizeof(float);
  static int smem_set[64];
  cudaError_t e = ensure_smem((const void*)lift_f32_kernel, smem, smem_set);
  if (e != cudaSuccess) return e;
  dim3 grid((G + gpc - 1) / gpc, batch);
  lift_f32_kernel<<<grid, 256, smem, st>>>(x, xdt, K, T, M, d, D, G, gpc, z, zero_ptr,
                                           zero_words);
  return cudaGetLastError();
}

}  // namespace lq
