// lq_gemv.cu -- small-batch +-1 contraction y = s . (b . z) over a precomputed z.
//
// Paper sec. 3 intro / review "Method": decode is an INT1 x FP product of the stored sign
// codes with the lifted activations, followed by the per-row scale diag(s). Each stored bit
// is the sign of the matching z entry, so a term is `z XOR (bit << 31)`; accumulation is
// fp32. Rows are split into K-slices; the last CTA of a row tile to finish sums the slices
// in slice order (a fixed order, no float atomics) and applies s.
#include "lq_internal.cuh"

namespace lq {

constexpr int kGemvThreads = 256;

__device__ __forceinline__ uint32_t ldg_stream(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

template <int TB>
__global__ void __launch_bounds__(kGemvThreads)
gemv_xor_kernel(const float* __restrict__ z, int64_t L, int batch,
                const uint32_t* __restrict__ packed, int64_t row_words, int N,
                const void* __restrict__ s, int sdt, float* __restrict__ y, int sw, int nsl,
                int rt, int ntiles, float* __restrict__ partials,
                uint32_t* __restrict__ counters) {
  extern __shared__ float zs[];          // [TB][32][sw + 1]: zs[t][m][w] = z[t][32*(w0+w) + m]
  const int pitch = sw + 1;
  const int sl = blockIdx.x, tile = blockIdx.y, tg = blockIdx.z;
  const int t0 = tg * TB;
  const int64_t data_words = (L + 31) / 32;
  const int64_t w0 = (int64_t)sl * sw;
  const int nw = (int)min((int64_t)sw, data_words - w0);

  for (int e = threadIdx.x; e < TB * 32 * sw; e += blockDim.x) {
    const int t = e / (32 * sw);
    const int ql = e - t * 32 * sw;
    const int w = ql >> 5, m = ql & 31;
    const int64_t q = 32 * w0 + ql;
    float v = 0.f;
    if (t0 + t < batch && q < L) v = z[(int64_t)(t0 + t) * L + q];
    zs[(t * 32 + m) * pitch + w] = v;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = tile * rt, row1 = min(N, row0 + rt);
  for (int row = row0 + warp; row < row1; row += kGemvThreads / 32) {
    float acc[TB];
#pragma unroll
    for (int t = 0; t < TB; ++t) acc[t] = 0.f;
    const uint32_t* prow = packed + (int64_t)row * row_words + w0;
    for (int w = lane; w < nw; w += 32) {
      const uint32_t bits = ldg_stream(prow + w);
      const float* zc = zs + w;
#pragma unroll
      for (int m = 0; m < 32; ++m) {
        const uint32_t sb = (bits << (31 - m)) & 0x80000000u;
#pragma unroll
        for (int t = 0; t < TB; ++t)
          acc[t] += __uint_as_float(__float_as_uint(zc[(t * 32 + m) * pitch]) ^ sb);
      }
    }
#pragma unroll
    for (int t = 0; t < TB; ++t)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
    if (lane == 0) {
#pragma unroll
      for (int t = 0; t < TB; ++t) {
        if (t0 + t >= batch) break;
        if (nsl == 1)
          y[(int64_t)(t0 + t) * N + row] = load_as_f32(s, sdt, row) * acc[t];
        else
          partials[((int64_t)sl * batch + t0 + t) * N + row] = acc[t];
      }
    }
  }
  if (nsl == 1) return;

  // Split-K completion: the last CTA of this (row tile, token group) reduces the slices.
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  uint32_t* ctr = counters + (int64_t)tg * ntiles + tile;
  if (threadIdx.x == 0) s_last = (atomicAdd(ctr, 1u) == (uint32_t)(nsl - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int nr = row1 - row0;
  for (int e = threadIdx.x; e < TB * nr; e += blockDim.x) {
    const int t = e / nr;
    const int row = row0 + (e - t * nr);
    if (t0 + t >= batch) continue;
    float acc = 0.f;
    for (int k = 0; k < nsl; ++k) acc += __ldcg(&partials[((int64_t)k * batch + t0 + t) * N + row]);
    y[(int64_t)(t0 + t) * N + row] = load_as_f32(s, sdt, row) * acc;
  }
  if (threadIdx.x == 0) *ctr = 0u;   // ready for the next call on this workspace
}

GemvPlan plan_gemv(int32_t batch, int64_t L, int32_t N) {
  GemvPlan p{};
  p.tb = batch <= 1 ? 1 : batch <= 2 ? 2 : batch <= 4 ? 4 : 8;
  p.ntg = (batch + p.tb - 1) / p.tb;
  p.sw = p.tb <= 2 ? 128 : p.tb == 4 ? 64 : 32;
  const int64_t data_words = (L + 31) / 32;
  p.nsl = (int)((data_words + p.sw - 1) / p.sw);
  p.rt = 64;
  p.ntiles = (N + p.rt - 1) / p.rt;
  p.smem = (size_t)p.tb * 32 * (p.sw + 1) * sizeof(float);
  return p;
}

template <int TB>
static cudaError_t launch_tb(const GemvPlan& p, const float* z, int64_t L, int32_t batch,
                             const uint32_t* packed, int64_t row_words, int32_t N,
                             const void* s, int sdt, float* y, float* partials,
                             uint32_t* counters, cudaStream_t st) {
  static int smem_set[64];
  cudaError_t e = ensure_smem((const void*)gemv_xor_kernel<TB>, p.smem, smem_set);
  if (e != cudaSuccess) return e;
  dim3 grid(p.nsl, p.ntiles, p.ntg);
  gemv_xor_kernel<TB><<<grid, kGemvThreads, p.smem, st>>>(z, L, batch, packed, row_words, N,
                                                          s, sdt, y, p.sw, p.nsl, p.rt,
                                                          p.ntiles, partials, counters);
  return cudaGetLastError();
}

cudaError_t launch_gemv(const GemvPlan& p, const float* z, int64_t L, int32_t batch,
                        const uint32_t* packed, int64_t row_words, int32_t N, const void* s,
                        int sdt, float* y, float* partials, uint32_t* counters,
                        cudaStream_t st) {
  switch (p.tb) {
    case 1: return launch_tb<1>(p, z, L, batch, packed, row_words, N, s, sdt, y, partials, counters, st);
    case 2: return launch_tb<2>(p, z, L, batch, packed, row_words, N, s, sdt, y, partials, counters, st);
    case 4: return launch_tb<4>(p, z, L, batch, packed, row_words, N, s, sdt, y, partials, counters, st);
    default: return launch_tb<8>(p, z, L, batch, packed, row_words, N, s, sdt, y, partials, counters, st);
  }
}

}  // namespace lq
