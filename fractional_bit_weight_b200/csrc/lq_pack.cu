// lq_pack.cu -- sign codes <-> LQ_FORMAT_V1 rows (offline step; not on the decode path).
//
// Paper (sec. 3.1): every length-d block is w ~= M w_q with w_q in {+1,-1}^D; the D signs of
// block g of row n are stored as bits g*D .. g*D+D-1 of the row, a set bit meaning -1 (the
// value of the IEEE sign bit of the +-1 it stands for).
#include "lq_internal.cuh"

namespace lq {

// One thread per output word: gathers 32 codes with a warp-wide coalesced read pattern
// (consecutive threads read consecutive 32-byte runs of the same row).
__global__ void pack_kernel(const int8_t* __restrict__ b, int32_t N, int64_t L, int64_t words,
                            uint32_t* __restrict__ packed) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)N * words) return;
  const int64_t n = idx / words;
  const int64_t w = idx - n * words;
  const int8_t* row = b + n * L;
  uint32_t v = 0;
  const int64_t q0 = w * 32;
#pragma unroll 8
  for (int i = 0; i < 32; ++i) {
    const int64_t q = q0 + i;
    if (q < L && row[q] < 0) v |= 1u << i;
  }
  packed[idx] = v;
}

__global__ void unpack_kernel(const uint32_t* __restrict__ packed, int32_t N, int64_t L,
                              int64_t words, int8_t* __restrict__ b) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)N * L) return;
  const int64_t n = idx / L;
  const int64_t q = idx - n * L;
  const uint32_t v = packed[n * words + (q >> 5)];
  b[idx] = ((v >> (q & 31)) & 1u) ? int8_t(-1) : int8_t(1);
}

static unsigned grid_for(int64_t n, int threads) {
  return (unsigned)((n + threads - 1) / threads);
}

cudaError_t launch_pack(const int8_t* b, int32_t N, int64_t L, int64_t words, uint32_t* packed,
                        cudaStream_t st) {
  const int64_t n = (int64_t)N * words;
  if (n == 0) return cudaSuccess;
  pack_kernel<<<grid_for(n, 256), 256, 0, st>>>(b, N, L, words, packed);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const uint32_t* packed, int32_t N, int64_t L, int64_t words,
                          int8_t* b, cudaStream_t st) {
  const int64_t n = (int64_t)N * L;
  if (n == 0) return cudaSuccess;
  unpack_kernel<<<grid_for(n, 256), 256, 0, st>>>(packed, N, L, words, b);
  return cudaGetLastError();
}

}  // namespace lq
