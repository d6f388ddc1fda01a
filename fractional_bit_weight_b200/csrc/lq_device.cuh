// lq_device.cuh -- device helpers shared by the liblq kernels (not part of the ABI).
#pragma once

#include "lq_internal.cuh"

namespace lq {

// Whitens Hadamard blocks [blk0, blk0 + nblk) of one input row into sm[0 .. nblk*Bh).
// All threads of the CTA take part; ends with a barrier.
__device__ __forceinline__ void whiten_blocks_smem(const void* __restrict__ x, int xdt, int64_t row_off, int K,
                                   const Whiten& T, int blk0, int nblk, float* sm) {
  const int Bh = T.block;
  const int n = nblk * Bh;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int k = blk0 * Bh + i;
    float v = 0.f;
    if (k < K) {
      v = load_as_f32(x, xdt, row_off + k);
      if (T.chan_scale) v *= T.chan_scale[k];
      if (T.sign && T.sign[k] < 0) v = -v;
    }
    sm[i] = v;
  }
  __syncthreads();
  for (int h = 1; h < Bh; h <<= 1) {
    for (int p = threadIdx.x; p < n / 2; p += blockDim.x) {
      const int lo = p & (h - 1);
      const int i = ((p - lo) << 1) | lo;  // bit h of i is clear; partner is i + h
      const float a = sm[i], b = sm[i + h];
      sm[i] = a + b;
      sm[i + h] = a - b;
    }
    __syncthreads();
  }
  if (T.inv_sqrt != 1.f) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) sm[i] *= T.inv_sqrt;
    __syncthreads();
  }
}

}  // namespace lq
