// lq_device.cuh -- device helpers shared by the liblq kernels (not part of the ABI).
#pragma once

#include "lq_internal.cuh"

namespace lq {

// v[r] = x[i0 + min(r, E - 1)] as fp32 for r < 8, all eight loads issued before the first use
__device__ __forceinline__ void load8_as_f32(const void* p, int dt, int64_t i0, int E,
                                             float (&v)[8]) {
  if (dt == LQ_BF16) {
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(p) + i0;
    __nv_bfloat16 h[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) h[r] = q[min(r, E - 1)];
#pragma unroll
    for (int r = 0; r < 8; ++r) v[r] = __bfloat162float(h[r]);
  } else if (dt == LQ_F16) {
    const __half* q = static_cast<const __half*>(p) + i0;
    __half h[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) h[r] = q[min(r, E - 1)];
#pragma unroll
    for (int r = 0; r < 8; ++r) v[r] = __half2float(h[r]);
  } else {
    const float* q = static_cast<const float*>(p) + i0;
#pragma unroll
    for (int r = 0; r < 8; ++r) v[r] = q[min(r, E - 1)];
  }
}

// One warp whitens one Hadamard block of Bh = 32*E inputs (1 <= E <= 8): the inputs
// [k0, k0 + Bh) of the row that starts at element row_off of x. Lane l holds inputs
// k0 + E*l + r (r < E). Every load of the lane is issued before the first use (indices past E
// repeat the last element and are discarded), the first log2(E) butterfly stages run in
// registers and the last five across lanes, on all eight registers at once so that the
// shuffles overlap. The lane's E outputs, times mul, go to out[E*l + r].
__device__ __forceinline__ void warp_whiten_block(const void* x, int xdt, int64_t row_off, int k0,
                                                  int E, const Whiten& T, float mul, float* out) {
  const int lane = threadIdx.x & 31;
  const int kl = k0 + E * lane;
  float v[8], cs[8];
  int8_t sg[8];
  load8_as_f32(x, xdt, row_off + kl, E, v);
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int k = kl + min(r, E - 1);
    cs[r] = T.chan_scale ? T.chan_scale[k] : 1.f;
    sg[r] = T.sign ? T.sign[k] : (int8_t)1;
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    v[r] *= cs[r];
    if (sg[r] < 0) v[r] = -v[r];
  }
#pragma unroll
  for (int h = 1; h < 8; h <<= 1)
    if (h < E)
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < E && (r & h) == 0) {
          const float a = v[r], c = v[r + h];
          v[r] = a + c;
          v[r + h] = a - c;
        }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
    float o[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) o[r] = __shfl_xor_sync(0xffffffffu, v[r], m);
#pragma unroll
    for (int r = 0; r < 8; ++r) v[r] = upper ? o[r] - v[r] : v[r] + o[r];
  }
#pragma unroll
  for (int r = 0; r < 8; ++r)
    if (r < E) out[E * lane + r] = v[r] * mul;
}


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
