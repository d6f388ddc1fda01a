// lq_gemm_dq.cu -- the large-batch path of lq_gemm that dequantises the weights once per call:
// W = blockwise M b in fp16 (paper sec. 3.1: w ~= M w_q with w_q in {-1,+1}^D, per block of d
// weights), then a dense 5th-generation tensor-core GEMM of T(x) against W.
//
// The lifted form (lq_gemm_tc.cu) contracts over L = ceil(K/d) * D coordinates; this form over
// Kp = ceil(K/d) * d, D/d (2.4 for LQ-24/10) times fewer MMA flops, at the price of writing and
// reading W once (2 bytes per weight). Three kernels:
//
//  * dq_weights_kernel: W[n][g*d + i] = sum_j M[i][j] b[n][g][j] for every block g of every
//    row, on the legacy tensor cores (mma.m16n8k16, fp32 accumulation): A holds the +-1 codes of
//    sixteen blocks (rows), exact in fp16, B is M^T (columns i) rounded to fp16.
//    The rounding of M adds at most 2^-12 of each |M[i][j]| to a sum of D such terms, about as
//    much as the final rounding of W to fp16 (relative 2^-12); with the fp16 rounding of T(x)
//    the expected relative error of y is ~3e-4, against the 2e-3 tolerance. Columns from Kp to
//    the padded width Kw are written as zero.
//  * xt_f16_kernel (one CTA per token): whitening T, then fp16 xt * 2^e with a power of two 2^e
//    that maps max |xt| to at most 2^14, zero from K to Kw.
//  * gemm_dq_kernel (persistent, one CTA per SM): 128-token x 256-row output tiles, token tile
//    fastest (a wave of CTAs shares a few W tiles in L2); one warp loads both operands with TMA
//    (128-byte swizzle, no multicast), one thread issues tcgen05.mma into two 128 x 256 fp32
//    accumulators in tensor memory, four warps read them back with tcgen05.ld and apply 2^-e
//    and s[n].
// Every wait on an mbarrier is bounded in time: on expiry the kernel records LQ_ETIMEOUT in the
// workspace status word, the roles leave their loops, in-flight copies and MMAs are waited for
// (again bounded) and tensor memory is released before the CTA exits.
#include <cuda.h>

#include "lq_device.cuh"
#include "lq_sm100.cuh"

namespace lq {
namespace dq {

using namespace lq::sm100;

constexpr int BM = 128;                     // tokens per tile
constexpr int BN = 256;                     // weight rows per tile
constexpr int BK = 64;                      // inputs per stage: one 128-byte fp16 row
constexpr int UK = 16;                      // K of one kind::f16 MMA
constexpr int NSTAGE = 4;
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int B_BYTES = BN * BK * 2;        // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kEpiWarps = 4;
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 6 * 32;
constexpr int kTmemCols = 2 * BN;
constexpr uint64_t kWaitNs = 2000000000ull;

struct Ctl {
  uint64_t full[NSTAGE];
  uint64_t empty[NSTAGE];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = 1024 + (size_t)NSTAGE * STAGE_BYTES + sizeof(Ctl);

struct DqArgs {
  const float* inv_scale;
  const void* s;
  float* y;
  uint32_t* status;
  int N, batch, nks, tiles_m, tiles, sdt, vec_store;
};

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __noinline__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile int* abort,
                                        bool honor_abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (honor_abort && *abort) return false;
    if (globaltimer() - t0 > kWaitNs) return false;
  }
}

__device__ __forceinline__ void give_up(Ctl* ctl, uint32_t* status) {
  *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
  atomicCAS(status, 0u, (uint32_t)LQ_ETIMEOUT);
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_dq_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                   const DqArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + (size_t)NSTAGE * STAGE_BYTES);
  volatile int* abort = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ctl->tmem_full[b], 1);
      mbar_init(&ctl->tmem_empty[b], kEpiWarps * 32);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) tmem_alloc(&ctl->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  if (warp < kEpiWarps) {
    // ---------------------------------------------------------------- epilogue
    int lt = 0;
    for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x, ++lt) {
      const int tm = tile % a.tiles_m, tn = tile / a.tiles_m;
      const int b = lt & 1;
      if (!__all_sync(0xffffffffu, wait_phase(&ctl->tmem_full[b], (lt >> 1) & 1, abort, true))) {
        give_up(ctl, a.status);
        break;
      }
      tc_fence_after();
      const int token = tm * BM + warp * 32 + lane;
      const bool tok_ok = token < a.batch;
      const float inv = tok_ok ? a.inv_scale[token] : 0.f;
      float* yrow = a.y + (int64_t)(tok_ok ? token : 0) * a.N;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(b * BN + c * 32), r);
        const int n0 = tn * BN + c * 32;
        const float sv = (n0 + lane < a.N) ? load_as_f32(a.s, a.sdt, n0 + lane) : 0.f;
        tmem_ld_wait();
        if (c == BN / 32 - 1) {
          tc_fence_before();
          mbar_arrive(&ctl->tmem_empty[b]);
        }
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
          v[j] = (__uint_as_float(r[j]) * inv) * __shfl_sync(0xffffffffu, sv, j);
        if (tok_ok) {
          if (a.vec_store && n0 + 32 <= a.N) {
            float4* dst = reinterpret_cast<float4*>(yrow + n0);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j < a.N) yrow[n0 + j] = v[j];
          }
        }
      }
    }
  } else if (warp == kTmaWarp) {
    // ---------------------------------------------------------------- both operands by TMA
    if (lane == 0) {
      prefetch_tmap(&tmap_x);
      prefetch_tmap(&tmap_w);
      uint32_t ctr = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.tiles; tile += gridDim.x) {
        const int tm = tile % a.tiles_m, tn = tile / a.tiles_m;
        for (int k = 0; k < a.nks; ++k, ++ctr) {
          const int slot = ctr % NSTAGE;
          if (!wait_phase(&ctl->empty[slot], ((ctr / NSTAGE) & 1) ^ 1, abort, true)) {
            give_up(ctl, a.status);
            ok = false;
            break;
          }
          uint8_t* sa = smem + (size_t)slot * STAGE_BYTES;
          mbar_arrive_expect_tx(&ctl->full[slot], STAGE_BYTES);
          tma_load_2d(sa, &tmap_x, &ctl->full[slot], k * BK, tm * BM);
          tma_load_2d(sa + A_BYTES, &tmap_w, &ctl->full[slot], k * BK, tn * BN);
        }
      }
      const uint32_t outstanding = ctr < NSTAGE ? ctr : NSTAGE;
      for (uint32_t i = 0; i < outstanding; ++i) {
        const uint32_t c = ctr - 1 - i;
        if (!wait_phase(&ctl->full[c % NSTAGE], (c / NSTAGE) & 1, abort, false))
          give_up(ctl, a.status);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(BM, BN);
      uint32_t ctr = 0;
      bool ok = true;
      int lt = 0;
      for (int tile = blockIdx.x; ok && tile < a.tiles; tile += gridDim.x, ++lt) {
        const int b = lt & 1;
        if (!wait_phase(&ctl->tmem_empty[b], ((lt >> 1) & 1) ^ 1, abort, true)) {
          give_up(ctl, a.status);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * BN);
        for (int k = 0; k < a.nks; ++k, ++ctr) {
          const int slot = ctr % NSTAGE;
          if (!wait_phase(&ctl->full[slot], (ctr / NSTAGE) & 1, abort, true)) {
            give_up(ctl, a.status);
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* sa = smem + (size_t)slot * STAGE_BYTES;
          const uint64_t ad = smem_desc_k_sw128(sa);
          const uint64_t bd = smem_desc_k_sw128(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)
            tc_mma_f16(d, ad + 2 * kk, bd + 2 * kk, idesc, (k | kk) != 0);
          tc_commit(&ctl->empty[slot]);
        }
        if (ok) tc_commit(&ctl->tmem_full[b]);
      }
      tc_commit(&ctl->drain);
      if (!wait_phase(&ctl->drain, 0, abort, false)) give_up(ctl, a.status);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ W = blockwise M b

__device__ __forceinline__ void hmma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                           uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// fp16 pair (+-1 of bit j, +-1 of bit j+1) of a block's code: bit 1 is -1, the fp16 sign bit
__device__ __forceinline__ uint32_t pm1_h2(uint32_t bits, int j) {
  return ((bits >> j) & 1u) << 15 | ((bits >> (j + 1)) & 1u) << 31 | 0x3C003C00u;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

constexpr int kDqWarps = 16;
constexpr int kDqGroups = 8;   // groups of 16 blocks per flush of the W staging buffer

// One warp per row (grid-stride over rows): the row's code words are copied to shared memory
// with coalesced 16-byte loads, then groups of 16 blocks go through the MMAs as C = A B, A the
// +-1 codes (16 blocks x 16 code positions, exact in fp16), B = M^T (16 code positions x 8 rows
// i of a block; a second column tile when d > 8), so a lane holds two consecutive outputs i of
// two blocks. They gather as fp16 pairs in a shared-memory piece of the W row, which the warp
// writes out with coalesced 16-byte stores. d <= 16, D <= 32. Dynamic shared memory per warp:
// the row's code words + 16 bytes, then kDqGroups * 16 * d fp16.
template <int NKS>
__global__ void __launch_bounds__(kDqWarps * 32)
    dq_weights_kernel(const uint32_t* __restrict__ packed, int64_t row_words, int N, int G,
                      const float* __restrict__ M, int d, int D, int Kw, __half* __restrict__ W) {
  extern __shared__ __align__(16) uint8_t dsm[];
  // fp16 +-1 pairs for the four values of two code bits (bit 1 is -1, the fp16 sign bit); the
  // lanes read different entries, four words on four banks
  __shared__ uint32_t pm1_pairs[4];
  if (threadIdx.x < 4)
    pm1_pairs[threadIdx.x] = ((threadIdx.x & 1u) << 15) | ((threadIdx.x >> 1) << 31) | 0x3C003C00u;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const size_t code_bytes = ((size_t)row_words * 4 + 16 + 15) / 16 * 16;
  const size_t piece = (size_t)kDqGroups * 16 * d;           // fp16 per flush
  uint8_t* mine = dsm + (size_t)warp * (code_bytes + (piece * 2 + 15) / 16 * 16);
  uint32_t* sc = reinterpret_cast<uint32_t*>(mine);
  __half* sw = reinterpret_cast<__half*>(mine + code_bytes);
  // B fragments of M^T: B[j][i] = M[i][j], j = 16 ks + 2t (+1), + 8 (+1); i = g + 8 nt
  uint32_t bm[NKS][2][2];
#pragma unroll
  for (int ks = 0; ks < NKS; ++ks)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = g + 8 * nt, j = 16 * ks + 2 * t + 8 * h;
        float m0 = 0.f, m1 = 0.f;
        if (i < d && j < D) m0 = M[i * D + j];
        if (i < d && j + 1 < D) m1 = M[i * D + j + 1];
        bm[ks][nt][h] = pack_h2(m0, m1);
      }
  const int ngrp = (G + 15) / 16;
  const int row_u4 = (int)(row_words / 4);                 // rows are 16-byte multiples
  const int gw = blockIdx.x * kDqWarps + warp, nw = gridDim.x * kDqWarps;
  for (int n = gw; n < N; n += nw) {
    const uint4* src = reinterpret_cast<const uint4*>(packed + (int64_t)n * row_words);
    for (int i = lane; i < row_u4; i += 32) reinterpret_cast<uint4*>(sc)[i] = __ldg(src + i);
    if (lane == 0) reinterpret_cast<uint4*>(sc)[row_u4] = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
    __half* wrow = W + (int64_t)n * Kw;
    for (int g0 = 0; g0 < ngrp; g0 += kDqGroups) {
      for (int gr = g0; gr < min(ngrp, g0 + kDqGroups); ++gr) {
        // the lane's blocks: rows g and g + 8 of A (blocks past G give zero codes)
        const int blk0 = gr * 16 + g, blk1 = blk0 + 8;
        uint32_t bits0 = 0, bits1 = 0;
        if (blk0 < G) {
          const int q = blk0 * D;
          bits0 = (uint32_t)(((uint64_t)sc[(q >> 5) + 1] << 32 | sc[q >> 5]) >> (q & 31));
        }
        if (blk1 < G) {
          const int q = blk1 * D;
          bits1 = (uint32_t)(((uint64_t)sc[(q >> 5) + 1] << 32 | sc[q >> 5]) >> (q & 31));
        }
        bits0 >>= 2 * t;
        bits1 >>= 2 * t;
        float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < NKS; ++ks) {
          // code positions 16 ks + 2t (+1) and + 8 (+1); positions >= D meet zero rows of B, so
          // the bits past a block (the next block's) do not matter
          uint32_t a[4];
          a[0] = pm1_pairs[(bits0 >> (16 * ks)) & 3u];
          a[1] = pm1_pairs[(bits1 >> (16 * ks)) & 3u];
          a[2] = pm1_pairs[(bits0 >> (16 * ks + 8)) & 3u];
          a[3] = pm1_pairs[(bits1 >> (16 * ks + 8)) & 3u];
          hmma_16816(c[0], a, bm[ks][0][0], bm[ks][0][1]);
          if (d > 8) hmma_16816(c[1], a, bm[ks][1][0], bm[ks][1][1]);
        }
        // C[blk][i]: this lane holds (blk0, i0), (blk0, i0 + 1), (blk1, i0), (blk1, i0 + 1)
        __half* pw = sw + (size_t)(gr - g0) * 16 * d;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int i0 = 8 * nt + 2 * t;
          if (i0 >= d) continue;
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            const int col = (g + 8 * hb) * d + i0;
            const float lo = c[nt][2 * hb], hi = c[nt][2 * hb + 1];
            if (i0 + 1 < d && (col & 1) == 0) {
              *reinterpret_cast<uint32_t*>(pw + col) = pack_h2(lo, hi);
            } else {
              pw[col] = __float2half_rn(lo);
              if (i0 + 1 < d) pw[col + 1] = __float2half_rn(hi);
            }
          }
        }
      }
      __syncwarp();
      // the piece covers W columns [g0*16*d, ...): blocks past G give columns >= G*d, which
      // must read zero; columns past Kw are not written
      const int k0 = g0 * 16 * d;
      const int kend = min(Kw, k0 + (int)piece);
      for (int k = k0 + 8 * lane; k < kend; k += 256) {
        uint4 v = *reinterpret_cast<const uint4*>(sw + (k - k0));
        if (k + 8 > G * d) {
          __half* hv = reinterpret_cast<__half*>(&v);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (k + e >= G * d) hv[e] = __float2half_rn(0.f);
        }
        *reinterpret_cast<uint4*>(wrow + k) = v;
      }
      __syncwarp();
    }
    // columns past the last piece (the padding to the 64-input stage)
    for (int k = ngrp * 16 * d + 8 * lane; k < Kw; k += 256)
      *reinterpret_cast<uint4*>(wrow + k) = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
  }
}

// ------------------------------------------------------------------ xt = T(x) in fp16

__device__ __forceinline__ float dq_block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = (l < (int)(blockDim.x >> 5)) ? red[l] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One CTA per token: xh[t][0 .. Kw) = fp16(xt * 2^e), zero from K; inv_scale[t] = 2^-e.
// Dynamic shared memory: K floats.
__global__ void __launch_bounds__(512)
    xt_f16_kernel(const void* __restrict__ x, int xdt, int K, Whiten T, int Kw,
                  __half* __restrict__ xh, float* __restrict__ inv_scale) {
  extern __shared__ __align__(16) float sx[];
  __shared__ float red[32];
  const int t = blockIdx.x, tid = threadIdx.x;
  const int64_t row = (int64_t)t * K;
  if (T.block >= 32 && T.block <= 256) {
    for (int b = tid >> 5; b < K / T.block; b += blockDim.x >> 5)
      warp_whiten_block(x, xdt, row, b * T.block, T.block >> 5, T, T.inv_sqrt, sx + b * T.block);
    __syncthreads();
  } else if (T.block > 0) {
    whiten_blocks_smem(x, xdt, row, K, T, 0, K / T.block, sx);
  } else {
    for (int k = tid; k < K; k += blockDim.x) sx[k] = load_as_f32(x, xdt, row + k);
    __syncthreads();
  }
  float amax = 0.f;
  for (int k = tid; k < K; k += blockDim.x) amax = fmaxf(amax, fabsf(sx[k]));
  amax = dq_block_max(amax, red);
  int sh = 0;
  if (amax > 0.f && isfinite(amax)) {
    int ex;
    frexpf(amax, &ex);   // amax < 2^ex
    sh = min(120, max(-120, 14 - ex));
  }
  const float scale = ldexpf(1.f, sh);
  if (tid == 0) inv_scale[t] = ldexpf(1.f, -sh);
  __half* out = xh + (int64_t)t * Kw;
  for (int k2 = tid; k2 < Kw / 2; k2 += blockDim.x) {
    const int k = 2 * k2;
    const float v0 = k < K ? sx[k] * scale : 0.f;
    const float v1 = k + 1 < K ? sx[k + 1] * scale : 0.f;
    reinterpret_cast<uint32_t*>(out)[k2] = pack_h2(v0, v1);
  }
}

}  // namespace dq

// ------------------------------------------------------------------ host side

DqPlan plan_gemm_dq(int32_t batch, int32_t N, int32_t K, int32_t d, int32_t D) {
  DqPlan p{};
  if (batch < 1 || d > 16 || D > 32) return p;
  if ((size_t)K * sizeof(float) > 200 * 1024) return p;   // xt_f16_kernel keeps xt in smem
  const int64_t G = ((int64_t)K + d - 1) / d;
  const int64_t Kw = (G * d + dq::BK - 1) / dq::BK * dq::BK;
  if (Kw > (1 << 24)) return p;
  const int64_t tn = ((int64_t)N + dq::BN - 1) / dq::BN;
  const int64_t tm = ((int64_t)batch + dq::BM - 1) / dq::BM;
  if (tn * tm > (1 << 30)) return p;
  p.Kw = (int)Kw;
  p.G = (int)G;
  p.nks = (int)(Kw / dq::BK);
  p.tiles_n = (int)tn;
  p.tiles_m = (int)tm;
  p.tiles = (int)(tn * tm);
  p.smem = dq::kSmemBytes;
  // the dequantisation kernel: per warp the row's code words (+16 bytes) and a piece of W
  const int64_t row_bytes = ((G * D + 7) / 8 + 15) / 16 * 16;
  p.dq_smem = (size_t)dq::kDqWarps * ((size_t)(row_bytes + 16 + 15) / 16 * 16 +
                                      ((size_t)dq::kDqGroups * 16 * d * 2 + 15) / 16 * 16);
  if (p.dq_smem > 220 * 1024) return p;
  p.dq_ctas_per_sm = (int)std::max<size_t>(1, std::min<size_t>(2, 220 * 1024 / p.dq_smem));
  p.xt_smem = (size_t)K * sizeof(float);
  p.w_bytes = (size_t)N * Kw * sizeof(__half);
  p.x_bytes = (size_t)batch * Kw * sizeof(__half);
  p.scale_bytes = (size_t)batch * sizeof(float);
  p.ok = true;
  return p;
}

cudaError_t launch_gemm_dq(const DqPlan& pl, const void* x, int xdt, int32_t batch, int32_t K,
                           Whiten T, const float* M, int32_t d, int32_t D,
                           const uint32_t* packed, int64_t row_bytes, int32_t N, const void* s,
                           int sdt, float* y, void* scratch, uint32_t* status, cudaStream_t st) {
  static int xt_set[64], gemm_set[64], dq_set[64], dq_set1[64];
  uint8_t* sp = static_cast<uint8_t*>(scratch);
  __half* W = reinterpret_cast<__half*>(sp);
  __half* xh = reinterpret_cast<__half*>(sp + pl.w_bytes);
  float* inv_scale = reinterpret_cast<float*>(sp + pl.w_bytes + pl.x_bytes);
  const int sms = tc_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;

  const void* dqk = D > 16 ? (const void*)dq::dq_weights_kernel<2> : (const void*)dq::dq_weights_kernel<1>;
  cudaError_t e = ensure_smem(dqk, pl.dq_smem, D > 16 ? dq_set : dq_set1);
  if (e != cudaSuccess) return e;
  const int dq_ctas = (int)std::min<int64_t>((int64_t)sms * pl.dq_ctas_per_sm,
                                             (N + dq::kDqWarps - 1) / dq::kDqWarps);
  if (D > 16)
    dq::dq_weights_kernel<2><<<dq_ctas, dq::kDqWarps * 32, pl.dq_smem, st>>>(
        packed, row_bytes / 4, N, pl.G, M, d, D, pl.Kw, W);
  else
    dq::dq_weights_kernel<1><<<dq_ctas, dq::kDqWarps * 32, pl.dq_smem, st>>>(
        packed, row_bytes / 4, N, pl.G, M, d, D, pl.Kw, W);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = ensure_smem((const void*)dq::xt_f16_kernel, pl.xt_smem, xt_set);
  if (e != cudaSuccess) return e;
  dq::xt_f16_kernel<<<batch, 512, pl.xt_smem, st>>>(x, xdt, K, T, pl.Kw, xh, inv_scale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  TensorMapEncodeFn enc = tensor_map_encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  CUtensorMap tx, tw;
  const cuuint32_t estride[2] = {1, 1};
  {
    const cuuint64_t gdim[2] = {(cuuint64_t)pl.Kw, (cuuint64_t)batch};
    const cuuint64_t gstride[1] = {(cuuint64_t)pl.Kw * sizeof(__half)};
    const cuuint32_t box[2] = {dq::BK, dq::BM};
    if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, xh, gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t gdim[2] = {(cuuint64_t)pl.Kw, (cuuint64_t)N};
    const cuuint64_t gstride[1] = {(cuuint64_t)pl.Kw * sizeof(__half)};
    const cuuint32_t box[2] = {dq::BK, dq::BN};
    if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, W, gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  e = ensure_smem((const void*)dq::gemm_dq_kernel, pl.smem, gemm_set);
  if (e != cudaSuccess) return e;
  dq::DqArgs a;
  a.inv_scale = inv_scale;
  a.s = s;
  a.y = y;
  a.status = status;
  a.N = N;
  a.batch = batch;
  a.nks = pl.nks;
  a.tiles_m = pl.tiles_m;
  a.tiles = pl.tiles;
  a.sdt = sdt;
  a.vec_store = (N % 4 == 0) && (reinterpret_cast<uintptr_t>(y) % 16 == 0);
  const int grid = std::min(pl.tiles, sms);
  dq::gemm_dq_kernel<<<grid, dq::kThreads, pl.smem, st>>>(tx, tw, a);
  return cudaGetLastError();
}

}  // namespace lq
