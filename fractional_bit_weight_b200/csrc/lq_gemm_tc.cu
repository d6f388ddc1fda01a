// lq_gemm_tc.cu -- the large-batch path of lq_gemm: a 5th-generation tensor-core (tcgen05)
// GEMM over the lifted activations and the +-1 codes.
//
// The operator is y[t][n] = s[n] * sum_q b[n][q] z[t][q], with z = blockdiag(M^T) T(x[t])
// (LiftQuant paper, sec. 3 intro: o = diag(s) W (M T a); the review's "Method": T* = lift o T
// folded into one linear map, then an INT1 x FP product). With many tokens this is a dense
// contraction of length L = ceil(K/d)*D, so it runs on the tensor cores:
//
//  * lift_f16_kernel (one CTA per token): whitening T, lift, and a per-token power-of-two scale
//    2^e chosen from a bound on |z|, written as fp16 z * 2^e. Inside every 32-coordinate word
//    the coordinates are stored in the order q0, q0+16, q0+1, q0+17, ..., q0+15, q0+31 -- the
//    order in which the GEMM unpacks a 32-bit code word into fp16 pairs (see pm1_pair).
//  * gemm_tc_kernel (persistent, one CTA per SM): 128-token x 256-row output tiles, in groups
//    of token tiles holding ~40 MB of z, each group swept across all row tiles token tile
//    fastest: the group's z stays resident in L2 and the CTAs of one wave share the codes of a
//    few row tiles; the codes are read once per group. A warp
//    loads the fp16 z tile with TMA (128-byte swizzle); eight warps expand the stored bits of
//    256 rows into +-1 fp16 in the same swizzled K-major layout; one thread issues
//    tcgen05.mma (fp32 accumulation in tensor memory, two accumulators so the epilogue of one
//    tile overlaps the main loop of the next); four warps read the accumulators back with
//    tcgen05.ld and apply 2^-e and s[n].
//
// Every wait on an mbarrier is bounded in time: on expiry the kernel records LQ_ETIMEOUT in
// the workspace status word, the other roles leave their loops, in-flight copies and MMAs are
// waited for (again bounded) and tensor memory is released before the CTA exits.
#include <cuda.h>

#include <cmath>
#include <mutex>

#include "lq_device.cuh"
#include "lq_sm100.cuh"

namespace lq {
namespace tc {

using namespace lq::sm100;

constexpr int BM = 128;                     // tokens per tile: MMA M, tensor-memory lanes
constexpr int BN = 256;                     // code rows per tile: MMA N
constexpr int BK = 64;                      // lifted coordinates per stage: one 128-byte row
constexpr int UK = 16;                      // K of one kind::f16 MMA
constexpr int NSTAGE = 4;
constexpr int A_BYTES = BM * BK * 2;        // 16 KB fp16 z tile
constexpr int B_BYTES = BN * BK * 2;        // 32 KB fp16 +-1 tile
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kEpiWarps = 4;                // warps 0..3: epilogue (tensor-memory lanes 0..127)
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kFirstProdWarp = 6;
constexpr int kProdWarps = BN / 32;         // one code row per producer thread
constexpr int kThreads = (kFirstProdWarp + kProdWarps) * 32;
constexpr int kTmemCols = 2 * BN;           // two fp32 accumulators of 128 x 256
constexpr int kPf = 8;                      // stages of code words prefetched per producer
constexpr uint64_t kWaitNs = 2000000000ull; // 2 s bound on any single wait

struct Ctl {
  uint64_t full_a[NSTAGE];   // TMA bytes of the z tile landed
  uint64_t full_b[NSTAGE];   // all producer threads wrote the +-1 tile
  uint64_t empty[NSTAGE];    // MMAs reading the stage completed
  uint64_t tmem_full[2];     // accumulator holds a finished tile
  uint64_t tmem_empty[2];    // epilogue has read the accumulator
  uint64_t drain;            // all MMAs of this CTA completed
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = 1024 + (size_t)NSTAGE * STAGE_BYTES + sizeof(Ctl);

struct TcArgs {
  const uint32_t* packed;
  int64_t row_words;        // 32-bit words per stored row
  const float* inv_scale;   // [batch] 2^-e of each token
  const void* s;
  float* y;
  uint32_t* status;         // workspace status word
  int N, batch, nks, tiles_n, tiles_m, tiles, sdt, vec_store;
  int group_m;   // token tiles per raster group
};

// Tile -> (token tile, row tile): groups of group_m token tiles, each swept across every row
// tile, token tile fastest inside a group. A group's z (group_m x 128 tokens) stays in L2 while
// its row tiles stream past, and a wave of CTAs shares the codes of a few row tiles; the codes
// are read once per group.
__device__ __forceinline__ void tile_coords(const TcArgs& a, int tile, int& tm, int& tn) {
  const int span = a.group_m * a.tiles_n;
  const int grp = tile / span, r = tile - grp * span;
  const int gm = min(a.group_m, a.tiles_m - grp * a.group_m);
  tm = grp * a.group_m + r % gm;
  tn = r / gm;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on one mbarrier phase. `honor_abort` lets a role leave as soon as another role
// has given up; drains pass false so that they only return once their own work has landed.
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

// fp16 pair (+-1 for bit i, +-1 for bit i+16) of a code word: stored bit 1 means -1, which is
// the fp16 sign bit; 0x3C00 is 1.0.
__device__ __forceinline__ uint32_t pm1_pair(uint32_t w, int i) {
  return ((w << (15 - i)) & 0x80008000u) | 0x3C003C00u;
}

// Expands 64 stored bits (two code words) of tile row p into the 128-byte K-major row p of
// the swizzled B tile: 16-byte chunk c of row p sits at chunk position c ^ (p % 8) inside
// its 8-row, 1024-byte atom.
__device__ __forceinline__ void expand_row(uint8_t* tile, int p, uint2 w) {
  uint8_t* row = tile + (p >> 3) * 1024 + (p & 7) * 128;
  const int sw = p & 7;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t wd = c < 4 ? w.x : w.y;
    const int i0 = 4 * (c & 3);
    uint4 v;
    v.x = pm1_pair(wd, i0 + 0);
    v.y = pm1_pair(wd, i0 + 1);
    v.z = pm1_pair(wd, i0 + 2);
    v.w = pm1_pair(wd, i0 + 3);
    *reinterpret_cast<uint4*>(row + ((c ^ sw) << 4)) = v;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_z, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + (size_t)NSTAGE * STAGE_BYTES);
  volatile int* abort = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&ctl->full_a[s], 1);
      mbar_init(&ctl->full_b[s], kProdWarps * 32);
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
      int tm, tn;
      tile_coords(a, tile, tm, tn);
      const int b = lt & 1;
      // tcgen05.ld below is warp-collective: every lane must take the same branch here
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
        // lane j fetches s[n0 + j]; every lane scales by its own token's 2^-e
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
    // ---------------------------------------------------------------- z tiles by TMA
    if (lane == 0) {
      prefetch_tmap(&tmap_z);
      uint32_t ctr = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.tiles; tile += gridDim.x) {
        int tm, tn;
        tile_coords(a, tile, tm, tn);
        for (int k = 0; k < a.nks; ++k, ++ctr) {
          const int slot = ctr % NSTAGE;
          if (!wait_phase(&ctl->empty[slot], ((ctr / NSTAGE) & 1) ^ 1, abort, true)) {
            give_up(ctl, a.status);
            ok = false;
            break;
          }
          uint8_t* sa = smem + (size_t)slot * STAGE_BYTES;
          mbar_arrive_expect_tx(&ctl->full_a[slot], A_BYTES);
          tma_load_2d(sa, &tmap_z, &ctl->full_a[slot], k * BK, tm * BM);
        }
      }
      // no copy may still be writing shared memory when the CTA exits
      const uint32_t outstanding = ctr < NSTAGE ? ctr : NSTAGE;
      for (uint32_t i = 0; i < outstanding; ++i) {
        const uint32_t c = ctr - 1 - i;
        if (!wait_phase(&ctl->full_a[c % NSTAGE], (c / NSTAGE) & 1, abort, false))
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
          const uint32_t ph = (ctr / NSTAGE) & 1;
          if (!wait_phase(&ctl->full_a[slot], ph, abort, true) ||
              !wait_phase(&ctl->full_b[slot], ph, abort, true)) {
            give_up(ctl, a.status);
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* sa = smem + (size_t)slot * STAGE_BYTES;
          const uint64_t ad = smem_desc_k_sw128(sa);
          const uint64_t bd = smem_desc_k_sw128(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)   // +32 bytes per K step inside the swizzle row
            tc_mma_f16(d, ad + 2 * kk, bd + 2 * kk, idesc, (k | kk) != 0);
          tc_commit(&ctl->empty[slot]);
        }
        if (ok) tc_commit(&ctl->tmem_full[b]);
      }
      tc_commit(&ctl->drain);
      if (!wait_phase(&ctl->drain, 0, abort, false)) give_up(ctl, a.status);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- +-1 expansion
    const int p = threadIdx.x - kFirstProdWarp * 32;
    uint32_t ctr = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < a.tiles; tile += gridDim.x) {
      int tm, tn;
      tile_coords(a, tile, tm, tn);
      const int n = tn * BN + p;
      const bool valid = n < a.N;
      const uint2* rp = reinterpret_cast<const uint2*>(a.packed + (valid ? (int64_t)n * a.row_words : 0));
      uint2 ring[kPf];
#pragma unroll
      for (int i = 0; i < kPf; ++i) ring[i] = (valid && i < a.nks) ? __ldg(rp + i) : make_uint2(0u, 0u);
      for (int k0 = 0; ok && k0 < a.nks; k0 += kPf) {
#pragma unroll
        for (int u = 0; u < kPf; ++u) {
          const int k = k0 + u;
          if (k < a.nks) {
            const int slot = ctr % NSTAGE;
            if (!wait_phase(&ctl->empty[slot], ((ctr / NSTAGE) & 1) ^ 1, abort, true)) {
              give_up(ctl, a.status);
              ok = false;
              break;
            }
            const uint2 w = ring[u];
            if (valid && k + kPf < a.nks) ring[u] = __ldg(rp + k + kPf);
            expand_row(smem + (size_t)slot * STAGE_BYTES + A_BYTES, p, w);
            fence_proxy_async_smem();
            mbar_arrive(&ctl->full_b[slot]);
            ++ctr;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ prologue

__device__ __forceinline__ float block_max(float v, float* red) {
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

constexpr int kLiftChunk = 4096;   // lifted coordinates per pass of the prologue

// One CTA per token: zh[t][0 .. Lp) fp16 (word-interleaved order, zero beyond L) and
// inv_scale[t] = 2^-e. Dynamic shared memory: M in rows of D4 = D rounded up to 4 columns
// (zero beyond D), xt zero-padded to Kp, then one pass of natural-order z.
// four CTAs per SM (53 KB of shared memory each at K = 8192): a register cap of 32
__global__ void __launch_bounds__(512, 4)
    lift_f16_kernel(const void* __restrict__ x, int xdt, int K, Whiten T,
                    const float* __restrict__ M, int d, int D, int Kp, int64_t L, int Lp,
                    __half* __restrict__ zh, float* __restrict__ inv_scale) {
  extern __shared__ __align__(16) float sm[];
  __shared__ float red[32];
  float* sM = sm;                          // [d][D4]
  float* sx = sm + LQ_MAX_D * LQ_MAX_D;    // xt, zero-padded to Kp
  float* zc = sx + ((Kp + 3) & ~3);        // z of one pass, natural order
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t row = (int64_t)t * K;
  const int D4 = (D + 3) & ~3;
  for (int k = tid; k < d * D4; k += blockDim.x) {
    const int i = k / D4, j = k - i * D4;
    sM[k] = j < D ? M[i * D + j] : 0.f;
  }
  if (T.block >= 32 && T.block <= 256) {
    // a warp per Hadamard block, no barrier between the butterfly stages
    for (int b = tid >> 5; b < K / T.block; b += blockDim.x >> 5)
      warp_whiten_block(x, xdt, row, b * T.block, T.block >> 5, T, T.inv_sqrt, sx + b * T.block);
  } else if (T.block > 0) {
    whiten_blocks_smem(x, xdt, row, K, T, 0, K / T.block, sx);   // ends with a barrier
  } else {
    for (int k = tid; k < K; k += blockDim.x) sx[k] = load_as_f32(x, xdt, row + k);
  }
  for (int k = K + tid; k < Kp; k += blockDim.x) sx[k] = 0.f;
  __syncthreads();

  // |z[g*D+j]| <= max|xt| * max_j sum_i |M[i][j]|: a power-of-two scale that maps this bound
  // to at most 2^14 keeps every fp16 value finite and normal-range for any input.
  float amax = 0.f;
  for (int k = tid; k < K; k += blockDim.x) amax = fmaxf(amax, fabsf(sx[k]));
  amax = block_max(amax, red);
  float cs = 0.f;
  for (int j = tid; j < D; j += blockDim.x) {
    float c = 0.f;
    for (int i = 0; i < d; ++i) c += fabsf(sM[i * D4 + j]);
    cs = fmaxf(cs, c);
  }
  const float cmax = block_max(cs, red);
  const float bound = amax * cmax;
  int sh = 0;
  if (bound > 0.f && isfinite(bound)) {
    int ex;
    frexpf(bound, &ex);   // bound < 2^ex
    sh = min(120, max(-120, 14 - ex));
  }
  const float scale = ldexpf(1.f, sh);
  if (tid == 0) inv_scale[t] = ldexpf(1.f, -sh);

  __half* zrow = zh + (int64_t)t * Lp;
  const int nb = D4 >> 2;
  for (int cq = 0; cq < Lp; cq += kLiftChunk) {
    const int qe = min(cq + kLiftChunk, Lp);             // stored positions [cq, qe)
    const int qv = (int)min((int64_t)qe, L);             // coordinates with a value
    // natural-order z of [cq, qv): a thread takes 4 columns of one group (lanes: consecutive
    // groups, same columns, so the 16-byte M loads are shared by the warp)
    if (cq < qv) {
      const int g_lo = cq / D, g_hi = (qv - 1) / D;
      const int ng = g_hi - g_lo + 1;
      for (int task = tid; task < ng * nb; task += blockDim.x) {
        const int jb = task / ng, gl = task - jb * ng;
        const int g = g_lo + gl;
        const float* xg = sx + g * d;
        const float* mc = sM + 4 * jb;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 2
        for (int i = 0; i < d; ++i) {
          const float xv = xg[i];
          const float4 m4 = *reinterpret_cast<const float4*>(mc + i * D4);
          a0 = fmaf(m4.x, xv, a0);
          a1 = fmaf(m4.y, xv, a1);
          a2 = fmaf(m4.z, xv, a2);
          a3 = fmaf(m4.w, xv, a3);
        }
        const int qb = g * D + 4 * jb;
        const float av[4] = {a0, a1, a2, a3};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = qb + u;
          if (4 * jb + u < D && q >= cq && q < qv) zc[q - cq] = av[u];
        }
      }
    }
    for (int ql = max(0, qv - cq) + tid; ql < qe - cq; ql += blockDim.x) zc[ql] = 0.f;
    __syncthreads();
    // 8 consecutive stored positions per item: positions q0 + 2i + h hold coordinate
    // q0 + i + 16h (passes start on multiples of 32, so a word never straddles two)
    for (int it = tid; it < (qe - cq) / 8; it += blockDim.x) {
      const int pos0 = cq + it * 8;
      const int q0 = pos0 & ~31;
      const int i0 = (pos0 & 31) >> 1;
      uint32_t packed[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float v0 = zc[q0 + i0 + r - cq] * scale;
        const float v1 = zc[q0 + i0 + r + 16 - cq] * scale;
        const __half2 hv = __floats2half2_rn(v0, v1);
        packed[r] = *reinterpret_cast<const uint32_t*>(&hv);
      }
      *reinterpret_cast<uint4*>(zrow + pos0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int sm_count() {
  static int cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace tc

TensorMapEncodeFn tensor_map_encode_fn() { return tc::encode_fn(); }
int tc_sm_count() { return tc::sm_count(); }

TcPlan plan_gemm_tc(int32_t batch, int64_t L, int32_t N, int32_t K, int32_t d) {
  TcPlan p{};
  if (batch < 1) return p;
  const int64_t Kp = ((int64_t)K + d - 1) / d * d;
  p.pro_smem = (size_t)(LQ_MAX_D * LQ_MAX_D + ((Kp + 3) & ~3) + tc::kLiftChunk) * sizeof(float);
  if (p.pro_smem > 200 * 1024) return p;
  const int64_t Lp = (L + tc::BK - 1) / tc::BK * tc::BK;
  if (Lp > (1 << 30)) return p;
  const int64_t tn = ((int64_t)N + tc::BN - 1) / tc::BN;
  const int64_t tm = ((int64_t)batch + tc::BM - 1) / tc::BM;
  if (tn * tm > (1 << 30)) return p;
  p.Lp = (int)Lp;
  p.nks = (int)(Lp / tc::BK);
  p.tiles_n = (int)tn;
  p.tiles_m = (int)tm;
  p.tiles = (int)(tn * tm);
  // token tiles per raster group: about 40 MB of fp16 z, a third of L2
  p.group_m = (int)std::max<int64_t>(1, std::min<int64_t>(tm, (40ll << 20) / ((int64_t)tc::BM * Lp * 2)));
  p.smem = tc::kSmemBytes;
  p.z_bytes = (size_t)batch * Lp * sizeof(__half);
  p.scale_bytes = (size_t)batch * sizeof(float);
  p.ok = true;
  return p;
}

cudaError_t launch_gemm_tc(const TcPlan& pl, const void* x, int xdt, int32_t batch, int32_t K,
                           Whiten T, const float* M, int32_t d, int32_t D, int64_t L,
                           const uint32_t* packed, int64_t row_bytes, int32_t N, const void* s,
                           int sdt, float* y, void* scratch, uint32_t* status, cudaStream_t st) {
  static int pro_set[64], gemm_set[64];
  __half* zh = static_cast<__half*>(scratch);
  float* inv_scale = reinterpret_cast<float*>(static_cast<uint8_t*>(scratch) + pl.z_bytes);
  const int Kp = (int)(((int64_t)K + d - 1) / d * d);

  cudaError_t e = ensure_smem((const void*)tc::lift_f16_kernel, pl.pro_smem, pro_set);
  if (e != cudaSuccess) return e;
  tc::lift_f16_kernel<<<batch, 512, pl.pro_smem, st>>>(x, xdt, K, T, M, d, D, Kp, L, pl.Lp, zh,
                                                       inv_scale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  tc::EncodeTiledFn enc = tc::encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t gdim[2] = {(cuuint64_t)pl.Lp, (cuuint64_t)batch};
  const cuuint64_t gstride[1] = {(cuuint64_t)pl.Lp * sizeof(__half)};
  const cuuint32_t box[2] = {tc::BK, tc::BM};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, zh, gdim, gstride, box, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  e = ensure_smem((const void*)tc::gemm_tc_kernel, pl.smem, gemm_set);
  if (e != cudaSuccess) return e;
  const int sms = tc::sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  tc::TcArgs a;
  a.packed = packed;
  a.row_words = row_bytes / 4;
  a.inv_scale = inv_scale;
  a.s = s;
  a.y = y;
  a.status = status;
  a.N = N;
  a.batch = batch;
  a.nks = pl.nks;
  a.tiles_n = pl.tiles_n;
  a.tiles_m = pl.tiles_m;
  a.tiles = pl.tiles;
  a.group_m = pl.group_m;
  a.sdt = sdt;
  a.vec_store = (N % 4 == 0) && (reinterpret_cast<uintptr_t>(y) % 16 == 0);
  const int grid = std::min(pl.tiles, sms);
  tc::gemm_tc_kernel<<<grid, tc::kThreads, pl.smem, st>>>(tmap, a);
  return cudaGetLastError();
}

}  // namespace lq
