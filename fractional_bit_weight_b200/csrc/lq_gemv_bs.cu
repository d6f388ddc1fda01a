// lq_gemv_bs.cu -- decode GEMV for small batches (batch <= 8) with the stored codes staged
// through shared memory.
//
// y[t][n] = s[n] * sum_q b[n][q] z[t][q], b in {+1,-1}, z = lift(T(x[t])) (paper sec. 3 intro:
// o = diag(s) W (M T a); review "Method": an INT1 x FP product plus small linear maps, no lookup
// table). With b = 1 - 2*bit the row sum is sum_q z_q - 2 * (sum of z over the set bits).
//
// One kernel per call, one CTA per SM, S K-slices x R row ranges:
//  * two producer warps stream the CTA's rows into a ring of shared-memory stages (32 rows x one
//    window of the slice) with 16-byte cp.async copies, completing each stage's mbarrier; each
//    CTA owns a contiguous range of rows, so the copies read long contiguous runs of HBM;
//  * meanwhile the 16 compute warps build the activation operand of their slice in shared
//    memory: a power of two S per token from a bound on |z| (|xt_i| <= ||block of sign * scale
//    * x||_2 times the largest column 1-norm of M), the whitening of the slice's Hadamard blocks,
//    the lift z = M^T xt per block of d inputs, and three int8 planes (base 254) of
//    z * S * 2^-p (p = q mod 8) in the register layout of the B operand of mma.m16n8k32. Every
//    CTA of a slice computes the same operand; none waits for another;
//  * the compute warps take the (32-row stage, 64-byte chunk) items of each stage in turn: one
//    AND per code word gives the int8 A operand (bit p of each byte as 0 or 2^p) and the B
//    entries carry 2^-p, so all eight bit positions accumulate into one int32 set, exact across
//    the whole slice (a row of <= 2^17 coordinates cannot overflow); at the end of a 32-row group
//    each warp adds its int32 sums into the CTA's per-row totals (integer shared-memory atomics,
//    exact in any order);
//  * y = s * (sum z + sum_plane w_plane * total_plane), w_plane = -2 * 254^-plane / S. With
//    several K-slices the CTAs of a row range add their int32 totals into a global array and the
//    last one to finish writes y (and clears the array for the next call).
// Every sum is exact or runs in a fixed order: the result does not depend on timing.
#include "lq_device.cuh"
#include "lq_sm100.cuh"

namespace lq {

namespace bs {
constexpr int kWarps = 16;                     // compute warps
constexpr int kProdWarps = 2;                  // producer warps
constexpr int kProd = kProdWarps * 32;
constexpr int kThreads = (kWarps + kProdWarps) * 32;
constexpr int kCompute = kWarps * 32;
constexpr int kRows = 32;                      // rows per stage
constexpr int kMaxStages = 8;
constexpr int kPlanes = 3;
constexpr int kTokU4 = 96;                     // uint4 per (chunk, token): 8 MMA pairs x 12 lanes
constexpr int kTokBytes = kTokU4 * 16;         // 1536
constexpr int kMaxTokens = 8;
constexpr int kZP = 576;                       // 512 z values + 8 pad floats per 128
constexpr int kCPP = 4;                        // chunks lifted and quantised per pass
constexpr uint64_t kWaitNs = 1000000000ull;    // bounded waits: 1 s
}  // namespace bs

struct BsParams {
  const void* x;
  int xdt;
  int batch;
  int K;
  Whiten T;
  const float* M;
  int d;
  int D;
  int64_t L;
  const uint8_t* packed;
  int64_t row_bytes;
  int N;
  const void* s;
  int sdt;
  float* y;
  // plan
  int nchunk;      // 512-bit chunks per row
  int sc;          // chunks per K-slice
  int S;           // K-slices
  int R;           // row ranges (CTA b: slice b % S, range b / S)
  int rq, rrem;    // range i has rq + (i < rrem) rows
  int wch;         // chunks per window (stage width)
  int stride;      // shared-memory row stride of a stage (bytes)
  int NS;          // stages in the ring
  int xs_floats;   // whitened inputs of the slice, per token
  int rows_max;    // rq + 1
  size_t frag_bytes;   // shared memory: fragments of the slice
  size_t prep_bytes;   // shared memory: whitening, z and M scratch
  // global scratch (S > 1 only)
  float* sumz;         // [S][batch] sum of z over each slice
  int* gacc;           // [batch][N][4] int32 totals, zero at rest
  uint32_t* counters;  // [R], zero at rest
  uint32_t* status;    // workspace status word
};

__device__ __forceinline__ void csync() { asm volatile("bar.sync 1, %0;" ::"n"(bs::kCompute) : "memory"); }

__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_status(uint32_t* status, uint32_t code) {
  atomicCAS(status, 0u, code);
}

// Waits for the phase of `bar` with the given parity; false after kWaitNs.
__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity) {
  if (sm100::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtime();
  while (!sm100::mbar_try_wait(bar, parity))
    if (gtime() - t0 > bs::kWaitNs) return false;
  return true;
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sm100::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void imma(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                     uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bs_warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float bs_warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// three int8 planes of base 254: a ~= P0 + P1/254 + P2/254^2 (|a| <= 64)
__device__ __forceinline__ void bs_planes3(float a, int (&P)[3]) {
  P[0] = __float2int_rn(a);
  float r = (a - (float)P[0]) * 254.f;
  P[1] = __float2int_rn(r);
  r = (r - (float)P[1]) * 254.f;
  P[2] = __float2int_rn(r);
}

// The power-of-two scale of every token (compute threads; ends with csync): |z| * S <= 64 with
// |z_j| <= max_j sum_i |M[i][j]| * max over Hadamard blocks of || (sign * scale * x)_block ||_2
// (identity T: max |x|).
__device__ void token_scales(const BsParams& P, float* s_tok, float* red) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Bh = P.T.block;
  __shared__ float s_cm;
  if (warp == 0) {
    float a = 0.f;
    if (lane < P.D)
      for (int i = 0; i < P.d; ++i) a += fabsf(P.M[i * P.D + lane]);
    a = bs_warp_max(a);
    if (lane == 0) s_cm = a;
  }
  csync();
  const float cm = s_cm;
  for (int t = 0; t < P.batch; ++t) {
    const int64_t off = (int64_t)t * P.K;
    float m = 0.f;   // max block norm^2 (identity: max x^2) seen by this thread
    if (Bh >= 32) {
      for (int b = warp; b < P.K / Bh; b += bs::kWarps) {
        float a = 0.f;
        for (int i = lane; i < Bh; i += 32) {
          const int k = b * Bh + i;
          float v = load_as_f32(P.x, P.xdt, off + k);
          if (P.T.chan_scale) v *= P.T.chan_scale[k];
          a = fmaf(v, v, a);
        }
        m = fmaxf(m, bs_warp_sum(a));
      }
    } else if (Bh > 0) {
      for (int b = tid; b < P.K / Bh; b += bs::kCompute) {
        float a = 0.f;
        for (int i = 0; i < Bh; ++i) {
          const int k = b * Bh + i;
          float v = load_as_f32(P.x, P.xdt, off + k);
          if (P.T.chan_scale) v *= P.T.chan_scale[k];
          a = fmaf(v, v, a);
        }
        m = fmaxf(m, a);
      }
    } else {
      for (int k = tid; k < P.K; k += bs::kCompute) {
        const float v = load_as_f32(P.x, P.xdt, off + k);
        m = fmaxf(m, v * v);
      }
    }
    m = bs_warp_max(m);
    if (lane == 0) red[warp] = m;
    csync();
    if (warp == 0) {
      float a = lane < bs::kWarps ? red[lane] : 0.f;
      a = bs_warp_max(a);
      if (lane == 0) {
        // sqrt rounds within an ulp and the sums of squares carry rounding of a few ulps; the
        // factor 1.001 keeps the bound above every |z| the lift computes
        const float bound = cm * sqrtf(a) * 1.001f;
        int ex = 0;
        frexpf(bound, &ex);   // bound = f * 2^ex, f in [0.5, 1)
        s_tok[t] = bound > 0.f ? ldexpf(1.f, 6 - ex) : 1.f;
      }
    }
    csync();
  }
}

// cp.async of 16 bytes, global -> shared, L2 only
__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// arrive on `bar` once every cp.async this thread issued so far has landed
__device__ __forceinline__ void cp_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(sm100::smem_u32(bar))
               : "memory");
}

// The activation operand of this CTA's slice (compute threads; ends with csync): whitened inputs
// of the slice's Hadamard blocks, then kCPP chunks per pass: z, the token's sum of z, and the
// three int8 planes of z * S * 2^-p stored in the B-operand layout at frag [chunk][token][...].
__device__ void build_operand(const BsParams& P, int c0, int nc, uint8_t* frag, float* prep,
                              const float* s_tok, float (*s_red)[bs::kWarps], float* s_sumz) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* xs = prep;                                         // [batch][xs_floats]
  float* zs = xs + (size_t)P.batch * P.xs_floats;           // [kCPP][batch][576]
  float* Ms = zs + (size_t)bs::kCPP * P.batch * bs::kZP;    // [d][D]
  const int q_lo = c0 * 512;
  const int q_hi = (int)min((int64_t)(c0 + nc) * 512, P.L);
  const int k0 = (q_lo / P.D) * P.d;
  const int k1 = min(((q_hi - 1) / P.D + 1) * P.d, P.K);
  const int Bh = P.T.block;
  int base = k0, span = k1 - k0;
  if (Bh > 0) {
    const int blk0 = k0 / Bh;
    base = blk0 * Bh;
    span = ((k1 + Bh - 1) / Bh - blk0) * Bh;
  }
  for (int i = bs::kCompute - 1 - tid; i < P.d * P.D; i += bs::kCompute) Ms[i] = P.M[i];
  // 1. whitened inputs of every token
  if (Bh >= 32 && Bh <= 256) {
    const int E = Bh >> 5;
    const int nblk = span / Bh;
    for (int task = warp; task < P.batch * nblk; task += bs::kWarps) {
      const int tok = task / nblk, b = task - tok * nblk;
      warp_whiten_block(P.x, P.xdt, (int64_t)tok * P.K, base + b * Bh, E, P.T, 1.f,
                        xs + tok * P.xs_floats + b * Bh);
    }
    csync();
  } else {
    for (int e = tid; e < P.batch * span; e += bs::kCompute) {
      const int tok = e / span, i = e - tok * span;
      const int k = base + i;
      float a = 0.f;
      if (k < P.K) {
        a = load_as_f32(P.x, P.xdt, (int64_t)tok * P.K + k);
        if (Bh > 0) {
          if (P.T.chan_scale) a *= P.T.chan_scale[k];
          if (P.T.sign && P.T.sign[k] < 0) a = -a;
        }
      }
      xs[tok * P.xs_floats + i] = a;
    }
    csync();
    if (Bh > 1) {
      const int half = span / 2;
      for (int h = 1; h < Bh; h <<= 1) {
        for (int pp = tid; pp < P.batch * half; pp += bs::kCompute) {
          const int tok = pp / half, pi = pp - tok * half;
          const int lo = pi & (h - 1);
          const int i = ((pi - lo) << 1) | lo;
          float* xt = xs + tok * P.xs_floats;
          const float a = xt[i], c2 = xt[i + h];
          xt[i] = a + c2;
          xt[i + h] = a - c2;
        }
        csync();
      }
    }
  }
  // 2. kCPP chunks per pass: thread tid owns value e = tid of each chunk and token
  float su[bs::kMaxTokens];
#pragma unroll
  for (int t = 0; t < bs::kMaxTokens; ++t) su[t] = 0.f;
  for (int cb = 0; cb < nc; cb += bs::kCPP) {
    const int ncp = min(bs::kCPP, nc - cb);
#pragma unroll
    for (int u = 0; u < bs::kCPP; ++u) {
      if (u < ncp) {
        const int qi = (c0 + cb + u) * 512 + tid;
        int gg = 0, jj = 0, dv = 0;
        if (qi < q_hi) {
          gg = qi / P.D;
          jj = qi - gg * P.D;
          dv = min(P.d, P.K - gg * P.d);
        }
#pragma unroll
        for (int tok = 0; tok < bs::kMaxTokens; ++tok) {
          if (tok < P.batch) {
            float acc = 0.f;
            const float* xg = xs + tok * P.xs_floats + (gg * P.d - base);
            for (int ii = 0; ii < dv; ++ii) acc = fmaf(Ms[ii * P.D + jj], xg[ii], acc);
            acc *= P.T.inv_sqrt;
            su[tok] += acc;
            zs[(u * P.batch + tok) * bs::kZP + tid + 8 * (tid >> 7)] = acc;
          }
        }
      }
    }
    csync();
    // quantise and store: item -> (chunk u, token, tt, j, h, p); its 4 values e0 + 8*i fill one
    // 32-bit word per plane: register h of the MMA (j, p) of lane 4*plane + tt of the token's block
    for (int gi = tid; gi < ncp * P.batch * 128; gi += bs::kCompute) {
      const int ut = gi >> 7, grp = gi & 127;
      const int u = ut / P.batch, tok = ut - u * P.batch;
      const int pl8 = grp & 7, tt = (grp >> 3) & 3, hl = (grp >> 5) & 1, jl = grp >> 6;
      uint32_t w4[bs::kPlanes] = {};
      const float Sp = s_tok[tok] * __int_as_float((127 - pl8) << 23);   // S * 2^-p, exact
      const int e0 = 128 * tt + 64 * jl + 32 * hl + pl8;
      const float* zc = zs + ut * bs::kZP + e0 + 8 * tt;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int Pq[bs::kPlanes];
        bs_planes3(zc[8 * i] * Sp, Pq);
#pragma unroll
        for (int pl = 0; pl < bs::kPlanes; ++pl) w4[pl] |= ((uint32_t)Pq[pl] & 0xffu) << (8 * i);
      }
      const int mma = jl * 8 + pl8;
      uint32_t* fw = reinterpret_cast<uint32_t*>(
          frag + ((size_t)(cb + u) * P.batch + tok) * bs::kTokBytes);
#pragma unroll
      for (int pl = 0; pl < bs::kPlanes; ++pl)
        fw[((mma >> 1) * 12 + 4 * pl + tt) * 4 + (mma & 1) * 2 + hl] = w4[pl];
    }
    csync();
  }
  // 3. the slice's sum of z per token, in a fixed order (lanes, then warps)
#pragma unroll
  for (int tok = 0; tok < bs::kMaxTokens; ++tok) {
    if (tok < P.batch) {
      const float v = bs_warp_sum(su[tok]);
      if (lane == 0) s_red[tok][warp] = v;
    }
  }
  csync();
  if (warp < P.batch) {
    float v = lane < bs::kWarps ? s_red[warp][lane] : 0.f;
    v = bs_warp_sum(v);
    if (lane == 0) s_sumz[warp] = v;
  }
  csync();
}

template <int NT>
__global__ void __launch_bounds__(bs::kThreads, 1) gemv_bs_kernel(const BsParams P) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[bs::kMaxStages], empty_bar[bs::kMaxStages];
  __shared__ float s_tok[bs::kMaxTokens];
  __shared__ float s_w[bs::kMaxTokens][bs::kPlanes];
  __shared__ float s_sumz[bs::kMaxTokens];
  __shared__ float s_red[bs::kMaxTokens][bs::kWarps];
  __shared__ int s_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sl = blockIdx.x % P.S, ri = blockIdx.x / P.S;
  const int c0 = sl * P.sc;
  const int nc = min(P.sc, P.nchunk - c0);
  const int ra = ri * P.rq + min(ri, P.rrem);
  const int rows = P.rq + (ri < P.rrem ? 1 : 0);
  const int ngroups = (rows + bs::kRows - 1) / bs::kRows;
  const int nwin = (nc + P.wch - 1) / P.wch;
  const int nst = ngroups * nwin;
  const int64_t slice_off = (int64_t)c0 * 64;
  const int64_t slice_bytes = min((int64_t)nc * 64, P.row_bytes - slice_off);

  const size_t stage_bytes = (size_t)bs::kRows * P.stride;
  uint8_t* frag_sm = smem;
  float* prep = reinterpret_cast<float*>(smem + P.frag_bytes);
  uint8_t* ring = smem + P.frag_bytes + P.prep_bytes;
  int* rowacc = reinterpret_cast<int*>(ring + (size_t)P.NS * stage_bytes);   // [rows_max][8*NT]

  if (tid == 0) {
    for (int i = 0; i < P.NS; ++i) {
      sm100::mbar_init(&full_bar[i], bs::kProd);
      sm100::mbar_init(&empty_bar[i], bs::kWarps);
    }
    sm100::mbar_fence_init();
  }
  __syncthreads();

  if (warp >= bs::kWarps) {
    // ---------------- producers: rows [ra, ra + rows), the slice's bytes, window by window;
    // 16-byte copies, consecutive lanes on consecutive pieces of a row
    const int p = tid - bs::kCompute;
    const uint32_t ring_u32 = sm100::smem_u32(ring);
    bool ok = true;
    for (int st = 0; st < nst; ++st) {
      const int k = st % P.NS;
      if (st >= P.NS && !bar_wait(&empty_bar[k], ((st / P.NS) & 1) ^ 1)) {
        if (p == 0) record_status(P.status, LQ_ETIMEOUT);
        ok = false;
        break;
      }
      const int grp = st / nwin, win = st - grp * nwin;
      const int r0 = grp * bs::kRows, nr = min(bs::kRows, rows - r0);
      const int64_t woff = slice_off + (int64_t)win * P.wch * 64;
      const int wpieces = (int)(min((int64_t)P.wch * 64, slice_off + slice_bytes - woff) / 16);
      const uint8_t* src = P.packed + (int64_t)(ra + r0) * P.row_bytes + woff;
      const uint32_t dst = ring_u32 + (uint32_t)(k * stage_bytes);
      for (int e = p; e < nr * wpieces; e += bs::kProd) {
        const int r = e / wpieces, c = e - r * wpieces;
        cp16(dst + (uint32_t)(r * P.stride + 16 * c), src + (int64_t)r * P.row_bytes + 16 * c);
      }
      cp_arrive(&full_bar[k]);
    }
    // no copy may still be in flight when the CTA exits
    asm volatile("cp.async.wait_all;" ::: "memory");
    (void)ok;
    return;
  }

  // ---------------- compute warps: 1. the activation operand of this slice
  token_scales(P, s_tok, &s_red[0][0]);
  build_operand(P, c0, nc, frag_sm, prep, s_tok, s_red, s_sumz);
  for (int i = tid; i < P.rows_max * 8 * NT; i += bs::kCompute) rowacc[i] = 0;
  if (tid < P.batch) {
    const float S = s_tok[tid];
    s_w[tid][0] = -2.f / S;
    s_w[tid][1] = (float)(-2.0 / 254.0) / S;
    s_w[tid][2] = (float)(-2.0 / (254.0 * 254.0)) / S;
    if (P.S > 1 && ri == 0) P.sumz[sl * P.batch + tid] = s_sumz[tid];
  }
  csync();

  // 2. main loop
  const int g = lane >> 2, t = lane & 3;
  const uint32_t ring_u32 = sm100::smem_u32(ring);
  const uint32_t frag_u32 = sm100::smem_u32(frag_sm);
  // this lane's B registers in tile nt: token 2*nt + (lane >> 4), lane (lane & 15) of its block
  uint32_t fofs[NT];
  bool live[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tk = 2 * nt + (lane >> 4);
    live[nt] = tk < P.batch && (lane & 15) < 12;
    fofs[nt] = (uint32_t)((tk * bs::kTokU4 + (lane & 15)) * 16);
  }
  const uint32_t chunk_bytes = (uint32_t)P.batch * bs::kTokBytes;

  int acc[NT][2][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int a = 0; a < 2; ++a) acc[nt][a][0] = acc[nt][a][1] = acc[nt][a][2] = acc[nt][a][3] = 0;

  int item0 = 0;   // index of the first item of the stage, counted over the CTA's stages
  for (int st = 0; st < nst; ++st) {
    const int k = st % P.NS;
    const int grp = st / nwin, win = st - grp * nwin;
    const int nitems = min(P.wch, nc - win * P.wch);
    const int nr = min(bs::kRows, rows - grp * bs::kRows);
    if (!bar_wait(&full_bar[k], (st / P.NS) & 1)) {
      if (lane == 0) record_status(P.status, LQ_ETIMEOUT);
    }
    const uint32_t sbase = ring_u32 + (uint32_t)(k * stage_bytes) + (uint32_t)(g * P.stride + 16 * t);
    const bool h1 = nr > 16;
    int it = item0 + ((warp - item0) % bs::kWarps + bs::kWarps) % bs::kWarps;
    for (; it < item0 + nitems; it += bs::kWarps) {
      const int cw = it - item0;                       // chunk within the window
      const int cs = win * P.wch + cw;                 // chunk within the slice
      const uint32_t arow = sbase + 64 * cw;
      uint4 u0 = lds128(arow), u1 = lds128(arow + 8 * P.stride);
      uint4 u2 = make_uint4(0, 0, 0, 0), u3 = u2;
      if (h1) {
        u2 = lds128(arow + 16 * P.stride);
        u3 = lds128(arow + 24 * P.stride);
      }
      const uint32_t fb = frag_u32 + (uint32_t)cs * chunk_bytes;
#pragma unroll
      for (int m2 = 0; m2 < 8; ++m2) {
        uint4 bv[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          bv[nt] = live[nt] ? lds128(fb + fofs[nt] + m2 * 12 * 16) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int mma = 2 * m2 + e;
          const int j = mma >> 3, p = mma & 7;
          const uint32_t msk = 0x01010101u << p;
          const uint32_t a0 = (j ? u0.z : u0.x) & msk, a2 = (j ? u0.w : u0.y) & msk;
          const uint32_t a1 = (j ? u1.z : u1.x) & msk, a3 = (j ? u1.w : u1.y) & msk;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint32_t b0 = e ? bv[nt].z : bv[nt].x, b1 = e ? bv[nt].w : bv[nt].y;
            imma(acc[nt][0], a0, a1, a2, a3, b0, b1);
          }
          if (h1) {
            const uint32_t c0r = (j ? u2.z : u2.x) & msk, c2r = (j ? u2.w : u2.y) & msk;
            const uint32_t c1r = (j ? u3.z : u3.x) & msk, c3r = (j ? u3.w : u3.y) & msk;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const uint32_t b0 = e ? bv[nt].z : bv[nt].x, b1 = e ? bv[nt].w : bv[nt].y;
              imma(acc[nt][1], c0r, c1r, c2r, c3r, b0, b1);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(&empty_bar[k]);
    item0 += nitems;
    // end of a 32-row group: this warp's int32 sums into the CTA's per-row totals
    if (win == nwin - 1) {
      const int rbase = grp * bs::kRows;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int rr = rbase + 16 * a + g + 8 * (r >> 1);
            const int col = 2 * t + (r & 1);           // column within the tile
            const int tok = 2 * nt + (col >> 2), pl = col & 3;
            if (rr < rows && pl < bs::kPlanes && tok < P.batch && acc[nt][a][r] != 0)
              atomicAdd(&rowacc[rr * 8 * NT + 8 * nt + col], acc[nt][a][r]);
            acc[nt][a][r] = 0;
          }
    }
  }
  csync();

  // 3. epilogue
  if (P.S == 1) {
    for (int e = tid; e < rows * P.batch; e += bs::kCompute) {
      const int tok = e / rows, rr = e - tok * rows;
      const int* ra4 = rowacc + rr * 8 * NT + 8 * (tok >> 1) + 4 * (tok & 1);
      const double v = (double)s_sumz[tok] + (double)s_w[tok][0] * (double)ra4[0] +
                       (double)s_w[tok][1] * (double)ra4[1] + (double)s_w[tok][2] * (double)ra4[2];
      const int row = ra + rr;
      P.y[(int64_t)tok * P.N + row] = load_as_f32(P.s, P.sdt, row) * (float)v;
    }
    return;
  }
  // several K-slices: integer totals into the global array, the last CTA of the range writes y
  for (int e = tid; e < rows * P.batch; e += bs::kCompute) {
    const int tok = e / rows, rr = e - tok * rows;
    const int* ra4 = rowacc + rr * 8 * NT + 8 * (tok >> 1) + 4 * (tok & 1);
    int* ga = P.gacc + ((int64_t)tok * P.N + ra + rr) * 4;
#pragma unroll
    for (int pl = 0; pl < bs::kPlanes; ++pl)
      if (ra4[pl] != 0) atomicAdd(ga + pl, ra4[pl]);
  }
  csync();
  if (tid == 0) {
    __threadfence();
    const bool last = atomicAdd(P.counters + ri, 1u) == (uint32_t)(P.S - 1);
    if (last) __threadfence();
    s_flag = last ? 1 : 0;
  }
  csync();
  if (!s_flag) return;
  if (tid < P.batch) {
    float su = 0.f;
    for (int k = 0; k < P.S; ++k) su += __ldcg(P.sumz + k * P.batch + tid);
    s_sumz[tid] = su;
  }
  csync();
  for (int e = tid; e < rows * P.batch; e += bs::kCompute) {
    const int tok = e / rows, rr = e - tok * rows;
    int* ga = P.gacc + ((int64_t)tok * P.N + ra + rr) * 4;
    const int v0 = atomicExch(ga + 0, 0), v1 = atomicExch(ga + 1, 0), v2 = atomicExch(ga + 2, 0);
    const double v = (double)s_sumz[tok] + (double)s_w[tok][0] * (double)v0 +
                     (double)s_w[tok][1] * (double)v1 + (double)s_w[tok][2] * (double)v2;
    const int row = ra + rr;
    P.y[(int64_t)tok * P.N + row] = load_as_f32(P.s, P.sdt, row) * (float)v;
  }
  if (tid == 0) P.counters[ri] = 0u;   // ready for the next call on this workspace
}

// ------------------------------------------------------------------ host side

namespace {
int bs_sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 0;
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}
// shared-memory row stride with stride % 128 == 64: the eight rows that one quarter-warp of a
// 16-byte load reads fall on disjoint banks
int padded_stride(int bytes) {
  const int s = (bytes + 63) / 64 * 64;
  return s % 128 == 64 ? s : s + 64;
}
}  // namespace

BsPlan plan_gemv_bs(int32_t batch, int64_t L, int32_t N, int32_t K, int32_t d, int32_t D,
                    int32_t Bh) {
  BsPlan p{};
  // int32 totals: every plane product is at most 127 * 128, so a row of <= 2^17 lifted
  // coordinates cannot overflow; the per-CTA whitening keeps blocks of at most 256 inputs
  if (batch < 1 || batch > bs::kMaxTokens || L > (1 << 17) || Bh > 256 || d * D > 1024)
    return p;
  p.nt = batch <= 2 ? 1 : batch <= 4 ? 2 : 4;
  p.nchunk = (int)((L + 511) / 512);
  const int sms = bs_sm_count();
  constexpr size_t kBudget = 224 * 1024;
  const int64_t row_chunks = (((L + 7) / 8 + 15) / 16 * 16 + 63) / 64;
  for (int S = 1; S <= 16; ++S) {
    const int sc = (p.nchunk + S - 1) / S;
    if (S > 1 && (p.nchunk + sc - 1) / sc != S) continue;   // no empty slice
    const int R = std::max(1, std::min(sms / S, (N + 15) / 16));
    const int rq = N / R;
    const int rows_max = rq + 1;
    const size_t frag = (size_t)sc * batch * bs::kTokBytes;
    const int span = (int)std::min<int64_t>(((int64_t)sc * 512 / D + 2) * d, (int64_t)K + Bh);
    const int xs = Bh > 0 ? ((span + Bh - 1) / Bh + 1) * Bh : span;
    const size_t prep =
        (((size_t)batch * xs + (size_t)bs::kCPP * batch * bs::kZP + 1024) * 4 + 127) / 128 * 128;
    const size_t acc_bytes = (size_t)rows_max * 8 * p.nt * 4;
    // windows of about 832 bytes of a row (13 chunks): stages of 32 rows x ~26 KB
    const int64_t slice_chunks = std::min<int64_t>(sc, row_chunks);
    const int nwin = (int)((slice_chunks + 12) / 13);
    const int wch = (int)((slice_chunks + nwin - 1) / nwin);
    const int stride = padded_stride(wch * 64);
    const size_t stage = (size_t)bs::kRows * stride;
    if (frag + prep + acc_bytes + 2 * stage > kBudget) continue;
    const int NS = std::min<int>((int)((kBudget - frag - prep - acc_bytes) / stage), bs::kMaxStages);
    if (NS < 3 && S < 16) continue;   // a narrower slice leaves room for a deeper ring
    p.S = S;
    p.sc = sc;
    p.R = R;
    p.rq = rq;
    p.rrem = N % R;
    p.rows_max = rows_max;
    p.wch = wch;
    p.stride = stride;
    p.NS = NS;
    p.xs_floats = xs;
    p.frag_smem = frag;
    p.prep_smem = prep;
    p.smem = frag + prep + (size_t)NS * stage + acc_bytes;
    p.ok = true;
    break;
  }
  if (!p.ok) return p;
  p.nctas = p.S * p.R;
  p.sumz_bytes = p.S > 1 ? (size_t)p.S * batch * 4 : 0;
  p.gacc_bytes = p.S > 1 ? (size_t)batch * N * 4 * 4 : 0;
  return p;
}

template <int NT>
static cudaError_t launch_bs_nt(const BsPlan& pl, const BsParams& P, cudaStream_t st) {
  static int smem_set[64];
  cudaError_t e = ensure_smem((const void*)gemv_bs_kernel<NT>, pl.smem, smem_set);
  if (e != cudaSuccess) return e;
  gemv_bs_kernel<NT><<<pl.nctas, bs::kThreads, pl.smem, st>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_gemv_bs(const BsPlan& pl, const void* x, int xdt, int32_t batch, int32_t K,
                           Whiten T, const float* M, int32_t d, int32_t D, int64_t L,
                           const uint32_t* packed, int64_t row_bytes, int32_t N, const void* s,
                           int sdt, float* y, const BsScratch& ws, cudaStream_t st) {
  BsParams P{};
  P.x = x;
  P.xdt = xdt;
  P.batch = batch;
  P.K = K;
  P.T = T;
  P.M = M;
  P.d = d;
  P.D = D;
  P.L = L;
  P.packed = reinterpret_cast<const uint8_t*>(packed);
  P.row_bytes = row_bytes;
  P.N = N;
  P.s = s;
  P.sdt = sdt;
  P.y = y;
  P.nchunk = pl.nchunk;
  P.sc = pl.sc;
  P.S = pl.S;
  P.R = pl.R;
  P.rq = pl.rq;
  P.rrem = pl.rrem;
  P.wch = pl.wch;
  P.stride = pl.stride;
  P.NS = pl.NS;
  P.xs_floats = pl.xs_floats;
  P.rows_max = pl.rows_max;
  P.frag_bytes = pl.frag_smem;
  P.prep_bytes = pl.prep_smem;
  P.sumz = ws.sumz;
  P.gacc = ws.gacc;
  P.counters = ws.counters;
  P.status = ws.status;
  switch (pl.nt) {
    case 1: return launch_bs_nt<1>(pl, P, st);
    case 2: return launch_bs_nt<2>(pl, P, st);
    default: return launch_bs_nt<4>(pl, P, st);
  }
}

}  // namespace lq
