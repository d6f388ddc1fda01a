// lq_gemv_bs.cu -- decode GEMV for small batches (batch <= 8) with the stored codes staged
// through shared memory.
//
// y[t][n] = s[n] * sum_q b[n][q] z[t][q], b in {+1,-1}, z = lift(T(x[t])) (paper sec. 3 intro:
// o = diag(s) W (M T a); review "Method": an INT1 x FP product plus small linear maps, no lookup
// table). With b = 1 - 2*bit the row sum is sum_q z_q - 2 * (sum of z over the set bits).
//
// One kernel per call, one CTA per SM, S K-slices x R row ranges:
//  * one producer thread streams the CTA's rows into a ring of shared-memory stages (R rows of
//    16 or 32) with bulk copies: a whole stage in one copy when the CTA reads whole rows (its rows
//    are contiguous in HBM), else one copy per row of the slice. The copies run on the async
//    (TMA) path and leave the load/store pipe to the compute warps;
//  * meanwhile the 16 compute warps build the activation operand of their slice in shared
//    memory: the slice's inputs staged once, a power of two S per token from a bound on |z|
//    (|xt_i| <= ||block of sign * scale * x||_2 times the largest column 1-norm of M), the
//    whitening in place, then one warp per 512-coordinate chunk lifts z = M^T xt per block of d
//    inputs and stores three int8 planes (base 254) of z * S * 2^-p (p = q mod 8) in the
//    register layout of the B operand of mma.m16n8k32. Every CTA of a slice builds the same
//    operand and none waits for another;
//  * the compute warps take the (stage rows, 64-byte chunk) items of each stage in turn: one AND
//    per code word gives the int8 A operand (bit p of each byte as 0 or 2^p) and the B entries
//    carry 2^-p, so all eight bit positions accumulate into int32 sums (two chains by bit-position
//    parity), exact across the whole slice (a row of <= 2^17 coordinates cannot overflow); at the
//    end of a row group each warp adds its sums into the CTA's per-row totals (integer
//    shared-memory atomics, exact in any order). The rows of a quarter-warp's 16-byte loads are
//    permuted so that they fall on disjoint shared-memory banks;
//  * y = s * (sum z + sum_plane w_plane * total_plane), w_plane = -2 * 254^-plane / S. With
//    several K-slices the CTAs of a row range add their int32 totals into a global array and the
//    last one to finish writes y (and clears the array for the next call).
// Every sum is exact or runs in a fixed order: the result does not depend on timing.
#include "lq_device.cuh"
#include "lq_sm100.cuh"

namespace lq {

namespace bs {
constexpr int kWarps = 16;                     // compute warps
constexpr int kThreads = (kWarps + 1) * 32;    // + the producer warp
constexpr int kCompute = kWarps * 32;
constexpr int kMaxStages = 8;
constexpr int kPlanes = 3;
constexpr int kTokU4 = 96;                     // uint4 per (chunk, token): 8 MMA pairs x 12 lanes
constexpr int kTokBytes = kTokU4 * 16;         // 1536
constexpr int kMaxTokens = 8;
constexpr int kZeroBytes = kTokBytes;          // a zero block: the B registers of absent lanes
constexpr int kMaxD = 16;                      // inputs per block (d) the lift holds in registers
constexpr int kMaxMs = 512;                    // floats of M in shared memory (d * D <= 512)
constexpr int kZw = 512 + 4 * 8;               // floats of one warp's z buffer (padded)
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
  int rows_per_stage;  // 16 or 32
  int wch;         // chunks per window (stage width)
  int stride;      // shared-memory row stride of a stage (bytes)
  int whole;       // 1: a stage is one copy of whole contiguous rows (stride == row_bytes)
  int NS;          // stages in the ring
  int early_stages;    // stages the producer issues before the operand is built
  uint32_t perm;   // 8 nibbles: stage row of MMA row g (g < 8) inside each group of 8
  int xs_floats;   // staged, whitened inputs of the slice, per token
  int rows_max;    // rq + 1
  size_t frag_bytes;   // shared memory: fragments of the slice, then the zero block
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

// The power-of-two scale S of a token from the largest squared Hadamard-block norm a2 of
// (scale * x) (identity T: the largest x^2): |z| * S <= 64 with |z_j| <= cm * sqrt(a2), cm the
// largest column 1-norm of M. sqrt rounds within an ulp and the sums of squares carry rounding
// of a few ulps; the factor 1.001 keeps the bound above every |z| the lift computes.
__device__ __forceinline__ float scale_from_bound(float cm, float a2) {
  const float bound = cm * sqrtf(a2) * 1.001f;
  int ex = 0;
  frexpf(bound, &ex);   // bound = f * 2^ex, f in [0.5, 1)
  return bound > 0.f ? ldexpf(1.f, 6 - ex) : 1.f;
}

// The largest column 1-norm of M (warp 0; compute threads, ends with csync).
__device__ float column_norm(const BsParams& P, float* s_cm) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    float a = 0.f;
    if (lane < P.D)
      for (int i = 0; i < P.d; ++i) a += fabsf(P.M[i * P.D + lane]);
    a = bs_warp_max(a);
    if (lane == 0) *s_cm = a;
  }
  csync();
  return *s_cm;
}

// Largest squared block norm of token t over inputs [k_lo, k_hi) read from global memory
// (block-aligned range; identity T: largest x^2). Compute threads; every thread returns its part
// (the caller reduces).
__device__ float block_norms_global(const BsParams& P, int t, int k_lo, int k_hi) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Bh = P.T.block;
  const int64_t off = (int64_t)t * P.K;
  float m = 0.f;
  if (Bh >= 32) {
    for (int b = k_lo / Bh + warp; b < k_hi / Bh; b += bs::kWarps) {
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
    for (int b = k_lo / Bh + tid; b < k_hi / Bh; b += bs::kCompute) {
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
    for (int k = k_lo + tid; k < k_hi; k += bs::kCompute) {
      const float v = load_as_f32(P.x, P.xdt, off + k);
      m = fmaxf(m, v * v);
    }
  }
  return m;
}

// Largest squared block norm of the staged inputs xs[0 .. span) (block-aligned, scaled, before
// the transform; the signs do not change a norm).
__device__ float block_norms_smem(const float* xs, int span, int Bh) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float m = 0.f;
  if (Bh >= 32) {
    for (int b = warp; b < span / Bh; b += bs::kWarps) {
      float a = 0.f;
      for (int i = lane; i < Bh; i += 32) a = fmaf(xs[b * Bh + i], xs[b * Bh + i], a);
      m = fmaxf(m, bs_warp_sum(a));
    }
  } else if (Bh > 0) {
    for (int b = tid; b < span / Bh; b += bs::kCompute) {
      float a = 0.f;
      for (int i = 0; i < Bh; ++i) a = fmaf(xs[b * Bh + i], xs[b * Bh + i], a);
      m = fmaxf(m, a);
    }
  } else {
    for (int i = tid; i < span; i += bs::kCompute) m = fmaxf(m, xs[i] * xs[i]);
  }
  return m;
}

// The activation operand of this CTA's slice (compute threads; ends with csync):
//  1. the inputs of the slice's Hadamard blocks, scaled and signed, staged as fp32 in xs (one
//     global read), from which the token's scale S comes (over all of K: from xs when the slice
//     covers K, else from global memory);
//  2. the transform in place: per block, H / sqrt(Bh);
//  3. per chunk, one warp: each lane lifts the 16 coordinates of four groups of the B-operand
//     layout (z = M^T xt over the d inputs of each coordinate's block), adds them to its sum of
//     z, and stores the three int8 planes of z * S * 2^-p at frag [chunk][token][...]; the
//     chunks need no barrier between them.
__device__ __forceinline__ void build_operand(const BsParams& P, int c0, int nc,
                                              uint8_t* __restrict__ frag, float* __restrict__ prep,
                                              float* s_tok, float (*s_red)[bs::kWarps],
                                              float* s_sumz, float* s_cm) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Bh = P.T.block;
  const int q_lo = c0 * 512;
  const int q_hi = (int)min((int64_t)(c0 + nc) * 512, P.L);
  const int k0 = (q_lo / P.D) * P.d;
  const int k1 = min(((q_hi - 1) / P.D + 1) * P.d, P.K);
  int base = k0, span = k1 - k0;
  if (Bh > 0) {
    const int blk0 = k0 / Bh;
    base = blk0 * Bh;
    span = ((k1 + Bh - 1) / Bh - blk0) * Bh;
  }
  float* __restrict__ xs = prep;                             // [batch][xs_floats]
  float* __restrict__ Ms = xs + (size_t)P.batch * P.xs_floats;   // [d][D]
  float* __restrict__ zbuf = Ms + bs::kMaxMs;                     // [warp][kZw]
  for (int i = tid; i < P.d * P.D; i += bs::kCompute) Ms[i] = __ldg(P.M + i);
  const float cm = column_norm(P, s_cm);
  // 1. staged inputs (zero past K), scaled and signed when T is a transform; eight loads per
  // thread are issued before their stores
  for (int tok = 0; tok < P.batch; ++tok) {
    for (int i0 = 0; i0 < span; i0 += 8 * bs::kCompute) {
      float v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int i = i0 + r * bs::kCompute + tid;
        const int k = base + i;
        float a = 0.f;
        if (i < span && k < P.K) {
          a = load_as_f32(P.x, P.xdt, (int64_t)tok * P.K + k);
          if (Bh > 0) {
            if (P.T.chan_scale) a *= __ldg(P.T.chan_scale + k);
            if (P.T.sign && __ldg(P.T.sign + k) < 0) a = -a;
          }
        }
        v[r] = a;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int i = i0 + r * bs::kCompute + tid;
        if (i < span) xs[tok * P.xs_floats + i] = v[r];
      }
    }
  }
  csync();
  // the token scales: every Hadamard block of the token (the staged ones when they are all)
  const bool whole_k = base == 0 && span >= P.K;
  for (int tok = 0; tok < P.batch; ++tok) {
    float m = whole_k ? block_norms_smem(xs + tok * P.xs_floats, P.K, Bh)
                      : block_norms_global(P, tok, 0, P.K);
    m = bs_warp_max(m);
    if (lane == 0) s_red[tok][warp] = m;
  }
  csync();
  if (warp < P.batch) {
    float a = lane < bs::kWarps ? s_red[warp][lane] : 0.f;
    a = bs_warp_max(a);
    if (lane == 0) s_tok[warp] = scale_from_bound(cm, a);
  }
  // 2. the transform of every block, in place (xt = H v / sqrt(Bh))
  if (Bh >= 32) {
    const int E = Bh >> 5;
    const int nblk = span / Bh;
    for (int task = warp; task < P.batch * nblk; task += bs::kWarps) {
      const int tok = task / nblk, b = task - tok * nblk;
      float* blk = xs + tok * P.xs_floats + b * Bh;
      float v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) v[r] = r < E ? blk[E * lane + r] : 0.f;
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
      __syncwarp();
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < E) blk[E * lane + r] = v[r] * P.T.inv_sqrt;
    }
    csync();
  } else if (Bh > 1) {
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
    for (int i = tid; i < P.batch * span; i += bs::kCompute) {
      const int tok = i / span;
      xs[tok * P.xs_floats + (i - tok * span)] *= P.T.inv_sqrt;
    }
    csync();
  }
  // 3. lift and quantise, one warp per chunk, through the warp's buffer zw of the chunk's z
  // (512 values, 8 floats of padding after every 128 so that step b reads without conflicts):
  //  a. lane -> (gi, j) = (lane / D, lane % D) for the first gpl * D lanes, gpl = 32 / D groups
  //     at a time: column j of M sits in registers and the d inputs of a group are broadcast
  //     loads; the values that fall in the chunk go to zw and into the lane's sum of z;
  //  b. lane -> groups lane + 32 m (m < 4) of the B-operand layout, group -> (p, tt, h, j): its
  //     4 coordinates e0 + 8 i fill one word per plane.
  const int gpl = 32 / P.D;
  const int gi = lane / P.D, jc = lane - gi * P.D;
  const bool lane_on = gi < gpl;
  float Mr[bs::kMaxD];
#pragma unroll
  for (int i = 0; i < bs::kMaxD; ++i) Mr[i] = (lane_on && i < P.d) ? Ms[i * P.D + jc] : 0.f;
  float* __restrict__ zw = zbuf + warp * bs::kZw;
  float su[bs::kMaxTokens];
#pragma unroll
  for (int t = 0; t < bs::kMaxTokens; ++t) su[t] = 0.f;
  for (int c = warp; c < nc; c += bs::kWarps) {
    const int q0 = (c0 + c) * 512;
    const int qe = min(q0 + 512, q_hi);
    const int gf = q0 / P.D, gl = (qe - 1) / P.D;
#pragma unroll
    for (int tok = 0; tok < bs::kMaxTokens; ++tok) {
      if (tok >= P.batch) continue;
      const float* __restrict__ xt = xs + tok * P.xs_floats - base;
      // a. z of the groups that meet the chunk (the chunk's tail past L stays zero)
      for (int g = gf + gi; g <= gl && lane_on; g += gpl) {
        const int kg = g * P.d;
        const int dv = min(P.d, P.K - kg);
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < bs::kMaxD; ++i)
          if (i < dv) a = fmaf(Mr[i], xt[kg + i], a);
        const int e = g * P.D + jc - q0;
        if (e >= 0 && e < qe - q0) {
          zw[e + (e >> 7) * 8] = a;
          su[tok] += a;
        }
      }
      if (qe - q0 < 512)
        for (int e = max(qe - q0, 0) + lane; e < 512; e += 32) zw[e + (e >> 7) * 8] = 0.f;
      __syncwarp();
      // b. quantise into the B-operand layout
      uint32_t* __restrict__ fw =
          reinterpret_cast<uint32_t*>(frag + ((size_t)c * P.batch + tok) * bs::kTokBytes);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int grp = lane + 32 * m;
        const int pl8 = grp & 7, tt = (grp >> 3) & 3, hl = (grp >> 5) & 1, jl = grp >> 6;
        const int e0 = 128 * tt + 64 * jl + 32 * hl + pl8;
        const float Sp = s_tok[tok] * __int_as_float((127 - pl8) << 23);   // S * 2^-p, exact
        uint32_t w4[bs::kPlanes] = {};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = e0 + 8 * i;
          int Pq[bs::kPlanes];
          bs_planes3(zw[e + (e >> 7) * 8] * Sp, Pq);
#pragma unroll
          for (int pl = 0; pl < bs::kPlanes; ++pl) w4[pl] |= ((uint32_t)Pq[pl] & 0xffu) << (8 * i);
        }
        const int mma = jl * 8 + pl8;
#pragma unroll
        for (int pl = 0; pl < bs::kPlanes; ++pl)
          fw[((mma >> 1) * 12 + 4 * pl + tt) * 4 + (mma & 1) * 2 + hl] = w4[pl];
      }
      __syncwarp();
    }
  }
  // the slice's sum of z per token, in a fixed order (lanes, then warps)
  csync();
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

// One item: HT tiles of 16 rows x one 64-byte chunk, NT tiles of B (8 columns each), CH
// accumulator chains per (tile, B tile).
template <int NT, int HT, int CH>
__device__ __forceinline__ void run_item(uint32_t arow, int stride, uint32_t fb, const uint32_t (&fofs)[NT],
                                         uint32_t mstep, int (&acc)[NT][HT][CH][4], bool upper) {
  uint4 u[HT][2];
#pragma unroll
  for (int h = 0; h < HT; ++h) {
    if (h == 0 || upper) {
      u[h][0] = lds128(arow + (uint32_t)(16 * h * stride));
      u[h][1] = lds128(arow + (uint32_t)((16 * h + 8) * stride));
    } else {
      u[h][0] = u[h][1] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int m2 = 0; m2 < 8; ++m2) {
    uint4 bv[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) bv[nt] = lds128(fb + fofs[nt] + m2 * mstep);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int mma = 2 * m2 + e;
      const int j = mma >> 3, p = mma & 7;
      const uint32_t msk = 0x01010101u << p;
#pragma unroll
      for (int h = 0; h < HT; ++h) {
        if (h > 0 && !upper) continue;
        const uint32_t a0 = (j ? u[h][0].z : u[h][0].x) & msk, a2 = (j ? u[h][0].w : u[h][0].y) & msk;
        const uint32_t a1 = (j ? u[h][1].z : u[h][1].x) & msk, a3 = (j ? u[h][1].w : u[h][1].y) & msk;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint32_t b0 = e ? bv[nt].z : bv[nt].x, b1 = e ? bv[nt].w : bv[nt].y;
          imma(acc[nt][h][CH == 2 ? e : 0], a0, a1, a2, a3, b0, b1);
        }
      }
    }
  }
}

template <int NT, int HT>
__global__ void __launch_bounds__(bs::kThreads, 1) gemv_bs_kernel(const BsParams P) {
  constexpr int CH = NT <= 2 ? 2 : 1;   // accumulator chains per (tile, B tile)
  constexpr int RS = 16 * HT;           // rows per stage
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[bs::kMaxStages], empty_bar[bs::kMaxStages];
  __shared__ __align__(8) uint64_t built_bar;
  __shared__ float s_tok[bs::kMaxTokens];
  __shared__ float s_w[bs::kMaxTokens][bs::kPlanes];
  __shared__ float s_sumz[bs::kMaxTokens];
  __shared__ float s_red[bs::kMaxTokens][bs::kWarps];
  __shared__ int s_flag;
  __shared__ float s_cm;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sl = blockIdx.x % P.S, ri = blockIdx.x / P.S;
  const int c0 = sl * P.sc;
  const int nc = min(P.sc, P.nchunk - c0);
  const int ra = ri * P.rq + min(ri, P.rrem);
  const int rows = P.rq + (ri < P.rrem ? 1 : 0);
  const int ngroups = (rows + RS - 1) / RS;
  const int nwin = (nc + P.wch - 1) / P.wch;
  const int nst = ngroups * nwin;
  const int64_t slice_off = (int64_t)c0 * 64;
  const int64_t slice_bytes = min((int64_t)nc * 64, P.row_bytes - slice_off);

  const size_t stage_bytes = (size_t)RS * P.stride + 64;   // + the tail a last chunk may read
  uint8_t* frag_sm = smem;
  float* prep = reinterpret_cast<float*>(smem + P.frag_bytes);
  uint8_t* ring = smem + P.frag_bytes + P.prep_bytes;
  int* rowacc = reinterpret_cast<int*>(ring + (size_t)P.NS * stage_bytes);   // [rows_max][8*NT]

  if (tid == 0) {
    for (int i = 0; i < P.NS; ++i) {
      sm100::mbar_init(&full_bar[i], 1);
      sm100::mbar_init(&empty_bar[i], bs::kWarps);
    }
    sm100::mbar_init(&built_bar, 1);
    sm100::mbar_fence_init();
  }
  __syncthreads();

  if (warp == bs::kWarps) {
    // ---------------- producer: rows [ra, ra + rows), the slice's bytes, window by window; one
    // bulk copy per row (a copy's transfer rate is limited, so many smaller copies in flight
    // stream faster than one large one), issued by four lanes after lane 0 set the byte count
    constexpr int kLanes = 4;
    bool ok = true;
    for (int st = 0; st < nst && ok; ++st) {
      const int k = st % P.NS;
      // the first stages go out at once; the rest wait until the operand is built, so that the
      // build's own requests (inputs, instructions) do not queue behind the whole ring
      if (st == P.early_stages && !bar_wait(&built_bar, 0)) {
        if (lane == 0) record_status(P.status, LQ_ETIMEOUT);
        ok = false;
        break;
      }
      if (st >= P.NS) {
        ok = bar_wait(&empty_bar[k], ((st / P.NS) & 1) ^ 1);
        if (!ok) {
          if (lane == 0) record_status(P.status, LQ_ETIMEOUT);
          break;
        }
      }
      const int grp = st / nwin, win = st - grp * nwin;
      const int r0 = grp * RS, nr = min(RS, rows - r0);
      const int64_t woff = slice_off + (int64_t)win * P.wch * 64;
      const uint32_t wbytes = (uint32_t)min((int64_t)P.wch * 64, slice_off + slice_bytes - woff);
      uint8_t* dst = ring + (size_t)k * stage_bytes;
      const uint8_t* src = P.packed + (int64_t)(ra + r0) * P.row_bytes + woff;
      if (lane == 0) sm100::mbar_arrive_expect_tx(&full_bar[k], (uint32_t)nr * wbytes);
      __syncwarp();
      if (lane < kLanes)
        for (int r = lane; r < nr; r += kLanes)
          bulk_g2s(dst + (size_t)r * P.stride, src + (int64_t)r * P.row_bytes, wbytes, &full_bar[k]);
    }
    // no copy may still be in flight when the CTA exits: wait for the last stages to land
    if (lane == 0)
      for (int st = max(0, nst - P.NS); st < nst && ok; ++st)
        if (!bar_wait(&full_bar[st % P.NS], (st / P.NS) & 1)) record_status(P.status, LQ_ETIMEOUT);
    return;
  }

  // ---------------- compute warps: 1. the activation operand of this slice
  if (tid < bs::kZeroBytes / 16)
    reinterpret_cast<uint4*>(frag_sm + P.frag_bytes - bs::kZeroBytes)[tid] = make_uint4(0, 0, 0, 0);
  build_operand(P, c0, nc, frag_sm, prep, s_tok, s_red, s_sumz, &s_cm);
  if (tid == 0) sm100::mbar_arrive(&built_bar);
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
  const int pg = (int)((P.perm >> (4 * g)) & 7u);   // stage row of MMA row g
  const uint32_t ring_u32 = sm100::smem_u32(ring);
  const uint32_t frag_u32 = sm100::smem_u32(frag_sm);
  const uint32_t zero_u32 = frag_u32 + (uint32_t)(P.frag_bytes - bs::kZeroBytes);
  // this lane's B registers in tile nt: token 2*nt + (lane >> 4), lane (lane & 15) of its block;
  // absent lanes read the zero block (all lanes load, none diverge)
  uint32_t fofs[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tk = 2 * nt + (lane >> 4);
    const bool live = tk < P.batch && (lane & 15) < 12;
    fofs[nt] = live ? (uint32_t)((tk * bs::kTokU4 + (lane & 15)) * 16) : 0xffffffffu;
  }
  const uint32_t chunk_bytes = (uint32_t)P.batch * bs::kTokBytes;
  constexpr uint32_t mstep = 192u;   // one MMA pair of a lane's B registers

  int acc[NT][HT][CH][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int h = 0; h < HT; ++h)
#pragma unroll
      for (int c = 0; c < CH; ++c) acc[nt][h][c][0] = acc[nt][h][c][1] = acc[nt][h][c][2] = acc[nt][h][c][3] = 0;

  int item0 = 0;   // index of the first item of the stage, counted over the CTA's stages
  for (int st = 0; st < nst; ++st) {
    const int k = st % P.NS;
    const int grp = st / nwin, win = st - grp * nwin;
    const int nitems = min(P.wch, nc - win * P.wch);
    const int nr = min(RS, rows - grp * RS);
    if (!bar_wait(&full_bar[k], (st / P.NS) & 1)) {
      if (lane == 0) record_status(P.status, LQ_ETIMEOUT);
    }
    const uint32_t sbase = ring_u32 + (uint32_t)(k * stage_bytes) + (uint32_t)(pg * P.stride + 16 * t);
    const bool upper = nr > 16;
    int it = item0 + ((warp - item0) % bs::kWarps + bs::kWarps) % bs::kWarps;
    for (; it < item0 + nitems; it += bs::kWarps) {
      const int cw = it - item0;                       // chunk within the window
      const uint32_t fb = frag_u32 + (uint32_t)(win * P.wch + cw) * chunk_bytes;
      uint32_t fo[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) fo[nt] = fofs[nt] == 0xffffffffu ? zero_u32 - fb : fofs[nt];
      run_item<NT, HT, CH>(sbase + 64 * cw, P.stride, fb, fo, mstep, acc, upper);
    }
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(&empty_bar[k]);
    item0 += nitems;
    // end of a row group: this warp's int32 sums into the CTA's per-row totals
    if (win == nwin - 1) {
      const int rbase = grp * RS;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < HT; ++h)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            int v = acc[nt][h][0][r];
            if (CH == 2) v += acc[nt][h][CH - 1][r];
            const int rr = rbase + 16 * h + pg + 8 * (r >> 1);
            const int col = 2 * t + (r & 1);           // column within the tile
            const int tok = 2 * nt + (col >> 2), pl = col & 3;
            if (rr < rows && pl < bs::kPlanes && tok < P.batch && v != 0)
              atomicAdd(&rowacc[rr * 8 * NT + 8 * nt + col], v);
#pragma unroll
            for (int c = 0; c < CH; ++c) acc[nt][h][c][r] = 0;
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
// shared-memory row stride with stride % 128 == 64: the rows that one quarter-warp of a 16-byte
// load reads (two consecutive rows of 64 bytes) fall on disjoint banks
int padded_stride(int bytes) {
  const int s = (bytes + 63) / 64 * 64;
  return s % 128 == 64 ? s : s + 64;
}
// MMA row g (g < 8) -> stage row, for rows `stride` bytes apart: a quarter-warp loads 64 bytes
// of MMA rows 2i and 2i+1, which must not share banks; with m = (stride / 16) mod 8 the two
// stage rows must differ by 4 (m odd), by 2 mod 4 (m = 2, 6) or by an odd number (m = 4).
// Returns 0 when no permutation helps (stride a multiple of 128).
uint32_t row_perm(int stride) {
  const int m = (stride / 16) % 8;
  static const int p4[8] = {0, 4, 1, 5, 2, 6, 3, 7}, p2[8] = {0, 2, 1, 3, 4, 6, 5, 7};
  const int* p = nullptr;
  static const int id[8] = {0, 1, 2, 3, 4, 5, 6, 7};
  if (stride % 16 != 0 || m == 0) return 0;
  p = (m & 1) ? p4 : (m == 4 ? id : p2);
  uint32_t v = 0;
  for (int g = 0; g < 8; ++g) v |= (uint32_t)p[g] << (4 * g);
  return v;
}
}  // namespace

BsPlan plan_gemv_bs(int32_t batch, int64_t L, int32_t N, int32_t K, int32_t d, int32_t D,
                    int32_t Bh) {
  BsPlan p{};
  // int32 totals: every plane product is at most 127 * 128, so a row of <= 2^17 lifted
  // coordinates cannot overflow; the per-CTA whitening keeps blocks of at most 256 inputs
  if (batch < 1 || batch > bs::kMaxTokens || L > (1 << 17) || Bh > 256 || d > bs::kMaxD ||
      D > 32 || d * D > bs::kMaxMs)
    return p;
  p.nt = batch <= 2 ? 1 : batch <= 4 ? 2 : 4;
  p.nchunk = (int)((L + 511) / 512);
  const int sms = bs_sm_count();
  constexpr size_t kBudget = 224 * 1024;
  const int64_t row_bytes = ((L + 7) / 8 + 15) / 16 * 16;
  for (int S = 1; S <= 16; ++S) {
    const int sc = (p.nchunk + S - 1) / S;
    // the inputs a slice lifts, widened to whole Hadamard blocks
    const int span = (int)std::min<int64_t>(((int64_t)sc * 512 / D + 2) * d, (int64_t)K);
    const int xs = Bh > 0 ? ((span + Bh - 1) / Bh + 1) * Bh : span;
    const size_t prep =
        (((size_t)batch * xs + bs::kMaxMs + (size_t)bs::kWarps * bs::kZw) * 4 + 127) / 128 * 128;
    if (S > 1 && (p.nchunk + sc - 1) / sc != S) continue;   // no empty slice
    const int R = std::max(1, std::min(sms / S, (N + 15) / 16));
    const int rq = N / R;
    const int rows_max = rq + 1;
    const size_t frag = (size_t)sc * batch * bs::kTokBytes + bs::kZeroBytes;
    const size_t acc_bytes = (size_t)rows_max * 8 * p.nt * 4;
    const size_t fixed = frag + prep + acc_bytes;
    if (fixed > kBudget) continue;
    // stages: whole rows in one copy when S == 1 and the row stride permits a conflict-free
    // permutation; else one copy per row of a window (of the slice) at a padded stride.
    // 32 rows per stage when at least three such stages fit, else 16.
    const int64_t slice_bytes = std::min<int64_t>((int64_t)sc * 64, row_bytes);
    const bool whole = false;   // one copy per row: see the producer
    int wch = sc, stride = (int)row_bytes;
    {
      // windows of >= 2 KB per row copy (the cost of a copy is paid per row) but <= 4 KB
      const int64_t slice_chunks = (slice_bytes + 63) / 64;
      const int nwin = (int)std::max<int64_t>(1, (slice_chunks + 63) / 64);
      wch = (int)((slice_chunks + nwin - 1) / nwin);
      stride = padded_stride(wch * 64);
    }
    int rs = 0, NS = 0;
    for (int r : {32, 16}) {
      const size_t stage = (size_t)r * stride + 64;
      const int ns = (int)std::min<size_t>((kBudget - fixed) / stage, bs::kMaxStages);
      if (ns >= 3 || (r == 16 && ns >= 2)) {
        rs = r;
        NS = ns;
        break;
      }
    }
    if (rs == 0) continue;
    if (NS < 3 && S < 16) continue;   // a narrower slice leaves room for a deeper ring
    p.S = S;
    p.sc = sc;
    p.R = R;
    p.rq = rq;
    p.rrem = N % R;
    p.rows_max = rows_max;
    p.rows_per_stage = rs;
    p.wch = wch;
    p.stride = stride;
    p.whole = whole ? 1 : 0;
    p.perm = row_perm(stride);
    p.NS = NS;
    p.early_stages = 1;
    p.xs_floats = xs;
    p.frag_smem = frag;
    p.prep_smem = prep;
    p.smem = fixed + (size_t)NS * ((size_t)rs * stride + 64);
    p.ok = p.perm != 0;
    if (p.ok) break;
  }
  if (!p.ok) return p;
  p.nctas = p.S * p.R;
  p.sumz_bytes = p.S > 1 ? (size_t)p.S * batch * 4 : 0;
  p.gacc_bytes = p.S > 1 ? (size_t)batch * N * 4 * 4 : 0;
  return p;
}

template <int NT, int HT>
static cudaError_t launch_bs_nt(const BsPlan& pl, const BsParams& P, cudaStream_t st) {
  static int smem_set[64];
  cudaError_t e = ensure_smem((const void*)gemv_bs_kernel<NT, HT>, pl.smem, smem_set);
  if (e != cudaSuccess) return e;
  gemv_bs_kernel<NT, HT><<<pl.nctas, bs::kThreads, pl.smem, st>>>(P);
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
  P.rows_per_stage = pl.rows_per_stage;
  P.wch = pl.wch;
  P.stride = pl.stride;
  P.whole = pl.whole;
  P.NS = pl.NS;
  P.early_stages = pl.early_stages;
  P.perm = pl.perm;
  P.xs_floats = pl.xs_floats;
  P.rows_max = pl.rows_max;
  P.frag_bytes = pl.frag_smem;
  P.prep_bytes = pl.prep_smem;
  P.sumz = ws.sumz;
  P.gacc = ws.gacc;
  P.counters = ws.counters;
  P.status = ws.status;
  const bool h2 = pl.rows_per_stage == 32;
  switch (pl.nt) {
    case 1: return h2 ? launch_bs_nt<1, 2>(pl, P, st) : launch_bs_nt<1, 1>(pl, P, st);
    case 2: return h2 ? launch_bs_nt<2, 2>(pl, P, st) : launch_bs_nt<2, 1>(pl, P, st);
    default: return h2 ? launch_bs_nt<4, 2>(pl, P, st) : launch_bs_nt<4, 1>(pl, P, st);
  }
}

}  // namespace lq
