// lq_gemv_bs.cu -- decode GEMV for small batches (batch <= 8) with the stored codes staged
// through shared memory by TMA.
//
// y[t][n] = s[n] * sum_q b[n][q] z[t][q], b in {+1,-1}, z = lift(T(x[t])) (paper sec. 3 intro:
// o = diag(s) W (M T a); review "Method": an INT1 x FP product plus small linear maps, no lookup
// table). With b = 1 - 2*bit the row sum is sum_q z_q - 2 * (sum of z over the set bits).
//
// Two kernels per call, the second launched with programmatic dependent launch:
//  prep, one CTA per 512-coordinate chunk of the lifted dimension: a power of two S per token
//    from a bound on |z| over all of K (|xt_i| <= ||block of sign * scale * x||_2 times the
//    largest column 1-norm of M), so every chunk of a token shares one S; the whitening of the
//    Hadamard blocks that feed the chunk; the lift z = M^T xt per block of d inputs (a lane
//    keeps one column of M in registers and reads a block's inputs as broadcast loads); three
//    int8 planes (base 254) of the B operand of mma.m16n8k32 per bit slot of a code byte (see
//    the item below), stored in its register layout; and the chunk's sum of z.
//  gemv, S K-slices x R row ranges, one CTA per SM:
//   * one producer thread streams the CTA's rows into a ring of shared-memory stages (32 or 16
//     rows x a window of an odd number of 64-byte chunks) with 2-D TMA boxes of 8 rows. The
//     codes are inputs of the call, so the stream starts at once, while the prep still runs;
//   * the 16 compute warps wait for the prep grid, copy their slice's fragments into shared
//     memory with one bulk copy per token, then take the (stage rows, 64-byte chunk) items of
//     each stage in turn. A code byte v holds bits b_0..b_7 of eight coordinates; eight MMAs
//     per byte take as A the raw byte read as unsigned (slot 0) and as signed (slot 7: it
//     differs by 256 b_7) and, after one AND per code word, 2^q b_q alone (slots 1-6). The
//     prep picks the slots' B entries so that the eight products weigh bit p by z_p S (up to
//     rounding), and all slots accumulate into int32 sums (two chains by slot parity), exact
//     across the whole row: a byte adds at most 127 (255 + 128 + 126) per digit plane, so a row
//     of <= 2^17 coordinates stays below 2^31. At the end of a row group each warp adds its sums into the
//     CTA's per-row totals (integer shared-memory atomics, exact in any order). A stage row is
//     a whole number of chunks, an odd one, so its stride is 64 mod 128 bytes and the two rows
//     of a quarter-warp's 16-byte loads fall on disjoint banks;
//   * y = s * (sum z + sum_plane w_plane * total_plane), w_plane = -2 * 254^-plane / S. With
//     several K-slices the CTAs of a row range add their int32 totals into a global array and
//     the last one to finish writes y (and clears the array for the next call).
// Every sum is exact or runs in a fixed order: the result does not depend on timing.
#include <cuda.h>

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
constexpr int kBoxRows = 8;                    // rows of one TMA box
constexpr int kMaxWindow = 31;                 // chunks of a stage row (a box is <= 2 KB wide)
constexpr int kMaxD = 16;                      // inputs per block (d) the lift holds in registers
constexpr int kMaxMs = 512;                    // floats of M in shared memory (d * D <= 512)
constexpr int kZc = 512 + 4 * 8;               // floats of one token's z of a chunk (padded)
constexpr int kPrepThreads = 512;
constexpr int kPrepWarps = kPrepThreads / 32;
constexpr uint64_t kWaitNs = 1000000000ull;    // bounded waits: 1 s
}  // namespace bs

struct BsPrepParams {
  const void* x;
  int xdt;
  int batch;
  int K;
  Whiten T;
  const float* M;
  int d;
  int D;
  int64_t L;
  int nchunk;
  int xs_floats;   // whitened inputs of one chunk, per token
  uint8_t* frags;  // [batch][nchunk][kTokBytes]
  float* csum;     // [nchunk][batch] sum of z over each chunk
  float* stok;     // [batch] the power-of-two scale S of each token
};

struct BsParams {
  const uint8_t* frags;
  const float* csum;
  const float* stok;
  int batch;
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
  int wch;         // chunks per window (stage width); stage row stride = 64 * wch
  int NS;          // stages in the ring
  int rows_max;    // rq + 1
  size_t frag_bytes;   // shared memory: fragments of the slice [token][sc], then the zero block
  // global scratch (S > 1 only)
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

// Waits for the phase of `bar` with the given parity; false after kWaitNs. The clock is read
// once per 32 tries, so that a waiting warp takes few issue slots from the others.
__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity) {
  if (sm100::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtime();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (sm100::mbar_try_wait(bar, parity)) return true;
    if (gtime() - t0 > bs::kWaitNs) return false;
  }
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sm100::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}

// shared-memory integer add without a returned value
__device__ __forceinline__ void red_add_shared(int* p, int v) {
  asm volatile("red.shared.add.s32 [%0], %1;" ::"r"(sm100::smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// A as unsigned bytes (kSigned: as signed bytes), B signed bytes, int32 accumulators
template <bool kSigned = false>
__device__ __forceinline__ void imma(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                     uint32_t a3, uint32_t b0, uint32_t b1) {
  if (kSigned)
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
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

// z * S * 2^-p in units of 254^-2, rounded to the nearest integer (|z| * S < 64: below 2^22)
__device__ __forceinline__ int bs_units(float zs, int p) {
  return __float2int_rn(zs * __int_as_float((127 - p) << 23) * 64516.f);
}

// the three balanced base-254 digits of an integer c: c = 254^2 P0 + 254 P1 + P2, P1 and P2 in
// [-127, 126] (|c| < 2^23: |P0| <= 128 / 1.27)
__device__ __forceinline__ void bs_digits3(int c, int (&P)[3]) {
  int q = c + 127;
  q = q >= 0 ? q / 254 : -((253 - q) / 254);   // floor
  P[2] = c - 254 * q;
  int r = q + 127;
  r = r >= 0 ? r / 254 : -((253 - r) / 254);
  P[1] = q - 254 * r;
  P[0] = r;
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

// This thread's part of the largest squared block norm of token t over all of K (identity T:
// the largest x^2). With blocks of >= 8 inputs, warps w0 .. w0 + nw - 1 share the pass: lane l
// of the i-th of them takes the 8 inputs from 8 (32 i + l) + 256 nw r in round r (the loads of
// four rounds in flight together) and the Bh / 8 lanes of one block add their sums by
// shuffles. The caller reduces over the CTA.
// prep_block_norms for Hadamard blocks of fewer than 8 inputs (and the identity: the largest
// x^2), one block per thread; out of line, as the prep's usual path does not take it
template <int XDT>
__device__ __noinline__ float prep_norms_small(const void* x, int K, const Whiten T, int64_t off) {
  const int tid = threadIdx.x;
  const int Bh = T.block;
  float m = 0.f;
  if (Bh > 0) {
    for (int b = tid; b < K / Bh; b += bs::kPrepThreads) {
      float a = 0.f;
      for (int i = 0; i < Bh; ++i) {
        const int k = b * Bh + i;
        float v = load_as_f32(x, XDT, off + k);
        if (T.chan_scale) v *= __ldg(T.chan_scale + k);
        a = fmaf(v, v, a);
      }
      m = fmaxf(m, a);
    }
  } else {
    for (int k = tid; k < K; k += bs::kPrepThreads) {
      const float v = load_as_f32(x, XDT, off + k);
      m = fmaxf(m, v * v);
    }
  }
  return m;
}

template <int XDT>
__device__ __forceinline__ float prep_block_norms(const BsPrepParams& P, int t, int w0, int nw) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Bh = P.T.block;
  const int64_t off = (int64_t)t * P.K;
  float m = 0.f;
  if (Bh >= 8) {
    // warps w0 .. w0 + nw - 1 only; K is a multiple of Bh (<= 256), so a block's lanes are all
    // in range or all out
    if (warp < w0 || warp >= w0 + nw) return 0.f;
#pragma unroll 4
    for (int kw = 8 * 32 * (warp - w0); kw < P.K; kw += 8 * 32 * nw) {
      const int k = kw + 8 * lane;
      const bool in = k < P.K;
      float v[8];
      load8_as_f32(P.x, XDT, off + (in ? k : 0), 8, v);
      if (P.T.chan_scale) {
        float cs[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) cs[r] = __ldg(P.T.chan_scale + (in ? k : 0) + r);
#pragma unroll
        for (int r = 0; r < 8; ++r) v[r] *= cs[r];
      }
      float a = 0.f;
#pragma unroll
      for (int r = 0; r < 8; ++r) a = fmaf(v[r], v[r], a);
      for (int o = 1; o < Bh / 8 && o < 32; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (in) m = fmaxf(m, a);
    }
  } else {
    m = prep_norms_small<XDT>(P.x, P.K, P.T, off);
  }
  return m;
}

// One CTA per chunk; see the file comment.
// The whitening of a chunk's inputs for Hadamard blocks of fewer than 32 inputs (and the
// identity), by the whole CTA through shared memory. Kept out of line: the prep's usual path
// (blocks of >= 32 inputs, one warp each) then stays compact.
template <int XDT>
__device__ __noinline__ void prep_whiten_small(const void* x, int batch, int K, const Whiten T,
                                               int xs_floats, int base, int span, float* xs) {
  const int tid = threadIdx.x;
  const int Bh = T.block;
  for (int e = tid; e < batch * span; e += bs::kPrepThreads) {
    const int tok = e / span, i = e - tok * span;
    const int k = base + i;
    float a = 0.f;
    if (k < K) {
      a = load_as_f32(x, XDT, (int64_t)tok * K + k);
      if (Bh > 0) {
        if (T.chan_scale) a *= __ldg(T.chan_scale + k);
        if (T.sign && __ldg(T.sign + k) < 0) a = -a;
      }
    }
    xs[tok * xs_floats + i] = a;
  }
  __syncthreads();
  if (Bh > 1) {
    const int half = span / 2;
    for (int h = 1; h < Bh; h <<= 1) {
      for (int pp = tid; pp < batch * half; pp += bs::kPrepThreads) {
        const int tok = pp / half, pi = pp - tok * half;
        const int lo = pi & (h - 1);
        const int i = ((pi - lo) << 1) | lo;
        float* xt = xs + tok * xs_floats;
        const float a = xt[i], c2 = xt[i + h];
        xt[i] = a + c2;
        xt[i + h] = a - c2;
      }
      __syncthreads();
    }
    for (int e = tid; e < batch * span; e += bs::kPrepThreads) {
      const int tok = e / span;
      xs[tok * xs_floats + (e - tok * span)] *= T.inv_sqrt;
    }
  }
}

// TB >= batch: the token loops of the lift compile for TB tokens only, and XDT is the dtype of x:
// the prep runs once per call from a cold instruction cache, so it carries only the code it runs
template <int TB, int XDT>
__global__ void __launch_bounds__(bs::kPrepThreads) gemv_bs_prep_kernel(const BsPrepParams P) {
  // let the dependent GEMV grid launch now: it streams codes at once and waits for this grid
  // before it reads what this grid writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(16) float psm[];
  __shared__ float s_red[bs::kMaxTokens][bs::kPrepWarps];
  __shared__ float s_sum[bs::kMaxTokens][bs::kPrepWarps];
  __shared__ float s_tok[bs::kMaxTokens];
  __shared__ float s_cm;
  float* xs = psm;                                    // [batch][xs_floats]
  float* Ms = xs + (size_t)P.batch * P.xs_floats;     // [d][D]
  float* zc = Ms + bs::kMaxMs;                        // [batch][kZc]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int q0 = c * 512;
  const int qe = (int)min((int64_t)q0 + 512, P.L);
  const int gf = q0 / P.D, gl = (qe - 1) / P.D;
  const int k0 = gf * P.d, k1 = min((gl + 1) * P.d, P.K);
  const int Bh = P.T.block;
  int base = k0, span = k1 - k0;
  if (Bh > 0) {
    const int blk0 = k0 / Bh;
    base = blk0 * Bh;
    span = ((k1 + Bh - 1) / Bh - blk0) * Bh;
  }
  for (int i = tid; i < P.d * P.D; i += bs::kPrepThreads) Ms[i] = __ldg(P.M + i);
  // 1. the chunk's inputs, whitened: xt = H (sign * scale * x) / sqrt(Bh) per block (first, so
  // that its loads go out together with the norm pass's)
  if (Bh >= 32) {
    const int E = Bh >> 5;
    const int nblk = span / Bh;
    for (int task = warp; task < P.batch * nblk; task += bs::kPrepWarps) {
      const int tok = task / nblk, b = task - tok * nblk;
      warp_whiten_block(P.x, XDT, (int64_t)tok * P.K, base + b * Bh, E, P.T, P.T.inv_sqrt,
                        xs + tok * P.xs_floats + b * Bh);
    }
  } else {
    prep_whiten_small<XDT>(P.x, P.batch, P.K, P.T, P.xs_floats, base, span, xs);
  }
  // 2. every token's largest squared block norm over all of K, by the warps that whitened
  // nothing when that leaves at least half of them (their loads then go out with the
  // whitening's instead of after them)
  int w0 = 0;
  if (Bh >= 32) {
    const int tasks = P.batch * (span / Bh);
    if (tasks <= bs::kPrepWarps / 2) w0 = tasks;
  }
  for (int tok = 0; tok < P.batch; ++tok) {
    const float m = bs_warp_max(prep_block_norms<XDT>(P, tok, w0, bs::kPrepWarps - w0));
    if (lane == 0) s_red[tok][warp] = m;
  }
  __syncthreads();
  // the largest column 1-norm of M
  if (warp == 0) {
    float a = 0.f;
    if (lane < P.D)
      for (int i = 0; i < P.d; ++i) a += fabsf(Ms[i * P.D + lane]);
    a = bs_warp_max(a);
    if (lane == 0) s_cm = a;
  }
  __syncthreads();
  if (tid < P.batch) {
    float a = 0.f;
    for (int w = 0; w < bs::kPrepWarps; ++w) a = fmaxf(a, s_red[tid][w]);
    const float S = scale_from_bound(s_cm, a);
    s_tok[tid] = S;
    if (c == 0) P.stok[tid] = S;
  }
  // 3. the lift: lane -> (gi, j) = (lane / D, lane % D) for the first gpl * D lanes, gpl = 32 / D
  // groups at a time per warp; column j of M in registers, a group's d inputs broadcast
  const int gpl = 32 / P.D;
  const int gi = lane / P.D, jc = lane - gi * P.D;
  const bool lane_on = gi < gpl;
  float Mr[bs::kMaxD];
#pragma unroll
  for (int i = 0; i < bs::kMaxD; ++i) Mr[i] = (lane_on && i < P.d) ? Ms[i * P.D + jc] : 0.f;
  float su[TB];
#pragma unroll
  for (int t = 0; t < TB; ++t) su[t] = 0.f;
  if (lane_on) {
    for (int g = gf + warp * gpl + gi; g <= gl; g += bs::kPrepWarps * gpl) {
      const int kg = g * P.d;
      const int dv = min(P.d, P.K - kg);
      const int e = g * P.D + jc - q0;
      const bool in = e >= 0 && e < qe - q0;
#pragma unroll
      for (int tok = 0; tok < TB; ++tok) {
        if (tok >= P.batch) continue;
        const float* xt = xs + tok * P.xs_floats + (kg - base);
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < bs::kMaxD; ++i)
          if (i < dv) a = fmaf(Mr[i], xt[i], a);
        if (in) {
          zc[tok * bs::kZc + e + (e >> 7) * 8] = a;
          su[tok] += a;
        }
      }
    }
  }
  // the tail of the last chunk (past L) is zero
  for (int e = (qe - q0) + tid; e < 512; e += bs::kPrepThreads)
    for (int tok = 0; tok < P.batch; ++tok) zc[tok * bs::kZc + e + (e >> 7) * 8] = 0.f;
#pragma unroll
  for (int tok = 0; tok < TB; ++tok) {
    if (tok < P.batch) {
      const float v = bs_warp_sum(su[tok]);
      if (lane == 0) s_sum[tok][warp] = v;
    }
  }
  __syncthreads();
  // the chunk's sum of z, in a fixed order (lanes, then warps)
  if (tid < P.batch) {
    float a = 0.f;
    for (int w = 0; w < bs::kPrepWarps; ++w) a += s_sum[tid][w];
    P.csum[(int64_t)c * P.batch + tid] = a;
  }
  // 4. quantise: thread -> (token, group of the B-operand layout), group -> (slot, tt, h, j); its
  // 4 bytes e0 / 8 + i fill one word per plane. With I_p the code bit p's value z * S * 2^-p in
  // units of 254^-2, a byte's eight products come from six masked bytes (slots 1-6: B = I_q -
  // I_0) and the raw byte read twice: unsigned (slot 0, B = h) and signed (slot 7, B = I_0 - h),
  // h = (I_0 + I_7) / 2. Bit 0 then weighs I_0, bit q 2^q I_q and bit 7 128 (2h - I_0) = 2^7 I_7.
  for (int it = tid; it < P.batch * 128; it += bs::kPrepThreads) {
    const int tok = it >> 7, grp = it & 127;
    const int pl8 = grp & 7, tt = (grp >> 3) & 3, hl = (grp >> 5) & 1, jl = grp >> 6;
    const int e0 = 128 * tt + 64 * jl + 32 * hl;      // bit 0 of the group's first byte
    const float S = s_tok[tok];
    uint32_t w4[bs::kPlanes] = {};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float* zb = zc + tok * bs::kZc + (e0 + 8 * i) + ((e0 + 8 * i) >> 7) * 8;
      // I_0 rounds to the nearest integer of I_7's parity (one unit at most), so that h is
      // exact and bit 7 weighs I_7 itself: an odd sum would bias every set bit 7 by -128 units
      const int I7 = bs_units(zb[7] * S, 7);
      const float t0 = zb[0] * S * 64516.f;
      int I0 = __float2int_rn(t0);
      if ((I0 ^ I7) & 1) I0 += t0 > (float)I0 ? 1 : -1;
      const int h = (I0 + I7) >> 1;
      const int cq = pl8 == 0 ? h : pl8 == 7 ? I0 - h : bs_units(zb[pl8] * S, pl8) - I0;
      int Pq[bs::kPlanes];
      bs_digits3(cq, Pq);
#pragma unroll
      for (int pl = 0; pl < bs::kPlanes; ++pl) w4[pl] |= ((uint32_t)Pq[pl] & 0xffu) << (8 * i);
    }
    uint32_t* fw = reinterpret_cast<uint32_t*>(P.frags + ((size_t)tok * P.nchunk + c) * bs::kTokBytes);
    const int mma = jl * 8 + pl8;
#pragma unroll
    for (int pl = 0; pl < bs::kPlanes; ++pl)
      fw[((mma >> 1) * 12 + 4 * pl + tt) * 4 + (mma & 1) * 2 + hl] = w4[pl];
  }
}

// One item: the first HA of HT tiles of 16 rows (those that hold rows) x one 64-byte chunk, NT
// tiles of B (8 columns each), CH accumulator chains per (tile, B tile).
template <int NT, int HT, int CH, int HA>
__device__ __forceinline__ void run_item(uint32_t arow, int stride, uint32_t fb, const uint32_t (&fofs)[NT],
                                         uint32_t mstep, int (&acc)[NT][HT][CH][4]) {
  static_assert(HA >= 1 && HA <= HT, "tiles with rows");
  uint4 u[HA][2];
#pragma unroll
  for (int h = 0; h < HA; ++h) {
    u[h][0] = lds128(arow + (uint32_t)(16 * h * stride));
    u[h][1] = lds128(arow + (uint32_t)((16 * h + 8) * stride));
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
      // slots 0 and 7 take the raw bytes (unsigned, signed), slots 1-6 bit p alone
      const uint32_t msk = (p == 0 || p == 7) ? 0xffffffffu : 0x01010101u << p;
      const int ch = CH == 4 ? 2 * (m2 & 1) + e : CH == 2 ? e : 0;
#pragma unroll
      for (int h = 0; h < HA; ++h) {
        const uint32_t a0 = (j ? u[h][0].z : u[h][0].x) & msk, a2 = (j ? u[h][0].w : u[h][0].y) & msk;
        const uint32_t a1 = (j ? u[h][1].z : u[h][1].x) & msk, a3 = (j ? u[h][1].w : u[h][1].y) & msk;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint32_t b0 = e ? bv[nt].z : bv[nt].x, b1 = e ? bv[nt].w : bv[nt].y;
          if (p == 7)
            imma<true>(acc[nt][h][ch], a0, a1, a2, a3, b0, b1);
          else
            imma(acc[nt][h][ch], a0, a1, a2, a3, b0, b1);
        }
      }
    }
  }
}

// This warp's items of one stage: chunks first, first + 16, ... of the window.
template <int NT, int HT, int CH, int HA>
__device__ __forceinline__ void run_window(int first, int nitems, uint32_t fwin, uint32_t sbase, int stride,
                                           const uint32_t (&fofs)[NT], uint32_t zero_u32, uint32_t mstep,
                                           int (&acc)[NT][HT][CH][4]) {
  for (int cw = first; cw < nitems; cw += bs::kWarps) {
    const uint32_t fb = fwin + (uint32_t)cw * bs::kTokBytes;
    uint32_t fo[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) fo[nt] = fofs[nt] == 0xffffffffu ? zero_u32 - fb : fofs[nt];
    run_item<NT, HT, CH, HA>(sbase + 64 * cw, stride, fb, fo, mstep, acc);
  }
}

template <int NT, int HT>
__global__ void __launch_bounds__(bs::kThreads, 1)
    gemv_bs_kernel(const __grid_constant__ CUtensorMap tmap, const BsParams P) {
  // accumulator chains per (tile, B tile): two chains by bit-position parity for one or two B
  // tiles (four measured slower: more registers and more adds in every flush)
  constexpr int CH = NT <= 2 ? 2 : 1;
  constexpr int RS = 16 * HT;           // rows per stage
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[bs::kMaxStages], empty_bar[bs::kMaxStages];
  __shared__ __align__(8) uint64_t frag_bar;
  __shared__ float s_w[bs::kMaxTokens][bs::kPlanes];
  __shared__ float s_sumz[bs::kMaxTokens];
  __shared__ int s_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sl = blockIdx.x % P.S, ri = blockIdx.x / P.S;
  const int c0 = sl * P.sc;
  const int nc = min(P.sc, P.nchunk - c0);
  const int ra = ri * P.rq + min(ri, P.rrem);
  const int rows = P.rq + (ri < P.rrem ? 1 : 0);
  const int ngroups = (rows + RS - 1) / RS;
  const int nwin = (nc + P.wch - 1) / P.wch;
  const int nst = ngroups * nwin;
  const int stride = 64 * P.wch;

  const size_t stage_bytes = (size_t)RS * stride;
  uint8_t* frag_sm = smem;
  uint8_t* ring = smem + P.frag_bytes;
  int* rowacc = reinterpret_cast<int*>(ring + (size_t)P.NS * stage_bytes);   // [rows_max][8*NT]

  if (tid == 0) {
    for (int i = 0; i < P.NS; ++i) {
      sm100::mbar_init(&full_bar[i], 1);
      sm100::mbar_init(&empty_bar[i], bs::kWarps);
    }
    sm100::mbar_init(&frag_bar, 1);
    sm100::mbar_fence_init();
  }
  __syncthreads();

  if (warp == bs::kWarps) {
    // ---------------- producer: rows [ra, ra + rows), the slice's chunks, window by window, in
    // boxes of 8 rows (the boxes past the range's rows are not fetched; past N or past the end
    // of a row the box reads zeros)
    if (lane != 0) return;
    sm100::prefetch_tmap(&tmap);
    bool ok = true;
    for (int st = 0; st < nst && ok; ++st) {
      const int k = st % P.NS;
      if (st >= P.NS && !bar_wait(&empty_bar[k], ((st / P.NS) & 1) ^ 1)) {
        record_status(P.status, LQ_ETIMEOUT);
        ok = false;
        break;
      }
      const int grp = st / nwin, win = st - grp * nwin;
      const int r0 = grp * RS, nr = min(RS, rows - r0);
      const int nbox = (nr + bs::kBoxRows - 1) / bs::kBoxRows;
      uint8_t* dst = ring + (size_t)k * stage_bytes;
      sm100::mbar_arrive_expect_tx(&full_bar[k], (uint32_t)(nbox * bs::kBoxRows * stride));
      const int xc = (c0 + win * P.wch) * 8;   // in 8-byte elements: 64-byte aligned
      for (int b = 0; b < nbox; ++b)
        sm100::tma_load_2d(dst + (size_t)b * bs::kBoxRows * stride, &tmap, &full_bar[k], xc,
                           ra + r0 + b * bs::kBoxRows);
    }
    // no copy may still be in flight when the CTA exits: wait for the last stages to land
    for (int st = max(0, nst - P.NS); st < nst && ok; ++st)
      if (!bar_wait(&full_bar[st % P.NS], (st / P.NS) & 1)) record_status(P.status, LQ_ETIMEOUT);
    return;
  }

  // ---------------- compute warps: 1. the slice's fragments, written by the prep grid
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) {
    const uint32_t bytes = (uint32_t)nc * bs::kTokBytes;
    sm100::mbar_arrive_expect_tx(&frag_bar, bytes * (uint32_t)P.batch);
    for (int tok = 0; tok < P.batch; ++tok)
      bulk_g2s(frag_sm + (size_t)tok * P.sc * bs::kTokBytes,
               P.frags + ((size_t)tok * P.nchunk + c0) * bs::kTokBytes, bytes, &frag_bar);
  }
  if (tid < bs::kZeroBytes / 16)
    reinterpret_cast<uint4*>(frag_sm + P.frag_bytes - bs::kZeroBytes)[tid] = make_uint4(0, 0, 0, 0);
  for (int i = tid; i < P.rows_max * 8 * NT; i += bs::kCompute) rowacc[i] = 0;
  if (tid < P.batch) {
    const float S = __ldcg(P.stok + tid);
    s_w[tid][0] = -2.f / S;
    s_w[tid][1] = (float)(-2.0 / 254.0) / S;
    s_w[tid][2] = (float)(-2.0 / (254.0 * 254.0)) / S;
  }
  // the token's sum of z over every chunk, in a fixed order (lanes, then the lane tree)
  if (warp < P.batch && (P.S == 1)) {
    float a = 0.f;
    for (int c = lane; c < P.nchunk; c += 32) a += __ldcg(P.csum + (int64_t)c * P.batch + warp);
    a = bs_warp_sum(a);
    if (lane == 0) s_sumz[warp] = a;
  }
  if (!bar_wait(&frag_bar, 0) && tid == 0) record_status(P.status, LQ_ETIMEOUT);
  csync();

  // 2. main loop
  const int g = lane >> 2, t = lane & 3;
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
    fofs[nt] = live ? (uint32_t)((tk * P.sc * bs::kTokU4 + (lane & 15)) * 16) : 0xffffffffu;
  }
  constexpr uint32_t mstep = 192u;   // one MMA pair of a lane's B registers

  int acc[NT][HT][CH][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int h = 0; h < HT; ++h)
#pragma unroll
      for (int c = 0; c < CH; ++c) acc[nt][h][c][0] = acc[nt][h][c][1] = acc[nt][h][c][2] = acc[nt][h][c][3] = 0;

  // the stage's slot k and phase, row group and window advance without divisions; the items
  // of a stage are its window's chunks, dealt round-robin to the warps and continuing from one
  // stage to the next: this warp's first item of the stage is `first`
  int k = 0, ph = 0, grp = 0, win = 0, first = warp;
  for (int st = 0; st < nst; ++st) {
    const int nitems = min(P.wch, nc - win * P.wch);
    const int nr = min(RS, rows - grp * RS);
    if (!bar_wait(&full_bar[k], (uint32_t)ph)) {
      if (lane == 0) record_status(P.status, LQ_ETIMEOUT);
    }
    const uint32_t sbase = ring_u32 + (uint32_t)(k * stage_bytes) + (uint32_t)(g * stride + 16 * t);
    const uint32_t fwin = frag_u32 + (uint32_t)(win * P.wch) * bs::kTokBytes;
    // the stage's tiles of 16 rows that hold rows of the range
    const int live = (nr + 15) >> 4;
    if (live >= HT) {
      run_window<NT, HT, CH, HT>(first, nitems, fwin, sbase, stride, fofs, zero_u32, mstep, acc);
    } else {
      run_window<NT, HT, CH, 1>(first, nitems, fwin, sbase, stride, fofs, zero_u32, mstep, acc);
    }
    first = (first - nitems) & (bs::kWarps - 1);
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(&empty_bar[k]);
    // end of a row group: this warp's int32 sums into the CTA's per-row totals
    if (win == nwin - 1) {
      const int rbase = grp * RS;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < HT; ++h)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            int v = 0;
#pragma unroll
            for (int c = 0; c < CH; ++c) v += acc[nt][h][c][r];
            const int rr = rbase + 16 * h + g + 8 * (r >> 1);
            const int col = 2 * t + (r & 1);           // column within the tile
            const bool live = rr < rows && (col & 3) < bs::kPlanes && 2 * nt + (col >> 2) < P.batch;
            red_add_shared(&rowacc[min(rr, rows - 1) * 8 * NT + 8 * nt + col], live ? v : 0);
#pragma unroll
            for (int c = 0; c < CH; ++c) acc[nt][h][c][r] = 0;
          }
      ++grp;
      win = 0;
    } else {
      ++win;
    }
    if (++k == P.NS) {
      k = 0;
      ph ^= 1;
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
  if (warp < P.batch) {
    float a = 0.f;
    for (int c = lane; c < P.nchunk; c += 32) a += __ldcg(P.csum + (int64_t)c * P.batch + warp);
    a = bs_warp_sum(a);
    if (lane == 0) s_sumz[warp] = a;
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

// Chunks fetched past a slice of sc chunks read in windows of w: past the last slice they lie
// past the end of the row (the box reads zeros there, no traffic); inside they are the next
// slice's bytes, read for nothing.
int window_waste(int sc, int w) { return (sc + w - 1) / w * w - sc; }
}  // namespace

BsPlan plan_gemv_bs(int32_t batch, int64_t L, int32_t N, int32_t K, int32_t d, int32_t D,
                    int32_t Bh) {
  BsPlan p{};
  // int32 totals: every plane product is at most 127 * 128, so a row of <= 2^17 lifted
  // coordinates cannot overflow; the prep keeps blocks of at most 256 inputs
  if (batch < 1 || batch > bs::kMaxTokens || L > (1 << 17) || Bh > 256 || d > bs::kMaxD ||
      D > 32 || d * D > bs::kMaxMs)
    return p;
  (void)K;
  p.nt = batch <= 2 ? 1 : batch <= 4 ? 2 : 4;
  p.nchunk = (int)((L + 511) / 512);
  // the whitened inputs of one chunk: its groups' inputs widened to whole Hadamard blocks
  const int span = (512 / D + 2) * d;
  p.xs_floats = Bh > 0 ? ((span + Bh - 1) / Bh + 1) * Bh : span;
  p.prep_smem = ((size_t)batch * p.xs_floats + bs::kMaxMs + (size_t)batch * bs::kZc) * 4;
  if (p.prep_smem > 200 * 1024) return p;
  const int sms = bs_sm_count();
  constexpr size_t kBudget = 224 * 1024;
  // K-slices and stages: 32-row stages if any slicing leaves room for >= 3 of them, else 16-row
  // ones; the fewest slices (their cross-slice sum costs more than wider stages gain); then the
  // most useful bytes per stage (rows x the slice's chunks per window: the stage, not the byte,
  // carries the fixed cost of the loop). A window is an odd number of chunks (a row stride of 64
  // mod 128 bytes), at most kMaxWindow, at least 8 chunks where the slice has them; windows may
  // run past a slice by at most 1/32 of it (at least one chunk) inside the row, freely past its
  // end.
  for (int r : {32, 16}) {
    for (int S = 1; S <= 16 && !p.ok; ++S) {
      const int sc = (p.nchunk + S - 1) / S;
      if (S > 1 && (p.nchunk + sc - 1) / sc != S) continue;   // no empty slice
      const int R = std::max(1, std::min(sms / S, (N + 15) / 16));
      const int rq = N / R;
      const int rows_max = rq + 1;
      const size_t frag = (size_t)sc * batch * bs::kTokBytes + bs::kZeroBytes;
      const size_t acc_bytes = (size_t)rows_max * 8 * p.nt * 4;
      const size_t fixed = frag + acc_bytes;
      if (fixed > kBudget) continue;
      double best = 0.0;
      for (int w = 1; w <= bs::kMaxWindow; w += 2) {
        const int nwin = (sc + w - 1) / w;
        if (S > 1 && window_waste(sc, w) > std::max(1, sc / 32)) continue;
        const size_t stage = (size_t)r * 64 * w;
        const int NS = (int)std::min<size_t>((kBudget - fixed) / stage, bs::kMaxStages);
        if (NS < 3) continue;
        const double useful = (double)sc / nwin;
        if (useful < std::min(8, sc)) continue;   // box rows of >= 512 bytes stream at full rate
        if (useful > best) {
          best = useful;
          p.S = S;
          p.sc = sc;
          p.R = R;
          p.rq = rq;
          p.rrem = N % R;
          p.rows_max = rows_max;
          p.rows_per_stage = r;
          p.wch = w;
          p.stride = 64 * w;
          p.NS = NS;
          p.frag_smem = frag;
          p.smem = fixed + (size_t)NS * stage;
          p.ok = true;
        }
      }
    }
    if (p.ok) break;
  }
  if (!p.ok) return p;
  p.nctas = p.S * p.R;
  p.frag_bytes = (size_t)batch * p.nchunk * bs::kTokBytes;
  p.csum_bytes = (size_t)p.nchunk * batch * 4;
  p.stok_bytes = (size_t)batch * 4;
  p.gacc_bytes = p.S > 1 ? (size_t)batch * N * 4 * 4 : 0;
  return p;
}

template <int TB, int XDT>
static cudaError_t launch_prep_t(const BsPrepParams& Q, const BsPlan& pl, cudaStream_t st) {
  static int smem_set[64];
  cudaError_t e = ensure_smem((const void*)gemv_bs_prep_kernel<TB, XDT>, pl.prep_smem, smem_set);
  if (e != cudaSuccess) return e;
  gemv_bs_prep_kernel<TB, XDT><<<pl.nchunk, bs::kPrepThreads, pl.prep_smem, st>>>(Q);
  return cudaGetLastError();
}

template <int TB>
static cudaError_t launch_prep(const BsPrepParams& Q, const BsPlan& pl, cudaStream_t st) {
  if (Q.xdt == LQ_BF16) return launch_prep_t<TB, LQ_BF16>(Q, pl, st);
  if (Q.xdt == LQ_F16) return launch_prep_t<TB, LQ_F16>(Q, pl, st);
  return launch_prep_t<TB, LQ_F32>(Q, pl, st);
}

template <int NT, int HT>
static cudaError_t launch_bs_nt(const BsPlan& pl, const CUtensorMap& tmap, const BsParams& P,
                                cudaStream_t st) {
  static int smem_set[64];
  cudaError_t e = ensure_smem((const void*)gemv_bs_kernel<NT, HT>, pl.smem, smem_set);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.nctas);
  cfg.blockDim = dim3(bs::kThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemv_bs_kernel<NT, HT>, tmap, P);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemv_bs(const BsPlan& pl, const void* x, int xdt, int32_t batch, int32_t K,
                           Whiten T, const float* M, int32_t d, int32_t D, int64_t L,
                           const uint32_t* packed, int64_t row_bytes, int32_t N, const void* s,
                           int sdt, float* y, const BsScratch& ws, cudaStream_t st) {
  TensorMapEncodeFn enc = tensor_map_encode_fn();
  if (enc == nullptr) return cudaErrorNotSupported;
  // the codes as [N][row_bytes / 8] 8-byte elements; a box is 8 rows x one window
  CUtensorMap tmap;
  {
    const cuuint64_t gdim[2] = {(cuuint64_t)(row_bytes / 8), (cuuint64_t)N};
    const cuuint64_t gstride[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)(pl.wch * 8), (cuuint32_t)bs::kBoxRows};
    const cuuint32_t estride[2] = {1, 1};
    if (enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<uint32_t*>(packed), gdim, gstride,
            box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  BsPrepParams Q{};
  Q.x = x;
  Q.xdt = xdt;
  Q.batch = batch;
  Q.K = K;
  Q.T = T;
  Q.M = M;
  Q.d = d;
  Q.D = D;
  Q.L = L;
  Q.nchunk = pl.nchunk;
  Q.xs_floats = pl.xs_floats;
  Q.frags = ws.frags;
  Q.csum = ws.csum;
  Q.stok = ws.stok;
  cudaError_t e = batch <= 1 ? launch_prep<1>(Q, pl, st)
                  : batch <= 2 ? launch_prep<2>(Q, pl, st)
                  : batch <= 4 ? launch_prep<4>(Q, pl, st)
                               : launch_prep<bs::kMaxTokens>(Q, pl, st);
  if (e != cudaSuccess) return e;

  BsParams P{};
  P.frags = ws.frags;
  P.csum = ws.csum;
  P.stok = ws.stok;
  P.batch = batch;
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
  P.NS = pl.NS;
  P.rows_max = pl.rows_max;
  P.frag_bytes = pl.frag_smem;
  P.gacc = ws.gacc;
  P.counters = ws.counters;
  P.status = ws.status;
  const bool h2 = pl.rows_per_stage == 32;
  switch (pl.nt) {
    case 1: return h2 ? launch_bs_nt<1, 2>(pl, tmap, P, st) : launch_bs_nt<1, 1>(pl, tmap, P, st);
    case 2: return h2 ? launch_bs_nt<2, 2>(pl, tmap, P, st) : launch_bs_nt<2, 1>(pl, tmap, P, st);
    default: return h2 ? launch_bs_nt<4, 2>(pl, tmap, P, st) : launch_bs_nt<4, 1>(pl, tmap, P, st);
  }
}

}  // namespace lq
