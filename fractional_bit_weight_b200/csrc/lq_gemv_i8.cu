// lq_gemv_i8.cu -- decode GEMV for small batches (batch <= 8).
//
// y[t][n] = s[n] * sum_q b[n][q] z[t][q] with b in {+1,-1}, z = lift(T(x[t]))
// (paper sec. 3 intro: o = diag(s) W (M T a); review "Method": an INT1 x FP product plus small
// linear maps, with no lookup table). With b = 1 - 2*bit,
//     sum_q b_q z_q = sum_q z_q - 2 * sum_{q: bit_q = 1} z_q,
// so each row needs only the subset sum of z over its set bits.
//
// Two kernels per call, the second launched with programmatic dependent launch:
//  prep, one CTA per 512-bit chunk of the lifted dimension: whitens the Hadamard blocks that
//    feed the chunk (a warp per block: the first butterfly stages in registers, the rest with
//    lane shuffles), lifts them, z = M^T xt per block of d inputs, picks a power-of-two scale S
//    from max|z| of the chunk, and splits z*S*2^-p, p = q mod 8, into three int8 planes (base
//    254, ~23 bits, at least 16 of them kept at p = 7) stored in the register layout of the B
//    operand of mma.m16n8k32 (8 columns = 2 tokens x 4 plane slots, the fourth slot empty),
//    with the chunk's column weights -2*254^-plane/S and its sum of z.
//  gemv, S slices of chunks x R row ranges, one CTA each (one per SM): starts streaming its
//    stored bits into registers at once, waits for prep, copies its slice's fragments to shared
//    memory, then runs the (32-row tile pair, chunk) items of its rows, pair-major, in 16 equal
//    contiguous runs, one per warp. A 32-bit word of stored bits becomes an int8 A operand with
//    one AND, (w & 0x01010101 << p): bit p of each byte as 0 or 2^p; the B entries carry 2^-p,
//    so all eight bit positions accumulate into one int32 set per item, which the chunk's column
//    weights turn into fp32. Warps park the fp32 partial of every pair they touched in their own
//    shared-memory slot, summed in warp order at the end; with S > 1 the last CTA of a row range
//    to finish adds the slices in slice order and applies s.
// Fragments are computed once per call and every sum runs in a fixed order, so the result does
// not depend on timing.
#include "lq_device.cuh"

namespace lq {

namespace g8 {
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kPlanes = 3;                        // int8 planes per value (plane slot 3 empty)
// one token's B registers for one chunk: the 12 lanes 16*(token&1) + 4*plane + tt, 16 MMAs
constexpr int kTokLanes = 4 * kPlanes;
constexpr int kTokBytesPerChunk = 16 * kTokLanes * 8;   // 1536
constexpr int kMaxTokens = 8;
constexpr int kPrefetch = 4;                      // items of stored bits in flight per warp
constexpr int kMaxPairsPerWarp = 3;               // fp32 partial slots per warp
// With four token tiles (5..8 tokens) the slots and registers are four times larger: two slots
// per warp keep shared memory under the limit, two items in flight keep the registers in check.
__host__ __device__ constexpr int max_pairs(int nt) { return nt >= 4 ? 2 : kMaxPairsPerWarp; }
__host__ __device__ constexpr int prefetch(int nt) { return nt >= 4 ? 2 : kPrefetch; }
constexpr int kSlotFloatsPerNT = 2 * 32 * 4;      // one tile pair: 2 tiles x 32 lanes x 4 regs
}  // namespace g8

struct PrepParams {
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
  int sc;               // chunks per slice (fragments are stored slice by slice)
  int xs_floats;        // whitening scratch per token
  uint2* frags;         // [S][2*NT tokens][sc][16 MMAs][12 lanes]
  float* wtab;          // [nchunk][NT][8]
  float* csum;          // [nchunk][batch]
};

struct G8Params {
  const uint8_t* packed;
  int64_t row_bytes;
  int N;
  const void* s;
  int sdt;
  float* y;
  int batch;
  const uint2* frags;
  const float* wtab;
  const float* csum;
  float* partials;      // [S][batch][N] when S > 1
  uint32_t* counters;   // [R] when S > 1
  int nchunk;           // 512-bit chunks per row
  int sc;               // chunks per slice
  int S;                // slices
  int R;                // row ranges: range i has rq + (i < rrem) rows
  int rq, rrem;         // N / R and N % R
};

// d += A * B (no side effects: the compiler may schedule it freely)
__device__ __forceinline__ void imma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = A * B, the first MMA of an accumulation chain (C = 0)
__device__ __forceinline__ void imma_u8s8_first(int (&d)[4], uint32_t a0, uint32_t a1,
                                                uint32_t a2, uint32_t a3, uint32_t b0,
                                                uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};\n"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

__device__ __forceinline__ uint4 ldg_stream_v4(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// three int8 planes of base 254: a ~= P0 + P1/254 + P2/254^2 (|a| < 64)
__device__ __forceinline__ void planes3(float a, int (&P)[3]) {
  P[0] = __float2int_rn(a);
  float r = (a - (float)P[0]) * 254.f;
  P[1] = __float2int_rn(r);
  r = (r - (float)P[1]) * 254.f;
  P[2] = __float2int_rn(r);
}

constexpr int kPrepThreads = 512;
static_assert(kPrepThreads == 512, "the prep reductions assume 16 warps");

// One CTA per chunk; see the file comment.
template <int NT>
__global__ void __launch_bounds__(kPrepThreads) gemv_i8_prep_kernel(const PrepParams P) {
  // let the dependent gemv grid launch now; it waits for this grid before reading our output
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float s_red[2][g8::kMaxTokens][kPrepThreads / 32];
  __shared__ float s_scale[g8::kMaxTokens];
  float* xs = reinterpret_cast<float*>(smem);                       // [batch][xs_floats]
  float* zs = xs + (size_t)P.batch * P.xs_floats;                   // [batch][512 + pad]
  float* Ms = zs + (size_t)P.batch * 576;                           // [d][D]
  constexpr int kZP = 576;   // 512 values + 8 pad floats per 128 (bank-conflict-free reads)

  const int c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q0 = c * 512;                       // the plan keeps L below 2^30
  const int q1 = min(q0 + 512, (int)P.L);
  const int nq = q1 - q0;
  const int g_lo = q0 / P.D, g_hi = (q1 - 1) / P.D;
  const int k0 = g_lo * P.d;
  const int k1 = min((g_hi + 1) * P.d, P.K);
  const int Bh = P.T.block;
  int base = k0, span = k1 - k0;
  if (Bh > 0) {
    const int blk0 = k0 / Bh;
    base = blk0 * Bh;
    span = ((k1 + Bh - 1) / Bh - blk0) * Bh;
  }
  // M: copied by the highest threads first, which the warp-level whitening below leaves idle
  for (int i = kPrepThreads - 1 - tid; i < P.d * P.D; i += kPrepThreads) Ms[i] = P.M[i];
  // 1. whitened inputs of every token
  if (Bh >= 32 && Bh <= 256) {
    const int E = Bh >> 5;
    const int nblk = span / Bh;
    for (int task = warp; task < P.batch * nblk; task += kPrepThreads / 32) {
      const int tok = task / nblk, b = task - tok * nblk;
      warp_whiten_block(P.x, P.xdt, (int64_t)tok * P.K, base + b * Bh, E, P.T, 1.f,
                        xs + tok * P.xs_floats + b * Bh);
    }
    __syncthreads();
  } else {
    for (int e = tid; e < P.batch * span; e += kPrepThreads) {
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
    __syncthreads();
    if (Bh > 1) {
      const int half = span / 2;
      for (int h = 1; h < Bh; h <<= 1) {
        for (int pp = tid; pp < P.batch * half; pp += kPrepThreads) {
          const int tok = pp / half, pi = pp - tok * half;
          const int lo = pi & (h - 1);
          const int i = ((pi - lo) << 1) | lo;
          float* xt = xs + tok * P.xs_floats;
          const float a = xt[i], c2 = xt[i + h];
          xt[i] = a + c2;
          xt[i + h] = a - c2;
        }
        __syncthreads();
      }
    }
  }
  // 2. lift: thread tid owns value e = tid of every token; per-warp max and sum
  {
    const int e = tid;
    int gg = 0, jj = 0, dv = 0;
    if (e < nq) {
      const int qi = q0 + e;
      gg = qi / P.D;
      jj = qi - gg * P.D;
      dv = min(P.d, P.K - gg * P.d);
    }
    for (int tok = 0; tok < P.batch; ++tok) {
      float acc = 0.f;
      const float* xg = xs + tok * P.xs_floats + (gg * P.d - base);
      for (int ii = 0; ii < dv; ++ii) acc = fmaf(Ms[ii * P.D + jj], xg[ii], acc);
      acc *= P.T.inv_sqrt;
      zs[tok * kZP + e + 8 * (e >> 7)] = acc;
      float m = fabsf(acc), su = acc;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        su += __shfl_xor_sync(0xffffffffu, su, o);
      }
      if (lane == 0) {
        s_red[0][tok][warp] = m;
        s_red[1][tok][warp] = su;
      }
    }
  }
  __syncthreads();
  // warp w < 2*NT serves token slot w: the 16 warp maxima and sums reduced across lanes, the
  // power-of-two scale S (|z| * S < 64), the chunk's sum of z and its plane weights (the
  // empty fourth slot gets 0)
  if (warp < 2 * NT) {
    const int tok = warp;
    float m = 0.f, su = 0.f;
    if (tok < P.batch && lane < kPrepThreads / 32) {
      m = s_red[0][tok][lane];
      su = s_red[1][tok][lane];
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      su += __shfl_xor_sync(0xffffffffu, su, o);
    }
    int ex = 0;
    frexpf(m, &ex);                                         // m = f * 2^ex, f in [0.5, 1)
    const float S = m > 0.f ? ldexpf(1.f, 6 - ex) : 1.f;
    if (lane == 0 && tok < P.batch) {
      s_scale[tok] = S;
      P.csum[(int64_t)c * P.batch + tok] = su;
    }
    if (lane < 4) {
      float w = 0.f;
      if (tok < P.batch && lane < g8::kPlanes) {
        w = -2.f / S;
        for (int k = 0; k < lane; ++k) w *= (float)(1.0 / 254.0);
      }
      P.wtab[(int64_t)c * NT * 8 + (tok >> 1) * 8 + (tok & 1) * 4 + lane] = w;
    }
  }
  __syncthreads();
  // 3. quantise and store: thread -> (token, tt, j, h, p); its 4 values e0 + 8*i fill one
  // 32-bit word per plane: register h of lane 4*plane + tt for MMA (j, p) in the token's half
  // (only tokens < batch are stored; the GEMV gives absent tokens zero B registers)
  const int sl = c / P.sc, cl = c - sl * P.sc;
  for (int gi = tid; gi < P.batch * 128; gi += kPrepThreads) {
    const int tok = gi >> 7, grp = gi & 127;
    const int pl8 = grp & 7, tt = (grp >> 3) & 3, hl = (grp >> 5) & 1, jl = grp >> 6;
    uint32_t w4[g8::kPlanes] = {};
    {
      const float Sp = s_scale[tok] * __int_as_float((127 - pl8) << 23);   // S * 2^-p, exact
      const int e0 = 128 * tt + 64 * jl + 32 * hl + pl8;
      const float* zc = zs + tok * kZP + e0 + 8 * tt;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int Pq[g8::kPlanes];
        planes3(zc[8 * i] * Sp, Pq);
#pragma unroll
        for (int pl = 0; pl < g8::kPlanes; ++pl) w4[pl] |= ((uint32_t)Pq[pl] & 0xffu) << (8 * i);
      }
    }
    // token tok's block: register hl of lane 4*plane + tt (of the token's half) for MMA (j, p)
    uint32_t* fw = reinterpret_cast<uint32_t*>(P.frags) +
                   (((size_t)sl * 2 * NT + tok) * P.sc + cl) * (g8::kTokBytesPerChunk / 4);
#pragma unroll
    for (int pl = 0; pl < g8::kPlanes; ++pl)
      fw[((jl * 8 + pl8) * g8::kTokLanes + 4 * pl + tt) * 2 + hl] = w4[pl];
  }
}

template <int NT>
__global__ void __launch_bounds__(g8::kThreads, 1) gemv_i8_kernel(const G8Params P) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ float s_sumz[g8::kMaxTokens];
  __shared__ int s_pfirst[g8::kWarps];
  __shared__ int s_wrange[2][g8::kWarps * g8::kMaxPairsPerWarp];
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int sl = blockIdx.x % P.S, ri = blockIdx.x / P.S;
  const int c0 = sl * P.sc;
  const int nc = min(P.sc, P.nchunk - c0);
  // no divisions on the way to the first loads: row ranges from the host's N / R and N % R,
  // warp runs by a shift (16 warps)
  const int ra = ri * P.rq + min(ri, P.rrem);
  const int rb = ra + P.rq + (ri < P.rrem ? 1 : 0);
  const int npair = (rb - ra + 31) >> 5;
  const int items = npair * nc;
  static_assert(g8::kWarps == 16, "warp runs are computed with a shift by 4");
  const int i0 = (warp * items) >> 4;
  const int i1 = ((warp + 1) * items) >> 4;
  const int n = i1 - i0;
  const int pfirst = i0 / nc;

  constexpr int kSlotFloats = g8::kSlotFloatsPerNT * NT;
  constexpr int kTokU2 = g8::kTokBytesPerChunk / 8;                   // uint2 per token-chunk
  uint2* sfr = reinterpret_cast<uint2*>(smem);                        // [batch][sc][16][12]
  uint2* zblk = sfr + (size_t)P.batch * P.sc * kTokU2;                // 256 zeros
  float* slots = reinterpret_cast<float*>(zblk + 256);
  constexpr int kMP = g8::max_pairs(NT), kPF = g8::prefetch(NT);
  float* wts = slots + (size_t)g8::kWarps * kMP * kSlotFloats;                  // [sc][NT][8]

  // ---- 1. start streaming: item i = (pair i / nc, chunk c0 + i % nc)
  const int64_t last_off = P.row_bytes - 16;
  int lpr = pfirst, lc = i0 - pfirst * nc;       // position of the next item to load
  const uint8_t* rowp[4];
  auto set_rows = [&](int pr) {
    const int r = ra + pr * 32 + g;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int row = r + 8 * k;
      rowp[k] = P.packed + (int64_t)(row < rb ? row : ra) * P.row_bytes + 16 * t;
    }
  };
  auto load_next = [&](uint4 (&u)[4]) {
    int64_t off = (int64_t)(c0 + lc) * 64;
    off = off + 16 * t > last_off ? last_off - 16 * t : off;   // last chunk: stay in the row
    // rows past the range read row ra; their sums are computed but never stored
    u[0] = ldg_stream_v4(rowp[0] + off);
    u[1] = ldg_stream_v4(rowp[1] + off);
    u[2] = ldg_stream_v4(rowp[2] + off);
    u[3] = ldg_stream_v4(rowp[3] + off);
    if (++lc == nc) {
      lc = 0;
      if (++lpr < npair) set_rows(lpr);
    }
  };
  if (n > 0) set_rows(lpr);
  uint4 q[kPF][4];
#pragma unroll
  for (int k = 0; k < kPF; ++k)
    if (k < n) load_next(q[k]);
  if (lane == 0) s_pfirst[warp] = pfirst;
  // the row scale of this thread's first output (element e = tid: row ra + tid % rows), loaded
  // now so that the epilogue does not wait for it
  const int rows = rb - ra;
  const float sv0 = tid < rows * P.batch ? load_as_f32(P.s, P.sdt, ra + tid % rows) : 0.f;

  // ---- 2. this slice's fragments and column weights (written by the prep kernel)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  {
    // the blocks of tokens 0 .. batch-1 are a contiguous prefix of the slice's fragments
    const int nvec = P.batch * P.sc * g8::kTokBytesPerChunk / 16;
    const uint4* src = reinterpret_cast<const uint4*>(P.frags) +
                       (size_t)sl * 2 * NT * P.sc * g8::kTokBytesPerChunk / 16;
    uint4* dst = reinterpret_cast<uint4*>(sfr);
    for (int i = tid; i < nvec; i += g8::kThreads) {
      const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst + i);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src + i) : "memory");
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
    if (tid < 128) reinterpret_cast<uint4*>(zblk)[tid] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = tid; i < nc * NT * 8; i += g8::kThreads) wts[i] = P.wtab[(size_t)c0 * NT * 8 + i];
    if (warp < P.batch) {   // warp t: this slice's sum of z of token t, one load per lane
      float a = 0.f;
      for (int c = lane; c < nc; c += 32) a += P.csum[(int64_t)(c0 + c) * P.batch + warp];
      a = warp_sum(a);
      if (lane == 0) s_sumz[warp] = a;
    }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  }
  __syncthreads();

  // ---- 3. main loop
  float accf[2][NT][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      accf[a][nt][0] = accf[a][nt][1] = accf[a][nt][2] = accf[a][nt][3] = 0.f;
  int ppr = pfirst, pc = i0 - pfirst * nc;         // position of the next item to process
  // this lane's B registers in tile nt: token 2*nt + (lane >> 4), entry lane & 15 of that
  // token's half; a token past the batch reads the zero block at every chunk
  const uint2* fbase[NT];
  int fstride[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tk = 2 * nt + (lane >> 4);
    const bool live = tk < P.batch && (lane & 15) < g8::kTokLanes;
    fbase[nt] = (live ? sfr + (size_t)tk * P.sc * kTokU2 : zblk) + (lane & 15);
    fstride[nt] = live ? kTokU2 : 0;
  }
  auto park = [&]() {
    float* sp = slots + ((size_t)(warp * kMP + (ppr - pfirst)) * 2 * 32 + lane) * 4 * NT;
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        *reinterpret_cast<float4*>(sp + a * 32 * 4 * NT + nt * 4) =
            make_float4(accf[a][nt][0], accf[a][nt][1], accf[a][nt][2], accf[a][nt][3]);
        accf[a][nt][0] = accf[a][nt][1] = accf[a][nt][2] = accf[a][nt][3] = 0.f;
      }
  };
  auto process = [&](const uint4 (&u)[4]) {
    // one accumulation chain per (tile nt, 16-row half a); the masked A registers of each
    // (k-half j, bit p) are shared by all tiles
    int ac[NT][2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t a0 = j ? u[0].z : u[0].x, a2 = j ? u[0].w : u[0].y;
      const uint32_t a1 = j ? u[1].z : u[1].x, a3 = j ? u[1].w : u[1].y;
      const uint32_t b0 = j ? u[2].z : u[2].x, b2 = j ? u[2].w : u[2].y;
      const uint32_t b1 = j ? u[3].z : u[3].x, b3 = j ? u[3].w : u[3].y;
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const uint32_t msk = 0x01010101u << p;
        const uint32_t m0 = a0 & msk, m1 = a1 & msk, m2 = a2 & msk, m3 = a3 & msk;
        const uint32_t n0 = b0 & msk, n1 = b1 & msk, n2 = b2 & msk, n3 = b3 & msk;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint2 bv = fbase[nt][pc * fstride[nt] + (j * 8 + p) * g8::kTokLanes];
          if (j == 0 && p == 0) {
            imma_u8s8_first(ac[nt][0], m0, m1, m2, m3, bv.x, bv.y);
            imma_u8s8_first(ac[nt][1], n0, n1, n2, n3, bv.x, bv.y);
          } else {
            imma_u8s8(ac[nt][0], m0, m1, m2, m3, bv.x, bv.y);
            imma_u8s8(ac[nt][1], n0, n1, n2, n3, bv.x, bv.y);
          }
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float2 w = *reinterpret_cast<const float2*>(wts + (pc * NT + nt) * 8 + 2 * t);
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        accf[a][nt][0] = fmaf((float)ac[nt][a][0], w.x, accf[a][nt][0]);
        accf[a][nt][1] = fmaf((float)ac[nt][a][1], w.y, accf[a][nt][1]);
        accf[a][nt][2] = fmaf((float)ac[nt][a][2], w.x, accf[a][nt][2]);
        accf[a][nt][3] = fmaf((float)ac[nt][a][3], w.y, accf[a][nt][3]);
      }
    }
    // end of this pair's chunks: park the pair's partial in the warp's slot
    if (++pc == nc) {
      pc = 0;
      park();
      ++ppr;
    }
  };

  for (int kb = 0; kb < n; kb += kPF) {
#pragma unroll
    for (int k = 0; k < kPF; ++k) {
      if (kb + k < n) {
        process(q[k]);
        if (kb + k + kPF < n) load_next(q[k]);
      }
    }
  }
  if (n > 0 && pc != 0) park();   // the run ended inside a pair
  if (n == 0) {
    // an empty run (fewer items than warps) can fall inside a pair's warp range: its first
    // slot, the one the pair maps to, reads as zero
    float* sp = slots + (size_t)warp * kMP * kSlotFloats;
    for (int i = lane; i < kSlotFloats; i += 32) sp[i] = 0.f;
  }
  // warps whose runs overlap pair pr: first w with ((w+1)*items)>>4 > pr*nc, last w with
  // (w*items)>>4 < (pr+1)*nc
  for (int pr = tid; pr < npair; pr += g8::kThreads) {
    s_wrange[0][pr] = (16 * (pr * nc + 1) + items - 1) / items - 1;
    s_wrange[1][pr] = (16 * (pr + 1) * nc + items - 1) / items - 1;
  }
  __syncthreads();

  // ---- 4. per (row, token): this slice's value = its sum of z + warps' partials in warp order
  for (int e = tid; e < rows * P.batch; e += g8::kThreads) {
    const int tok = e / rows;
    const int rr = e - tok * rows;
    const int pr = rr >> 5, a = (rr >> 4) & 1, r = rr & 15;
    const int nt = tok >> 1, cb = (tok & 1) * 4;
    // the four plane columns of (row, token) in a parked C fragment
    int off[4];
#pragma unroll
    for (int pl = 0; pl < 4; ++pl) {
      const int col = cb + pl;
      off[pl] = (4 * (r & 7) + (col >> 1)) * 4 * NT + nt * 4 + 2 * (r >> 3) + (col & 1);
    }
    const int wlo = s_wrange[0][pr], whi = s_wrange[1][pr];
    float v = 0.f;
#pragma unroll 4
    for (int w = wlo; w <= whi; ++w) {
      const float* sp =
          slots + ((size_t)(w * kMP + (pr - s_pfirst[w])) * 2 + a) * 32 * 4 * NT;
      v += (sp[off[0]] + sp[off[1]]) + (sp[off[2]] + sp[off[3]]);
    }
    const int row = ra + rr;
    const float part = s_sumz[tok] + v;
    if (P.S == 1)
      P.y[(int64_t)tok * P.N + row] = (e == tid ? sv0 : load_as_f32(P.s, P.sdt, row)) * part;
    else
      P.partials[((int64_t)sl * P.batch + tok) * P.N + row] = part;
  }
  if (P.S == 1) return;

  // ---- cross-slice completion by the last CTA of this row range (one fence and one atomic,
  // by thread 0, after the barrier that orders the CTA's partial stores before them)
  __syncthreads();
  uint32_t* ctr = P.counters + ri;
  if (tid == 0) {
    __threadfence();
    const bool last = atomicAdd(ctr, 1u) == (uint32_t)(P.S - 1);
    if (last) __threadfence();
    s_last = last;
  }
  __syncthreads();
  if (!s_last) return;
  for (int e = tid; e < rows * P.batch; e += g8::kThreads) {
    const int tok = e / rows;
    const int row = ra + (e - tok * rows);
    const float sv = e == tid ? sv0 : load_as_f32(P.s, P.sdt, row);
    const float* pp = P.partials + (int64_t)tok * P.N + row;
    const int64_t stride = (int64_t)P.batch * P.N;
    // slices added in slice order; eight loads in flight per step
    float a = 0.f;
    for (int k0 = 0; k0 < P.S; k0 += 8) {
      float pk[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) pk[j] = k0 + j < P.S ? __ldcg(pp + (k0 + j) * stride) : 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) a += pk[j];
    }
    P.y[(int64_t)tok * P.N + row] = sv * a;
  }
  if (tid == 0) *ctr = 0u;   // ready for the next call on this workspace
}

// ------------------------------------------------------------------ host side

static int sm_count() {
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

G8Plan plan_gemv_i8(int32_t batch, int64_t L, int32_t N, int32_t K, int32_t d, int32_t D,
                    int32_t Bh) {
  (void)K;
  G8Plan p{};
  p.ok = batch >= 1 && batch <= g8::kMaxTokens && L <= (int64_t)1 << 30 && d * D <= 1024;
  if (!p.ok) return p;
  const int ntok = (batch + 1) / 2;
  p.nt = ntok <= 1 ? 1 : ntok <= 2 ? 2 : 4;
  p.nchunk = (int)((L + 511) / 512);
  const int sms = sm_count();
  auto smem_of = [&](int sc) {
    return (size_t)batch * sc * g8::kTokBytesPerChunk + 256 * 8 +
           (size_t)g8::kWarps * g8::max_pairs(p.nt) * g8::kSlotFloatsPerNT * p.nt * 4 +
           (size_t)sc * p.nt * 8 * 4;
  };
  // a warp's run must touch at most max_pairs(nt) pairs: ceil(npair/16) + 1 <= max_pairs(nt)
  auto pairs_ok = [&](int R) {
    const int npair = ((N + R - 1) / R + 31) / 32;
    return (npair + g8::kWarps - 1) / g8::kWarps + 1 <= g8::max_pairs(p.nt);
  };
  // Slices of about 30 KB of fragments (20 chunks of one token): every CTA of a slice copies
  // them from L2, which costs more than the cross-slice sums beyond that size. Where that
  // leaves more rows per CTA than the warps' partial slots hold, the slices widen (fewer
  // slices, so more row ranges) until the rows fit or the fragments outgrow shared memory.
  p.ok = false;
  for (int sc = std::min(std::max(1, 20 / batch), p.nchunk); sc <= p.nchunk; ++sc) {
    const int S = (p.nchunk + sc - 1) / sc;
    const int R = std::max(1, std::min(sms / std::min(S, sms), (N + 31) / 32));
    const int scs = (p.nchunk + S - 1) / S;
    if (smem_of(scs) > 220 * 1024) break;
    if (!pairs_ok(R)) continue;
    p.S = S;
    p.sc = scs;
    p.R = R;
    p.ok = true;
    break;
  }
  if (!p.ok) return p;
  p.nctas = p.S * p.R;
  p.smem = smem_of(p.sc);
  const int span = (512 / D + 2) * d;
  p.xs_floats = Bh > 0 ? ((span + Bh - 1) / Bh + 1) * Bh : span;
  p.prep_smem = ((size_t)batch * p.xs_floats + (size_t)batch * 576 + 1024) * 4;
  p.frag_bytes = (size_t)p.S * 2 * p.nt * p.sc * g8::kTokBytesPerChunk;
  p.wtab_bytes = (size_t)p.nchunk * p.nt * 8 * 4;
  p.csum_bytes = (size_t)p.nchunk * batch * 4;
  p.ok = p.ok && p.smem <= 220 * 1024 && p.prep_smem <= 200 * 1024;
  return p;
}

template <int NT>
static cudaError_t launch_nt(const G8Plan& pl, const PrepParams& Q, const G8Params& P,
                             cudaStream_t st) {
  static int prep_set[64], smem_set[64];
  cudaError_t e = ensure_smem((const void*)gemv_i8_prep_kernel<NT>, pl.prep_smem, prep_set);
  if (e != cudaSuccess) return e;
  e = ensure_smem((const void*)gemv_i8_kernel<NT>, pl.smem, smem_set);
  if (e != cudaSuccess) return e;
  // the prep kernel is an ordinary launch (launched with programmatic dependence on the
  // previous call's GEMV it measured slower); the GEMV is launched with programmatic dependence
  // on the prep kernel, so its CTAs start streaming stored bits while the prep runs
  gemv_i8_prep_kernel<NT><<<pl.nchunk, kPrepThreads, pl.prep_smem, st>>>(Q);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.nctas);
  cfg.blockDim = dim3(g8::kThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemv_i8_kernel<NT>, P);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemv_i8(const G8Plan& pl, const void* x, int xdt, int32_t batch, int32_t K,
                           Whiten T, const float* M, int32_t d, int32_t D, int64_t L,
                           const uint32_t* packed, int64_t row_bytes, int32_t N, const void* s,
                           int sdt, float* y, void* scratch, float* partials,
                           uint32_t* counters, cudaStream_t st) {
  uint8_t* sp = static_cast<uint8_t*>(scratch);
  PrepParams Q{};
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
  Q.sc = pl.sc;
  Q.xs_floats = pl.xs_floats;
  Q.frags = reinterpret_cast<uint2*>(sp);
  Q.wtab = reinterpret_cast<float*>(sp + pl.frag_bytes);
  Q.csum = reinterpret_cast<float*>(sp + pl.frag_bytes + pl.wtab_bytes);
  G8Params P{};
  P.packed = reinterpret_cast<const uint8_t*>(packed);
  P.row_bytes = row_bytes;
  P.N = N;
  P.s = s;
  P.sdt = sdt;
  P.y = y;
  P.batch = batch;
  P.frags = Q.frags;
  P.wtab = Q.wtab;
  P.csum = Q.csum;
  P.partials = partials;
  P.counters = counters;
  P.nchunk = pl.nchunk;
  P.sc = pl.sc;
  P.S = pl.S;
  P.R = pl.R;
  P.rq = N / pl.R;
  P.rrem = N % pl.R;
  switch (pl.nt) {
    case 1: return launch_nt<1>(pl, Q, P, st);
    case 2: return launch_nt<2>(pl, Q, P, st);
    default: return launch_nt<4>(pl, Q, P, st);
  }
}

}  // namespace lq
