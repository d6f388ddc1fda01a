// lq_encode.cu -- nearest-codeword encoding of weight blocks (the inner minimisation of Eq. (1)
// of the paper, sec. 3.1: w ~= M b, b in {+1,-1}^D, for every length-d block w of a row).
//
// Two searches, both deterministic:
//  exact:  all 2^D codewords (D <= 24);
//  seeded: the review's pseudo-inverse initialisation ("Method"; its "Limitations" put the
//          practical cap at D - d <= 20), read as: the first d coordinates are solved, the
//          other D - d enumerated. For every free part f (b_{d+k} = -1 exactly when bit k of f
//          is set) u = M_S^-1 (w - M_F b_F) with M_S = M[:, 0..d), M_F = M[:, d..D), and
//          b_i = +1 when u_i >= 0, else -1 (i < d).
// The winner is the candidate with the smallest ||w - M b||^2, ties keeping the smallest index
// (codeword c, or free part f).
//
// One warp per block (persistent CTAs take blocks round-robin). The 32 lanes split the
// candidates into contiguous ranges of 2^(bits-5) and walk each range in Gray-code order, so
// one coordinate flips per step and the residual r = w - M b (exact) or r_F = w - M_F b_F,
// u = M_S^-1 r_F and e = r_F - M_S b_S (seeded) change by one column each, d operations per
// step instead of d^2: u moves by a column of P = M_S^-1 M_F, e by the same column of M_F plus
// one column of M_S for every solved sign that flips. For d <= 10 the seeded walk instead reads
// e = r_F - T[b_S] from a shared-memory table of M_S b_S over all 2^d solved sign patterns. Every 256 steps the lane recomputes its
// state from the definition, which bounds fp32 drift. The warp then takes the minimum of
// (distance, index) over its lanes. Arithmetic is fp32; where two candidates lie within fp32
// rounding of each other the pick may differ from an fp64 search, never its distance by more
// than that rounding.
#include "lq_device.cuh"

namespace lq {
namespace enc {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxd = 16;
constexpr int kRefresh = 256;   // steps between exact recomputations of a lane's state

struct Params {
  const float* w;    // [N][K]
  int64_t N;
  int K, d, D, G;
  const float* M;    // [d][D]
  int8_t* b;         // [N][G][D]
  float* err;        // [N][G] or nullptr
};

// Shared tables, zero beyond d rows / columns so that loops may run to the template size. The
// walks read one column per step, the same for every lane of a warp: the column-major copies
// CM and CP serve those reads as 16-byte broadcast loads.
struct __align__(16) Tables {
  float CM[32][kMaxd];      // CM[j][i] = M[i][j]
  float CP[32][kMaxd];      // CP[k][i] = P[i][k] (seeded)
  float M[kMaxd][32];       // M, [i][j]
  float Minv[kMaxd][kMaxd]; // M_S^-1 (seeded)
  float P[kMaxd][32];       // M_S^-1 M_F, [i][k] (seeded)
  float A[kMaxd][2 * kMaxd];// Gauss-Jordan scratch
  int singular;
};

// column j of a column-major table (kMaxd floats, 16-byte aligned) into registers
template <int DM>
__device__ __forceinline__ void load_column(const float* col, float (&v)[DM]) {
  const float4* c4 = reinterpret_cast<const float4*>(col);
#pragma unroll
  for (int q = 0; q < (DM + 3) / 4; ++q) {
    const float4 a = c4[q];
    if (4 * q + 0 < DM) v[4 * q + 0] = a.x;
    if (4 * q + 1 < DM) v[4 * q + 1] = a.y;
    if (4 * q + 2 < DM) v[4 * q + 2] = a.z;
    if (4 * q + 3 < DM) v[4 * q + 3] = a.w;
  }
}

// M_S^-1 by Gauss-Jordan with partial pivoting (one thread; d <= 16), then P = M_S^-1 M_F.
__device__ void build_tables(const Params& p, Tables& t) {
  const int tid = threadIdx.x;
  for (int e = tid; e < kMaxd * 32; e += blockDim.x) {
    const int i = e >> 5, j = e & 31;
    t.M[i][j] = (i < p.d && j < p.D) ? p.M[i * p.D + j] : 0.f;
    t.P[i][j] = 0.f;
  }
  for (int e = tid; e < kMaxd * kMaxd; e += blockDim.x) t.Minv[e / kMaxd][e % kMaxd] = 0.f;
  __syncthreads();
  if (tid == 0) {
    const int d = p.d;
    int singular = 0;
    for (int i = 0; i < d; ++i)
      for (int c = 0; c < 2 * d; ++c) t.A[i][c] = c < d ? t.M[i][c] : (c - d == i ? 1.f : 0.f);
    for (int c = 0; c < d && !singular; ++c) {
      int piv = c;
      for (int i = c + 1; i < d; ++i)
        if (fabsf(t.A[i][c]) > fabsf(t.A[piv][c])) piv = i;
      if (t.A[piv][c] == 0.f) {
        singular = 1;
        break;
      }
      if (piv != c)
        for (int k = 0; k < 2 * d; ++k) {
          const float tmp = t.A[c][k];
          t.A[c][k] = t.A[piv][k];
          t.A[piv][k] = tmp;
        }
      const float inv = 1.f / t.A[c][c];
      for (int k = 0; k < 2 * d; ++k) t.A[c][k] *= inv;
      for (int i = 0; i < d; ++i)
        if (i != c) {
          const float m = t.A[i][c];
          if (m != 0.f)
            for (int k = 0; k < 2 * d; ++k) t.A[i][k] = fmaf(-m, t.A[c][k], t.A[i][k]);
        }
    }
    t.singular = singular;
    if (!singular)
      for (int i = 0; i < d; ++i)
        for (int c = 0; c < d; ++c) t.Minv[i][c] = t.A[i][d + c];
  }
  __syncthreads();
  const int F = p.D - p.d;
  for (int e = tid; e < p.d * F; e += blockDim.x) {
    const int i = e / F, k = e - i * F;
    float a = 0.f;
    for (int c = 0; c < p.d; ++c) a = fmaf(t.Minv[i][c], t.M[c][p.d + k], a);
    t.P[i][k] = a;
  }
  __syncthreads();
  for (int e = tid; e < 32 * kMaxd; e += blockDim.x) {
    const int j = e / kMaxd, i = e - j * kMaxd;
    t.CM[j][i] = t.M[i][j];
    t.CP[j][i] = t.P[i][j];
  }
  __syncthreads();
}

__device__ __forceinline__ void warp_argmin(float& dist, uint32_t& idx) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float od = __shfl_xor_sync(0xffffffffu, dist, o);
    const uint32_t oi = __shfl_xor_sync(0xffffffffu, idx, o);
    if (od < dist || (od == dist && oi < idx)) {
      dist = od;
      idx = oi;
    }
  }
}

// Exhaustive search over the 2^D codewords of one block (w in registers, DM >= d).
template <int DM>
__device__ void search_exact(const Params& p, const Tables& t, const float (&w)[DM], int lane,
                             float& best_dist, uint32_t& best_code) {
  const int D = p.D;
  const int lg = D >= 5 ? D - 5 : 0;                 // log2 of each lane's range
  const uint32_t cnt = 1u << lg;
  best_dist = INFINITY;
  best_code = 0xffffffffu;
  if (D < 5 && lane >= (1 << D)) return;
  const uint32_t c0 = (uint32_t)lane << lg;
  float r[DM];
  uint32_t code = c0;
  for (uint32_t s = 0; s < cnt; ++s) {
    if ((s & (kRefresh - 1)) == 0) {               // state from the definition
      const volatile float* Mv = &t.M[0][0];
#pragma unroll
      for (int i = 0; i < DM; ++i) {
        float a = w[i];
        for (int j = 0; j < D; ++j) a -= Mv[i * 32 + j] * (((code >> j) & 1) ? -1.f : 1.f);
        r[i] = a;
      }
    }
    float dist = 0.f;
#pragma unroll
    for (int i = 0; i < DM; ++i) dist = fmaf(r[i], r[i], dist);
    if (dist < best_dist || (dist == best_dist && code < best_code)) {
      best_dist = dist;
      best_code = code;
    }
    if (s + 1 < cnt) {                              // flip coordinate ctz(s+1): b_j -> -b_j
      const int j = __ffs(s + 1) - 1;
      const float sg2 = ((code >> j) & 1) ? -2.f : 2.f;
      float cj[DM];
      load_column<DM>(t.CM[j], cj);
#pragma unroll
      for (int i = 0; i < DM; ++i) r[i] = fmaf(sg2, cj[i], r[i]);
      code ^= 1u << j;
    }
  }
}

// Seeded search over the 2^(D-d) free parts of one block.
template <int DM>
__device__ void search_seeded(const Params& p, const Tables& t, const float (&w)[DM], int lane,
                              float& best_dist, uint32_t& best_f, uint32_t& best_mask) {
  const int d = p.d, F = p.D - p.d;
  const int lg = F >= 5 ? F - 5 : 0;
  const uint32_t cnt = 1u << lg;
  best_dist = INFINITY;
  best_f = 0xffffffffu;
  best_mask = 0;
  if (F < 5 && lane >= (1 << F)) return;
  float u[DM], e[DM];
  uint32_t f = (uint32_t)lane << lg, mask = 0;      // mask bit i: b_i = -1 (i < d)
  for (uint32_t s = 0; s < cnt; ++s) {
    if ((s & (kRefresh - 1)) == 0) {
      // the tables are read through volatile pointers here so that the compiler does not keep
      // all of M_S^-1 and M_S in registers across the walk for this rare step
      const volatile float* Mv = &t.M[0][0];
      const volatile float* Iv = &t.Minv[0][0];
      float rF[DM];
#pragma unroll
      for (int i = 0; i < DM; ++i) {
        float a = w[i];
        for (int k = 0; k < F; ++k) a -= Mv[i * 32 + d + k] * (((f >> k) & 1) ? -1.f : 1.f);
        rF[i] = a;
      }
      mask = 0;
#pragma unroll
      for (int i = 0; i < DM; ++i) {
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < DM; ++c) a = fmaf(Iv[i * kMaxd + c], rF[c], a);
        u[i] = a;
        if (i < d && a < 0.f) mask |= 1u << i;
      }
#pragma unroll
      for (int i = 0; i < DM; ++i) {
        float a = rF[i];
#pragma unroll
        for (int c = 0; c < DM; ++c)
          if (c < d) a -= Mv[i * 32 + c] * (((mask >> c) & 1) ? -1.f : 1.f);
        e[i] = a;
      }
    }
    float dist = 0.f;
#pragma unroll
    for (int i = 0; i < DM; ++i) dist = fmaf(e[i], e[i], dist);
    if (dist < best_dist || (dist == best_dist && f < best_f)) {
      best_dist = dist;
      best_f = f;
      best_mask = mask;
    }
    if (s + 1 < cnt) {                              // flip free coordinate k = ctz(s+1)
      const int k = __ffs(s + 1) - 1;
      const float sg2 = ((f >> k) & 1) ? -2.f : 2.f;  // r_F moves by sg2 * M[:, d+k]
      float mk[DM], pk[DM];
      load_column<DM>(t.CM[d + k], mk);
      load_column<DM>(t.CP[k], pk);
      // e moves with r_F, u by the column of P
#pragma unroll
      for (int i = 0; i < DM; ++i) {
        e[i] = fmaf(sg2, mk[i], e[i]);
        u[i] = fmaf(sg2, pk[i], u[i]);
      }
      f ^= 1u << k;
      uint32_t nmask = 0;
#pragma unroll
      for (int i = 0; i < DM; ++i)
        if (i < d && u[i] < 0.f) nmask |= 1u << i;
      // every solved sign that flips moves e by 2 * (old b_c) * M_S[:, c]
      for (uint32_t fl = nmask ^ mask; fl; fl &= fl - 1) {
        const int c = __ffs(fl) - 1;
        const float g2 = ((mask >> c) & 1) ? -2.f : 2.f;
        float mc[DM];
        load_column<DM>(t.CM[c], mc);
#pragma unroll
        for (int i = 0; i < DM; ++i) e[i] = fmaf(g2, mc[i], e[i]);
      }
      mask = nmask;
    }
  }
}

// Seeded search with a table of M_S b_S over all 2^d solved sign patterns (d <= 10): the walk
// keeps r_F and u, and e = r_F - T[mask] is read per step instead of being moved by one column
// of M_S per solved sign that flips. T: [2^d][DP] floats, DP = DM rounded up to 4.
template <int DM>
__device__ void search_seeded_table(const Params& p, const Tables& t, const float* __restrict__ T,
                                    const float (&w)[DM], int lane, float& best_dist,
                                    uint32_t& best_f, uint32_t& best_mask) {
  constexpr int DP = (DM + 3) / 4 * 4;
  const int d = p.d, F = p.D - p.d;
  const int lg = F >= 5 ? F - 5 : 0;
  const uint32_t cnt = 1u << lg;
  best_dist = INFINITY;
  best_f = 0xffffffffu;
  best_mask = 0;
  if (F < 5 && lane >= (1 << F)) return;
  float rF[DM], u[DM];
  uint32_t f = (uint32_t)lane << lg, mask = 0;      // mask bit i: b_i = -1 (i < d)
  for (uint32_t s = 0; s < cnt; ++s) {
    if ((s & (kRefresh - 1)) == 0) {
      const volatile float* Mv = &t.M[0][0];
      const volatile float* Iv = &t.Minv[0][0];
#pragma unroll
      for (int i = 0; i < DM; ++i) {
        float a = w[i];
        for (int k = 0; k < F; ++k) a -= Mv[i * 32 + d + k] * (((f >> k) & 1) ? -1.f : 1.f);
        rF[i] = a;
      }
      mask = 0;
#pragma unroll
      for (int i = 0; i < DM; ++i) {
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < DM; ++c) a = fmaf(Iv[i * kMaxd + c], rF[c], a);
        u[i] = a;
        if (i < d && a < 0.f) mask |= 1u << i;
      }
    }
    float tm[DM];
    load_column<DM>(T + (size_t)mask * DP, tm);
    float dist = 0.f;
#pragma unroll
    for (int i = 0; i < DM; ++i) {
      const float e = rF[i] - tm[i];
      dist = fmaf(e, e, dist);
    }
    if (dist < best_dist || (dist == best_dist && f < best_f)) {
      best_dist = dist;
      best_f = f;
      best_mask = mask;
    }
    if (s + 1 < cnt) {                              // flip free coordinate k = ctz(s+1)
      const int k = __ffs(s + 1) - 1;
      const float sg2 = ((f >> k) & 1) ? -2.f : 2.f;  // r_F moves by sg2 * M[:, d+k]
      float mk[DM], pk[DM];
      load_column<DM>(t.CM[d + k], mk);
      load_column<DM>(t.CP[k], pk);
      mask = 0;
#pragma unroll
      for (int i = 0; i < DM; ++i) {
        rF[i] = fmaf(sg2, mk[i], rF[i]);
        u[i] = fmaf(sg2, pk[i], u[i]);
        if (i < d && u[i] < 0.f) mask |= 1u << i;
      }
      f ^= 1u << k;
    }
  }
}

template <int DM, bool kSeeded, bool kTable>
__global__ void __launch_bounds__(kThreads, 4) encode_kernel(const Params p) {
  __shared__ Tables t;
  extern __shared__ __align__(16) float Tsm[];   // kTable: M_S b_S for every solved sign pattern
  build_tables(p, t);
  if (kTable) {
    constexpr int DP = (DM + 3) / 4 * 4;
    for (int e = threadIdx.x; e < (DP << p.d); e += blockDim.x) {
      const int m = e / DP, i = e - m * DP;
      float a = 0.f;
      if (i < p.d)
        for (int c = 0; c < p.d; ++c) a = fmaf(t.M[i][c], ((m >> c) & 1) ? -1.f : 1.f, a);
      Tsm[e] = a;
    }
    __syncthreads();
  }
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  const int64_t ntask = p.N * p.G;
  for (int64_t task = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); task < ntask;
       task += nwarps) {
    const int64_t n = task / p.G;
    const int g = (int)(task - n * p.G);
    // the block, zero beyond K and beyond d; every lane holds all of it
    float mine = 0.f;
    if (lane < p.d && (int64_t)g * p.d + lane < p.K)
      mine = p.w[n * p.K + (int64_t)g * p.d + lane];
    float w[DM];
#pragma unroll
    for (int i = 0; i < DM; ++i) w[i] = __shfl_sync(0xffffffffu, mine, i);
    float bd;
    uint32_t bi, bmask = 0;
    if (kSeeded && kTable)
      search_seeded_table<DM>(p, t, Tsm, w, lane, bd, bi, bmask);
    else if (kSeeded)
      search_seeded<DM>(p, t, w, lane, bd, bi, bmask);
    else
      search_exact<DM>(p, t, w, lane, bd, bi);
    const uint32_t own = bi;
    warp_argmin(bd, bi);
    uint32_t code;
    if (kSeeded) {
      // the solved signs of the winner come from the lane that found it
      const unsigned hit = __ballot_sync(0xffffffffu, own == bi);
      const uint32_t m = __shfl_sync(0xffffffffu, bmask, __ffs(hit) - 1);
      code = m | (bi << p.d);
    } else {
      code = bi;
    }
    int8_t* bo = p.b + (size_t)task * p.D;
    if (lane < p.D) bo[lane] = ((code >> lane) & 1) ? (int8_t)-1 : (int8_t)1;
    if (p.err) {
      // the winner's squared distance from the definition
      float r = 0.f;
      if (lane < p.d) {
        r = w[0];
#pragma unroll
        for (int i = 0; i < DM; ++i)
          if (i == lane) r = w[i];
        for (int j = 0; j < p.D; ++j) r -= t.M[lane][j] * (((code >> j) & 1) ? -1.f : 1.f);
      }
      float dist = r * r;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dist += __shfl_xor_sync(0xffffffffu, dist, o);
      if (lane == 0) p.err[task] = t.singular && kSeeded ? NAN : dist;
    }
  }
}

// the seeded search with the 2^d table, for d <= 10 (at most 48 KB of shared memory)
template <int DM>
static cudaError_t launch_table(const Params& p, int grid, cudaStream_t st) {
  static int set[64];
  const size_t bytes = (size_t)((DM + 3) / 4 * 4 << p.d) * sizeof(float);
  cudaError_t e = ensure_smem((const void*)encode_kernel<DM, true, true>, bytes, set);
  if (e != cudaSuccess) return e;
  encode_kernel<DM, true, true><<<grid, kThreads, bytes, st>>>(p);
  return cudaGetLastError();
}

template <bool kSeeded>
static cudaError_t launch_mode(const Params& p, int grid, cudaStream_t st) {
  const int d = p.d;
  if (kSeeded && d <= 10) {
    if (d <= 2) return launch_table<2>(p, grid, st);
    if (d <= 4) return launch_table<4>(p, grid, st);
    if (d <= 8) return launch_table<8>(p, grid, st);
    return launch_table<10>(p, grid, st);
  }
  if (d <= 2) encode_kernel<2, kSeeded, false><<<grid, kThreads, 0, st>>>(p);
  else if (d <= 4) encode_kernel<4, kSeeded, false><<<grid, kThreads, 0, st>>>(p);
  else if (d <= 8) encode_kernel<8, kSeeded, false><<<grid, kThreads, 0, st>>>(p);
  else if (d <= 10) encode_kernel<10, kSeeded, false><<<grid, kThreads, 0, st>>>(p);
  else if (d <= 12) encode_kernel<12, kSeeded, false><<<grid, kThreads, 0, st>>>(p);
  else encode_kernel<16, kSeeded, false><<<grid, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace enc

cudaError_t launch_encode(const float* w, int64_t N, int32_t K, const float* M, int32_t d,
                          int32_t D, int32_t mode, int8_t* b, float* err, cudaStream_t st) {
  enc::Params p;
  p.w = w;
  p.N = N;
  p.K = K;
  p.d = d;
  p.D = D;
  p.G = (int)(((int64_t)K + d - 1) / d);
  p.M = M;
  p.b = b;
  p.err = err;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      sms = v;
  }
  const int64_t ntask = N * p.G;
  const int64_t want = (ntask + enc::kWarps - 1) / enc::kWarps;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 8));
  return mode == 1 ? enc::launch_mode<true>(p, grid, st) : enc::launch_mode<false>(p, grid, st);
}

}  // namespace lq
