// lq_abi.cu -- the extern "C" entry points of liblq: argument checks, planning, launches.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "lq_internal.cuh"

namespace {

thread_local char g_last_error[512] = "";

lq_status fail(lq_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

lq_status cuda_fail(cudaError_t e, const char* where) {
  return fail(LQ_ECUDA, "%s: %s", where, cudaGetErrorString(e));
}

void clear_error() { g_last_error[0] = '\0'; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_code(int32_t K, int32_t d, int32_t D) {
  return K >= 1 && d >= 1 && D >= d && D <= LQ_MAX_D;
}

int64_t lifted_bits(int32_t K, int32_t d, int32_t D) {
  return ((int64_t)K + d - 1) / d * D;
}

int64_t row_stride_bytes(int32_t K, int32_t d, int32_t D) {
  const int64_t bytes = (lifted_bits(K, d, D) + 7) / 8;
  return (bytes + 15) / 16 * 16;
}

bool valid_dtype(lq_dtype t) { return t == LQ_F32 || t == LQ_F16 || t == LQ_BF16; }

size_t dtype_size(lq_dtype t) { return t == LQ_F32 ? 4 : 2; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Validates a whitening descriptor against K and converts it.
lq_status make_whiten(const lq_whiten_desc* T, int32_t K, lq::Whiten* out) {
  out->sign = nullptr;
  out->chan_scale = nullptr;
  out->block = 0;
  out->inv_sqrt = 1.f;
  if (T == nullptr || T->block == 0) return LQ_OK;
  const int32_t B = T->block;
  if (B < 0 || (B & (B - 1)) != 0)
    return fail(LQ_EINVAL, "whitening block %d is not 0 or a power of two", B);
  if (B > LQ_MAX_HADAMARD)
    return fail(LQ_EUNSUPPORTED, "whitening block %d exceeds LQ_MAX_HADAMARD (%d)", B,
                LQ_MAX_HADAMARD);
  if (K % B != 0) return fail(LQ_EINVAL, "whitening block %d does not divide K = %d", B, K);
  out->sign = T->sign;
  out->chan_scale = T->chan_scale;
  out->block = B;
  out->inv_sqrt = (float)(1.0 / std::sqrt((double)B));
  if (out->chan_scale && !aligned(out->chan_scale, 4))
    return fail(LQ_EINVAL, "chan_scale is not 4-byte aligned");
  return LQ_OK;
}

// Workspace layout of lq_gemm (byte offsets, all 256-aligned).
struct WsLayout {
  int path;          // 0: int8 tensor-core GEMV (batch <= 8); 1: fp32 GEMV over z;
                     // 2: tcgen05 GEMM (batch >= lq::kTcMinBatch); 3: the int8 GEMV once per
                     // group of gs tokens (when no single-launch plan fits)
  size_t counters;   // uint32 completion counters of the split-K reduction
  size_t z;          // path 0: prep output (fragments, weights, sums); path 1: float z [batch][L]
  size_t partials;   // float [slices][batch][N]
  size_t total;
  lq::GemvPlan gemv;
  lq::G8Plan g8;
  lq::G8Plan g8r;    // path 3: the plan of the last, smaller group
  int gs;            // path 3: tokens per group
  lq::TcPlan tc;
};

WsLayout layout_gemm(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D, int32_t Bh) {
  WsLayout w{};
  const int64_t L = lifted_bits(K, d, D);
  w.g8 = lq::plan_gemv_i8(batch, L, N, K, d, D, Bh);
  w.tc = lq::plan_gemm_tc(batch, L, N, K, d);
  w.path = w.g8.ok ? 0 : (w.tc.ok && batch >= lq::kTcMinBatch ? 2 : 1);
  // no single-launch GEMV fits: the largest token group whose int8 GEMV plan does, once per
  // group
  for (int32_t gs : {8, 4, 2, 1}) {
    if (w.path != 1 || gs >= batch) continue;
    w.g8 = lq::plan_gemv_i8(gs, L, N, K, d, D, Bh);
    w.g8r = batch % gs ? lq::plan_gemv_i8(batch % gs, L, N, K, d, D, Bh) : w.g8;
    if (w.g8.ok && w.g8r.ok) {
      w.path = 3;
      w.gs = gs;
    }
  }
  // below kTcMinBatch tokens the tensor-core GEMM still wins once the groups are many: rough
  // B200 costs, each group streaming the codes at ~2 TB/s plus ~6 us, each wave of 128 x 256
  // tiles ~0.7 us per 64-coordinate stage
  if (w.path == 3 && w.tc.ok) {
    const double groups = (double)((batch + w.gs - 1) / w.gs);
    const double gemv_s = groups * ((double)N * (double)row_stride_bytes(K, d, D) / 2.0e12 + 6e-6);
    const int sms = 148;
    const double tc_s = (double)((w.tc.tiles + sms - 1) / sms) * w.tc.nks * 0.7e-6 + 10e-6;
    if (tc_s < gemv_s) w.path = 2;
  }
  if (w.path == 1 && w.tc.ok && batch > 8) w.path = 2;
  size_t ncounters = 0, npartials = 0, nz = 0;
  if (w.path == 3) {
    // the groups run one after the other on the stream and share the scratch
    for (const lq::G8Plan* g : {&w.g8, &w.g8r}) {
      const int nb = g == &w.g8 ? w.gs : (batch % w.gs ? batch % w.gs : w.gs);
      ncounters = std::max(ncounters, (size_t)g->R);
      npartials = std::max(npartials, g->S > 1 ? (size_t)g->S * nb * N : (size_t)0);
      nz = std::max(nz, (g->frag_bytes + g->wtab_bytes + g->csum_bytes + 3) / 4);
    }
  } else if (w.path == 2) {
    nz = (w.tc.z_bytes + w.tc.scale_bytes + 3) / 4;   // fp16 z, then the token scales
  } else if (w.path == 0) {
    ncounters = (size_t)w.g8.R;
    npartials = w.g8.S > 1 ? (size_t)w.g8.S * batch * N : 0;
    nz = (w.g8.frag_bytes + w.g8.wtab_bytes + w.g8.csum_bytes + 3) / 4;   // prep output
  } else {
    w.gemv = lq::plan_gemv(batch, L, N);
    ncounters = (size_t)w.gemv.ntg * w.gemv.ntiles;
    npartials = w.gemv.nsl > 1 ? (size_t)w.gemv.nsl * batch * N : 0;
    nz = (size_t)batch * L;
  }
  size_t off = sizeof(lq::WsHeader);
  w.counters = off;
  off = round_up(off + ncounters * sizeof(uint32_t), 256);
  w.z = off;
  off = round_up(off + nz * sizeof(float), 256);
  w.partials = off;
  off = round_up(off + npartials * sizeof(float), 256);
  w.total = off;
  return w;
}

constexpr int32_t kMaxBatch = 1 << 20;
constexpr int32_t kMaxK = 1 << 24;

}  // namespace

namespace lq {

void set_last_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

lq_status whiten_from_desc(const lq_whiten_desc* T, int32_t K, Whiten* out) {
  return make_whiten(T, K, out);
}

}  // namespace lq

extern "C" {

int32_t lq_abi_version(void) { return LQ_ABI_VERSION; }

int64_t lq_lifted_bits(int32_t K, int32_t d, int32_t D) {
  return valid_code(K, d, D) ? lifted_bits(K, d, D) : -1;
}

int64_t lq_row_stride_bytes(int32_t K, int32_t d, int32_t D) {
  return valid_code(K, d, D) ? row_stride_bytes(K, d, D) : -1;
}

const char* lq_status_string(lq_status s) {
  switch (s) {
    case LQ_OK: return "LQ_OK";
    case LQ_EINVAL: return "LQ_EINVAL: invalid argument";
    case LQ_EUNSUPPORTED: return "LQ_EUNSUPPORTED: valid but not supported";
    case LQ_ECUDA: return "LQ_ECUDA: CUDA error";
    case LQ_ETIMEOUT: return "LQ_ETIMEOUT: device-side wait expired";
    case LQ_EDEVICE: return "LQ_EDEVICE: device-side check failed";
  }
  return "unknown lq_status";
}

const char* lq_last_error(void) { return g_last_error; }

lq_status lq_pack(const int8_t* b_pm1, int32_t N, int32_t K, int32_t d, int32_t D,
                  uint32_t* packed, lq_stream stream) {
  clear_error();
  if (!valid_code(K, d, D)) return fail(LQ_EINVAL, "invalid code sizes K=%d d=%d D=%d", K, d, D);
  if (N < 0) return fail(LQ_EINVAL, "N = %d < 0", N);
  if (N == 0) return LQ_OK;
  if (!b_pm1 || !packed) return fail(LQ_EINVAL, "null pointer");
  if (!aligned(packed, 16)) return fail(LQ_EINVAL, "packed is not 16-byte aligned");
  cudaError_t e = lq::launch_pack(b_pm1, N, lifted_bits(K, d, D), row_stride_bytes(K, d, D) / 4,
                                  packed, (cudaStream_t)stream);
  return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_pack");
}

lq_status lq_encode(const float* w, int32_t N, int32_t K, const float* M, int32_t d, int32_t D,
                    int32_t mode, int8_t* b_pm1, float* err, lq_stream stream) {
  clear_error();
  if (!valid_code(K, d, D)) return fail(LQ_EINVAL, "invalid code sizes K=%d d=%d D=%d", K, d, D);
  if (N < 0) return fail(LQ_EINVAL, "N = %d < 0", N);
  if (mode != LQ_ENCODE_EXACT && mode != LQ_ENCODE_SEEDED)
    return fail(LQ_EINVAL, "unknown encode mode %d", mode);
  if (d > 16) return fail(LQ_EUNSUPPORTED, "lq_encode: d = %d > 16", d);
  if (mode == LQ_ENCODE_EXACT && D > 24)
    return fail(LQ_EUNSUPPORTED, "lq_encode: exact search with D = %d > 24", D);
  if (mode == LQ_ENCODE_SEEDED && D - d > 24)
    return fail(LQ_EUNSUPPORTED, "lq_encode: seeded search with D - d = %d > 24", D - d);
  if (N == 0) return LQ_OK;
  if (!w || !M || !b_pm1) return fail(LQ_EINVAL, "null pointer");
  if (!aligned(w, 4) || !aligned(M, 4) || (err && !aligned(err, 4)))
    return fail(LQ_EINVAL, "misaligned w/M/err");
  cudaError_t e = lq::launch_encode(w, N, K, M, d, D, mode, b_pm1, err, (cudaStream_t)stream);
  return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_encode");
}

lq_status lq_unpack(const uint32_t* packed, int32_t N, int32_t K, int32_t d, int32_t D,
                    int8_t* b_pm1, lq_stream stream) {
  clear_error();
  if (!valid_code(K, d, D)) return fail(LQ_EINVAL, "invalid code sizes K=%d d=%d D=%d", K, d, D);
  if (N < 0) return fail(LQ_EINVAL, "N = %d < 0", N);
  if (N == 0) return LQ_OK;
  if (!b_pm1 || !packed) return fail(LQ_EINVAL, "null pointer");
  if (!aligned(packed, 16)) return fail(LQ_EINVAL, "packed is not 16-byte aligned");
  cudaError_t e = lq::launch_unpack(packed, N, lifted_bits(K, d, D),
                                    row_stride_bytes(K, d, D) / 4, b_pm1, (cudaStream_t)stream);
  return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_unpack");
}

lq_status lq_whiten(const void* x, lq_dtype xdt, int32_t batch, int32_t K,
                    const lq_whiten_desc* T, float* xt, lq_stream stream) {
  clear_error();
  if (batch < 0 || batch > kMaxBatch) return fail(LQ_EINVAL, "batch = %d out of range", batch);
  if (K < 1 || K > kMaxK) return fail(LQ_EINVAL, "K = %d out of range", K);
  if (!valid_dtype(xdt)) return fail(LQ_EINVAL, "unknown x dtype %d", (int)xdt);
  if (batch == 0) return LQ_OK;
  if (!x || !xt) return fail(LQ_EINVAL, "null pointer");
  if (!aligned(x, dtype_size(xdt)) || !aligned(xt, 4)) return fail(LQ_EINVAL, "misaligned x/xt");
  lq::Whiten w;
  lq_status st = make_whiten(T, K, &w);
  if (st != LQ_OK) return st;
  cudaError_t e = lq::launch_whiten(x, (int)xdt, batch, K, w, xt, (cudaStream_t)stream);
  return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_whiten");
}

lq_status lq_lift(const void* x, lq_dtype xdt, int32_t batch, int32_t K,
                  const lq_whiten_desc* T, const float* M, int32_t d, int32_t D, float* z,
                  lq_stream stream) {
  clear_error();
  if (!valid_code(K, d, D)) return fail(LQ_EINVAL, "invalid code sizes K=%d d=%d D=%d", K, d, D);
  if (batch < 0 || batch > kMaxBatch) return fail(LQ_EINVAL, "batch = %d out of range", batch);
  if (K > kMaxK) return fail(LQ_EINVAL, "K = %d out of range", K);
  if (!valid_dtype(xdt)) return fail(LQ_EINVAL, "unknown x dtype %d", (int)xdt);
  if (batch == 0) return LQ_OK;
  if (!x || !M || !z) return fail(LQ_EINVAL, "null pointer");
  if (!aligned(x, dtype_size(xdt)) || !aligned(M, 4) || !aligned(z, 4))
    return fail(LQ_EINVAL, "misaligned x/M/z");
  lq::Whiten w;
  lq_status st = make_whiten(T, K, &w);
  if (st != LQ_OK) return st;
  cudaError_t e = lq::launch_lift_f32(x, (int)xdt, batch, K, w, M, d, D, z, nullptr, 0,
                                      (cudaStream_t)stream);
  return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_lift");
}

size_t lq_gemm_workspace_bytes(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D) {
  if (!valid_code(K, d, D) || batch < 1 || batch > kMaxBatch || N < 1 || K > kMaxK) return 0;
  // the plan (and so the workspace) depends on the Hadamard block; return the largest
  size_t best = 0;
  for (int32_t Bh = 0; Bh <= LQ_MAX_HADAMARD; Bh = Bh ? 2 * Bh : 1)
    best = std::max(best, layout_gemm(batch, K, N, d, D, Bh).total);
  return best;
}

int32_t lq_gemm_launches(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D,
                         int32_t block) {
  if (!valid_code(K, d, D) || batch < 1 || batch > kMaxBatch || N < 1 || K > kMaxK) return 0;
  if (block < 0 || block > LQ_MAX_HADAMARD || (block & (block - 1)) != 0) return 0;
  const WsLayout lay = layout_gemm(batch, K, N, d, D, block);
  // every path: a prologue kernel and a contraction kernel, per token group on path 3
  return lay.path == 3 ? 2 * ((batch + lay.gs - 1) / lay.gs) : 2;
}

lq_status lq_gemm(const void* x, lq_dtype xdt, int32_t batch, const lq_whiten_desc* T,
                  const uint32_t* packed, const float* M, const void* s, lq_dtype sdt,
                  int32_t d, int32_t D, int32_t K, int32_t N, float* y, void* workspace,
                  size_t workspace_bytes, lq_stream stream) {
  clear_error();
  if (!valid_code(K, d, D)) return fail(LQ_EINVAL, "invalid code sizes K=%d d=%d D=%d", K, d, D);
  if (batch < 1 || batch > kMaxBatch) return fail(LQ_EINVAL, "batch = %d out of range", batch);
  if (N < 1) return fail(LQ_EINVAL, "N = %d < 1", N);
  if (K > kMaxK) return fail(LQ_EINVAL, "K = %d out of range", K);
  if (!valid_dtype(xdt) || !valid_dtype(sdt)) return fail(LQ_EINVAL, "unknown dtype");
  if (!x || !packed || !M || !s || !y || !workspace) return fail(LQ_EINVAL, "null pointer");
  if (!aligned(packed, 16)) return fail(LQ_EINVAL, "packed is not 16-byte aligned");
  if (!aligned(workspace, 256)) return fail(LQ_EINVAL, "workspace is not 256-byte aligned");
  if (!aligned(x, dtype_size(xdt)) || !aligned(s, dtype_size(sdt)) || !aligned(M, 4) ||
      !aligned(y, 4))
    return fail(LQ_EINVAL, "misaligned x/s/M/y");
  lq::Whiten w;
  lq_status st = make_whiten(T, K, &w);
  if (st != LQ_OK) return st;
  const WsLayout lay = layout_gemm(batch, K, N, d, D, w.block);
  if (workspace_bytes < lay.total)
    return fail(LQ_EINVAL, "workspace of %zu bytes is smaller than the %zu bytes needed",
                workspace_bytes, lay.total);
  char* ws = static_cast<char*>(workspace);
  cudaStream_t cs = (cudaStream_t)stream;
  const int64_t L = lifted_bits(K, d, D);
  uint32_t* counters = reinterpret_cast<uint32_t*>(ws + lay.counters);
  float* partials = reinterpret_cast<float*>(ws + lay.partials);
  if (lay.path == 2) {
    cudaError_t e = lq::launch_gemm_tc(lay.tc, x, (int)xdt, batch, K, w, M, d, D, L, packed,
                                       row_stride_bytes(K, d, D), N, s, (int)sdt, y, ws + lay.z,
                                       reinterpret_cast<uint32_t*>(ws), cs);
    return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_gemm (tensor-core gemm)");
  }
  if (lay.path == 0) {
    cudaError_t e = lq::launch_gemv_i8(lay.g8, x, (int)xdt, batch, K, w, M, d, D, L, packed,
                                       row_stride_bytes(K, d, D), N, s, (int)sdt, y, ws + lay.z,
                                       partials, counters, cs);
    return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_gemm (int8 gemv)");
  }
  if (lay.path == 3) {
    for (int32_t t0 = 0; t0 < batch; t0 += lay.gs) {
      const int32_t nb = std::min<int32_t>(lay.gs, batch - t0);
      const char* xt = static_cast<const char*>(x) + (size_t)t0 * K * dtype_size(xdt);
      cudaError_t e = lq::launch_gemv_i8(nb == lay.gs ? lay.g8 : lay.g8r, xt, (int)xdt, nb, K, w, M, d,
                                         D, L, packed, row_stride_bytes(K, d, D), N, s, (int)sdt,
                                         y + (size_t)t0 * N, ws + lay.z, partials, counters, cs);
      if (e != cudaSuccess) return cuda_fail(e, "lq_gemm (int8 gemv, token group)");
    }
    return LQ_OK;
  }
  if (lay.gemv.ntiles > 65535 || lay.gemv.ntg > 65535)
    return fail(LQ_EUNSUPPORTED, "N or batch too large for one launch");
  float* z = reinterpret_cast<float*>(ws + lay.z);
  cudaError_t e = lq::launch_lift_f32(x, (int)xdt, batch, K, w, M, d, D, z, counters,
                                      lay.gemv.ntg * lay.gemv.ntiles, cs);
  if (e != cudaSuccess) return cuda_fail(e, "lq_gemm (lift)");
  e = lq::launch_gemv(lay.gemv, z, L, batch, packed, row_stride_bytes(K, d, D) / 4, N, s,
                      (int)sdt, y, partials, counters, cs);
  return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_gemm (gemv)");
}

lq_status lq_device_status(void* workspace, int32_t* code, lq_stream stream) {
  clear_error();
  if (!workspace || !code) return fail(LQ_EINVAL, "null pointer");
  cudaStream_t cs = (cudaStream_t)stream;
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_fail(e, "lq_device_status");
  *code = (int32_t)v;
  if (v != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyAsync(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return cuda_fail(e, "lq_device_status");
    return (lq_status)v;
  }
  return LQ_OK;
}

}  // extern "C"
