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
  int path;          // LQ_ROUTE_*: 0 int8 tensor-core GEMV (batch <= 8, two kernels); 1 no plan
                     // fits; 2 tcgen05 GEMM (batch >= lq::kTcMinBatch); 3 the int8 GEMV once
                     // per group of gs tokens (when no single-launch plan fits); 4 the
                     // staged int8 GEMV (batch <= 8, prep + TMA-staged GEMV); 5 the
                     // dequantise-once GEMM (fp16 W, dense tcgen05 GEMM)
  size_t counters;   // uint32 completion counters of the split-K reduction
  size_t z;          // paths 0/3: prep output (fragments, weights, sums); 2: fp16 z and token
                     // scales; 4: prep output (fragments, chunk sums, token scales)
  size_t partials;   // float [slices][batch][N]
  size_t total;
  lq::G8Plan g8;
  lq::G8Plan g8g;    // path 3: the plan of a full group of gs tokens
  lq::G8Plan g8r;    // path 3: the plan of the last, smaller group
  int gs;            // path 3: tokens per group
  lq::TcPlan tc;
  lq::BsPlan bs;
  lq::DqPlan dq;
};

// The workspace layout of one lq_gemm call. `forced` >= 0 asks for that route (LQ_ROUTE_*),
// which becomes LQ_ROUTE_NONE if its plan does not fit the shape; -1 chooses automatically.
WsLayout layout_gemm(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D, int32_t Bh,
                     int32_t forced = -1) {
  WsLayout w{};
  const int64_t L = lifted_bits(K, d, D);
  w.g8 = lq::plan_gemv_i8(batch, L, N, K, d, D, Bh);
  w.tc = lq::plan_gemm_tc(batch, L, N, K, d);
  w.bs = lq::plan_gemv_bs(batch, L, N, K, d, D, Bh);
  w.dq = lq::plan_gemm_dq(batch, N, K, d, D);
  // token groups: the largest group whose int8 GEMV plan fits, once per group
  bool groups_ok = false;
  for (int32_t gs : {8, 4, 2, 1}) {
    if (gs >= batch) continue;
    w.g8g = lq::plan_gemv_i8(gs, L, N, K, d, D, Bh);
    w.g8r = batch % gs ? lq::plan_gemv_i8(batch % gs, L, N, K, d, D, Bh) : w.g8g;
    if (w.g8g.ok && w.g8r.ok) {
      w.gs = gs;
      groups_ok = true;
      break;
    }
  }
  w.path = w.g8.ok ? 0 : (w.tc.ok && batch >= lq::kTcMinBatch ? 2 : 1);
  if (w.path == 1 && groups_ok) w.path = 3;
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
  // the staged GEMV serves batches the register-streamed GEMV cannot take in one launch, and
  // one or two tokens on layers of >= 32 MB of codes, where its TMA stream measured faster on
  // B200 (Llama-3-70B MLP shapes: 29.9 against 31.5 us at one token); on smaller layers and at
  // 3..8 tokens the register-streamed GEMV measured faster
  if (w.bs.ok && w.path != 0) w.path = 4;
  if (w.bs.ok && w.path == 0 && batch <= 2 &&
      (double)N * (double)row_stride_bytes(K, d, D) >= 32.0 * 1024 * 1024)
    w.path = 4;
  // the tensor-core routes: the lifted GEMM contracts over L coordinates; the dequantise-once
  // GEMM over G*d inputs (D/d times fewer MMA flops) after writing and reading fp16 W once.
  // Rough B200 costs: ~1.0 PFLOP/s lifted, ~1.3 PFLOP/s dense, ~5 TB/s for W's two passes.
  if (w.path == 2 && w.dq.ok) {
    const double tc_s = 2.0 * batch * (double)N * (double)L / 1.0e15;
    const double dq_s = 2.0 * batch * (double)N * (double)w.dq.Kw / 1.3e15 +
                        2.0 * (double)w.dq.w_bytes / 5.0e12 + 10e-6;
    if (dq_s < tc_s) w.path = 5;
  }
  if (forced >= 0) {
    const bool fits = forced == 0 ? w.g8.ok : forced == 2 ? w.tc.ok : forced == 3 ? groups_ok
                    : forced == 4 ? w.bs.ok : forced == 5 ? w.dq.ok : false;
    w.path = fits ? forced : 1;
  }
  size_t ncounters = 0, npartials = 0, nz = 0;
  if (w.path == 5) {
    nz = (w.dq.w_bytes + w.dq.x_bytes + w.dq.scale_bytes + 3) / 4;
  } else if (w.path == 4) {
    ncounters = (size_t)w.bs.R;
    nz = (w.bs.frag_bytes + w.bs.csum_bytes + w.bs.stok_bytes + 3) / 4;   // prep output
    npartials = w.bs.gacc_bytes / 4;  // int32 totals
  } else if (w.path == 3) {
    // the groups run one after the other on the stream and share the scratch
    for (const lq::G8Plan* g : {&w.g8g, &w.g8r}) {
      const int nb = g == &w.g8g ? w.gs : (batch % w.gs ? batch % w.gs : w.gs);
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
  // paths 0, 2 and 4: a prologue kernel and a contraction kernel, per token group on path 3;
  // path 5: three; path 1: nothing (the call is rejected)
  if (lay.path == 1) return 0;
  if (lay.path == 5) return 3;   // W, xt, GEMM
  return lay.path == 3 ? 2 * ((batch + lay.gs - 1) / lay.gs) : 2;
}

lq_status lq_gemv_staged_plan(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D,
                              int32_t block, int64_t* out) {
  clear_error();
  if (out == nullptr) return fail(LQ_EINVAL, "null out");
  if (!valid_code(K, d, D) || batch < 1 || batch > kMaxBatch || N < 1 || K > kMaxK)
    return fail(LQ_EINVAL, "invalid sizes batch=%d K=%d N=%d d=%d D=%d", batch, K, N, d, D);
  if (block < 0 || block > LQ_MAX_HADAMARD || (block & (block - 1)) != 0)
    return fail(LQ_EINVAL, "invalid Hadamard block %d", block);
  const lq::BsPlan p = lq::plan_gemv_bs(batch, lifted_bits(K, d, D), N, K, d, D, block);
  const int64_t v[LQ_STAGED_PLAN_FIELDS] = {p.ok ? 1 : 0, p.S, p.sc, p.R, p.rq, p.rrem,
                                            p.rows_per_stage, p.wch, p.NS, p.nchunk,
                                            (int64_t)p.smem, (int64_t)p.prep_smem};
  for (int i = 0; i < LQ_STAGED_PLAN_FIELDS; ++i) out[i] = v[i];
  return LQ_OK;
}

int32_t lq_gemm_route(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D,
                      int32_t block) {
  if (!valid_code(K, d, D) || batch < 1 || batch > kMaxBatch || N < 1 || K > kMaxK) return -1;
  if (block < 0 || block > LQ_MAX_HADAMARD || (block & (block - 1)) != 0) return -1;
  return layout_gemm(batch, K, N, d, D, block).path;
}

}  // extern "C"

namespace {

lq_status gemm_impl(const void* x, lq_dtype xdt, int32_t batch, const lq_whiten_desc* T,
                    const uint32_t* packed, const float* M, const void* s, lq_dtype sdt,
                    int32_t d, int32_t D, int32_t K, int32_t N, float* y, void* workspace,
                    size_t workspace_bytes, lq_stream stream, int32_t forced) {
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
  const WsLayout lay = layout_gemm(batch, K, N, d, D, w.block, forced);
  if (workspace_bytes < lay.total)
    return fail(LQ_EINVAL, "workspace of %zu bytes is smaller than the %zu bytes needed",
                workspace_bytes, lay.total);
  char* ws = static_cast<char*>(workspace);
  cudaStream_t cs = (cudaStream_t)stream;
  const int64_t L = lifted_bits(K, d, D);
  uint32_t* counters = reinterpret_cast<uint32_t*>(ws + lay.counters);
  float* partials = reinterpret_cast<float*>(ws + lay.partials);
  if (lay.path == 4) {
    lq::BsScratch sc{};
    sc.frags = reinterpret_cast<uint8_t*>(ws + lay.z);
    sc.csum = reinterpret_cast<float*>(ws + lay.z + lay.bs.frag_bytes);
    sc.stok = reinterpret_cast<float*>(ws + lay.z + lay.bs.frag_bytes + lay.bs.csum_bytes);
    sc.gacc = reinterpret_cast<int*>(ws + lay.partials);
    sc.counters = counters;
    sc.status = reinterpret_cast<uint32_t*>(ws);
    cudaError_t e = lq::launch_gemv_bs(lay.bs, x, (int)xdt, batch, K, w, M, d, D, L, packed,
                                       row_stride_bytes(K, d, D), N, s, (int)sdt, y, sc, cs);
    return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_gemm (staged gemv)");
  }
  if (lay.path == 5) {
    cudaError_t e = lq::launch_gemm_dq(lay.dq, x, (int)xdt, batch, K, w, M, d, D, packed,
                                       row_stride_bytes(K, d, D), N, s, (int)sdt, y, ws + lay.z,
                                       reinterpret_cast<uint32_t*>(ws), cs);
    return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_gemm (dequantise-once gemm)");
  }
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
      cudaError_t e = lq::launch_gemv_i8(nb == lay.gs ? lay.g8g : lay.g8r, xt, (int)xdt, nb, K, w, M, d,
                                         D, L, packed, row_stride_bytes(K, d, D), N, s, (int)sdt,
                                         y + (size_t)t0 * N, ws + lay.z, partials, counters, cs);
      if (e != cudaSuccess) return cuda_fail(e, "lq_gemm (int8 gemv, token group)");
    }
    return LQ_OK;
  }
  return fail(LQ_EUNSUPPORTED, "no GEMV or GEMM plan fits batch=%d K=%d N=%d d=%d D=%d block=%d%s",
              batch, K, N, d, D, w.block, forced >= 0 ? " on the requested route" : "");
}

}  // namespace

extern "C" {

lq_status lq_gemm(const void* x, lq_dtype xdt, int32_t batch, const lq_whiten_desc* T,
                  const uint32_t* packed, const float* M, const void* s, lq_dtype sdt,
                  int32_t d, int32_t D, int32_t K, int32_t N, float* y, void* workspace,
                  size_t workspace_bytes, lq_stream stream) {
  return gemm_impl(x, xdt, batch, T, packed, M, s, sdt, d, D, K, N, y, workspace,
                   workspace_bytes, stream, -1);
}

lq_status lq_gemm_on_route(const void* x, lq_dtype xdt, int32_t batch, const lq_whiten_desc* T,
                           const uint32_t* packed, const float* M, const void* s, lq_dtype sdt,
                           int32_t d, int32_t D, int32_t K, int32_t N, float* y,
                           void* workspace, size_t workspace_bytes, int32_t route,
                           lq_stream stream) {
  clear_error();
  if (route < 0 || route > LQ_ROUTE_GEMM_DQ || route == LQ_ROUTE_NONE)
    return fail(LQ_EINVAL, "unknown route %d", route);
  return gemm_impl(x, xdt, batch, T, packed, M, s, sdt, d, D, K, N, y, workspace,
                   workspace_bytes, stream, route);
}

size_t lq_gemm_route_workspace_bytes(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D,
                                     int32_t block, int32_t route) {
  if (!valid_code(K, d, D) || batch < 1 || batch > kMaxBatch || N < 1 || K > kMaxK) return 0;
  if (block < 0 || block > LQ_MAX_HADAMARD || (block & (block - 1)) != 0) return 0;
  if (route < 0 || route > LQ_ROUTE_GEMM_DQ || route == LQ_ROUTE_NONE) return 0;
  const WsLayout lay = layout_gemm(batch, K, N, d, D, block, route);
  return lay.path == route ? lay.total : 0;
}

namespace {

struct CbLayout {
  size_t b, err, pA, pC, pE, total;
};

CbLayout layout_codebook(int64_t S, int32_t d, int32_t D, bool own_codes) {
  CbLayout l{};
  const size_t parts = lq::codebook_partials(S);
  size_t off = sizeof(lq::WsHeader);
  l.b = off;
  if (own_codes) off = round_up(off + (size_t)S * D, 256);
  l.err = off;
  off = round_up(off + (size_t)S * sizeof(float), 256);
  l.pA = off;
  off = round_up(off + parts * d * D * sizeof(double), 256);
  l.pC = off;
  off = round_up(off + parts * D * D * sizeof(long long), 256);
  l.pE = off;
  off = round_up(off + parts * sizeof(double), 256);
  l.total = off;
  return l;
}

lq_status check_codebook(int64_t S, int32_t d, int32_t D, int32_t mode) {
  if (S < 1 || S > ((int64_t)1 << 31)) return fail(LQ_EINVAL, "S = %lld out of range", (long long)S);
  if (d < 1 || D < d || D > LQ_MAX_D) return fail(LQ_EINVAL, "invalid code sizes d=%d D=%d", d, D);
  if (mode != LQ_ENCODE_EXACT && mode != LQ_ENCODE_SEEDED)
    return fail(LQ_EINVAL, "unknown encode mode %d", mode);
  if (d > 16) return fail(LQ_EUNSUPPORTED, "lq_codebook_round: d = %d > 16", d);
  if (mode == LQ_ENCODE_EXACT && D > 24)
    return fail(LQ_EUNSUPPORTED, "lq_codebook_round: exact search with D = %d > 24", D);
  if (mode == LQ_ENCODE_SEEDED && D - d > 24)
    return fail(LQ_EUNSUPPORTED, "lq_codebook_round: seeded search with D - d = %d > 24", D - d);
  return LQ_OK;
}

}  // namespace

size_t lq_codebook_workspace_bytes(int64_t S, int32_t d, int32_t D) {
  if (S < 1 || S > ((int64_t)1 << 31) || d < 1 || D < d || D > LQ_MAX_D) return 0;
  return layout_codebook(S, d, D, true).total;
}

lq_status lq_codebook_round(const float* w, int64_t S, float* M, int32_t d, int32_t D,
                            int32_t mode, int8_t* b_out, double* mse, void* workspace,
                            size_t workspace_bytes, lq_stream stream) {
  clear_error();
  lq_status st = check_codebook(S, d, D, mode);
  if (st != LQ_OK) return st;
  if (!w || !M || !workspace) return fail(LQ_EINVAL, "null pointer");
  if (!aligned(w, 4) || !aligned(M, 4) || !aligned(workspace, 256) || (mse && !aligned(mse, 8)))
    return fail(LQ_EINVAL, "misaligned w/M/workspace/mse");
  const CbLayout l = layout_codebook(S, d, D, b_out == nullptr);
  if (workspace_bytes < l.total)
    return fail(LQ_EINVAL, "workspace of %zu bytes is smaller than the %zu bytes needed",
                workspace_bytes, l.total);
  char* ws = static_cast<char*>(workspace);
  int8_t* b = b_out ? b_out : reinterpret_cast<int8_t*>(ws + l.b);
  cudaError_t e = lq::launch_codebook_round(
      w, S, M, d, D, mode, b, reinterpret_cast<float*>(ws + l.err),
      reinterpret_cast<double*>(ws + l.pA), reinterpret_cast<long long*>(ws + l.pC),
      reinterpret_cast<double*>(ws + l.pE), mse, (cudaStream_t)stream);
  return e == cudaSuccess ? LQ_OK : cuda_fail(e, "lq_codebook_round");
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
