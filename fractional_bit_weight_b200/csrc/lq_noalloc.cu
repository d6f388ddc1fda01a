// lq_noalloc.cu -- lq_gemm_noalloc: the small-batch decode GEMV (lq_gemm's int8 tensor-core
// path) with its scratch in a fixed device array that the library itself owns.
//
// Some callers cannot hand the library any device memory: a process whose device memory is
// entirely owned by a host framework or allocator it cannot call into (a plugin or an
// inference-server backend with a fixed memory budget), or code that runs where allocating is
// not allowed at all. For them this entry point needs no workspace argument; its scratch is
// g_noalloc_scratch below, LQ_NOALLOC_SCRATCH_BYTES bytes that every GPU which loads the
// library keeps until the process exits.
#include <cstdarg>
#include <cmath>
#include <cstdio>
#include <mutex>

#include "lq_internal.cuh"

namespace {

// The scratch of every lq_gemm_noalloc call on a device: split-K completion counters at offset
// 0 (they must start at zero; the kernel returns them to zero), then the activation fragments
// that each call's first kernel writes, then the fp32 slice partials.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
constexpr size_t kCounterBytes = 4096;   // room for 1024 row-range counters

std::mutex g_setup_mu;
void* g_scratch_ptr[kMaxDevices];         // device address of g_noalloc_scratch, per device

thread_local char g_err[512];

lq_status reject(lq_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  lq::set_last_error("%s", g_err);
  return st;
}

// Once per device, with that device current: find the device address of the scratch array (in
// host code its name is only a host-side stand-in) and clear the counter region.
lq_status scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return reject(LQ_ECUDA, "lq_gemm_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return reject(LQ_EUNSUPPORTED, "lq_gemm_noalloc: device %d", dev);
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return reject(LQ_ECUDA, "lq_gemm_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    e = cudaMemset(p, 0, kCounterBytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess)
      return reject(LQ_ECUDA, "lq_gemm_noalloc: clearing the scratch: %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return LQ_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" lq_status lq_gemm_noalloc(const void* x, lq_dtype xdt, int32_t batch,
                                     const lq_whiten_desc* T, const uint32_t* packed,
                                     const float* M, const void* s, lq_dtype sdt, int32_t d,
                                     int32_t D, int32_t K, int32_t N, float* y,
                                     lq_stream stream) {
  lq::set_last_error("%s", "");
  if (K < 1 || d < 1 || D < d || D > LQ_MAX_D || K > (1 << 24))
    return reject(LQ_EINVAL, "lq_gemm_noalloc: invalid code sizes K=%d d=%d D=%d", K, d, D);
  if (N < 1) return reject(LQ_EINVAL, "lq_gemm_noalloc: N = %d < 1", N);
  if (batch < 1 || batch > 8)
    return reject(LQ_EINVAL, "lq_gemm_noalloc: batch = %d; this entry point takes 1..8 tokens", batch);
  const bool dt_ok = [](lq_dtype t) { return t == LQ_F32 || t == LQ_F16 || t == LQ_BF16; }(xdt) &&
                     [](lq_dtype t) { return t == LQ_F32 || t == LQ_F16 || t == LQ_BF16; }(sdt);
  if (!dt_ok) return reject(LQ_EINVAL, "lq_gemm_noalloc: unknown dtype");
  if (!x || !packed || !M || !s || !y) return reject(LQ_EINVAL, "lq_gemm_noalloc: null pointer");
  const size_t xs = xdt == LQ_F32 ? 4 : 2, ss = sdt == LQ_F32 ? 4 : 2;
  if (!aligned(packed, 16) || !aligned(x, xs) || !aligned(s, ss) || !aligned(M, 4) || !aligned(y, 4))
    return reject(LQ_EINVAL, "lq_gemm_noalloc: misaligned pointer");
  lq::Whiten w;
  lq_status st = lq::whiten_from_desc(T, K, &w);
  if (st != LQ_OK) return st;

  const int64_t L = ((int64_t)K + d - 1) / d * D;
  const int64_t row_bytes = ((L + 7) / 8 + 15) / 16 * 16;
  const lq::G8Plan pl = lq::plan_gemv_i8(batch, L, N, K, d, D, w.block);
  const size_t prep_bytes = (pl.frag_bytes + pl.wtab_bytes + pl.csum_bytes + 255) / 256 * 256;
  const size_t partial_bytes = pl.S > 1 ? (size_t)pl.S * batch * N * sizeof(float) : 0;
  const size_t need = kCounterBytes + prep_bytes + partial_bytes;
  if ((size_t)pl.R * sizeof(uint32_t) > kCounterBytes || need > LQ_NOALLOC_SCRATCH_BYTES)
    return reject(LQ_EINVAL,
                  "lq_gemm_noalloc: this shape needs %zu bytes of scratch, more than the "
                  "LQ_NOALLOC_SCRATCH_BYTES = %zu the library holds; use lq_gemm with a workspace",
                  need, (size_t)LQ_NOALLOC_SCRATCH_BYTES);
  if (!pl.ok) return reject(LQ_EUNSUPPORTED, "lq_gemm_noalloc: shape not supported by the GEMV path");

  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != LQ_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  uint32_t* counters = reinterpret_cast<uint32_t*>(base);
  void* prep = base + kCounterBytes;
  float* partials = reinterpret_cast<float*>(base + kCounterBytes + prep_bytes);
  cudaError_t e = lq::launch_gemv_i8(pl, x, (int)xdt, batch, K, w, M, d, D, L, packed, row_bytes,
                                     N, s, (int)sdt, y, prep, partials, counters,
                                     (cudaStream_t)stream);
  if (e != cudaSuccess)
    return reject(LQ_ECUDA, "lq_gemm_noalloc: %s", cudaGetErrorString(e));
  return LQ_OK;
}
