// lq_internal.cuh -- declarations shared by the liblq CUDA sources (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "liblq.h"

namespace lq {

// Parameters of the whitening T after host-side validation.
struct Whiten {
  const int8_t* sign;       // [K] or nullptr
  const float* chan_scale;  // [K] or nullptr
  int32_t block;            // 0 = identity, else a power of two dividing K
  float inv_sqrt;           // 1/sqrt(block), computed on the host in double
};

// Byte offsets inside the caller's lq_gemm workspace.
struct WsHeader {
  uint32_t status;          // 0, or an lq_status recorded by a kernel
  uint32_t reserved[63];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

__device__ __forceinline__ float load_as_f32(const void* p, int dt, int64_t i) {
  if (dt == LQ_F32) return static_cast<const float*>(p)[i];
  if (dt == LQ_F16) return __half2float(static_cast<const __half*>(p)[i]);
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

// Records the reason for a rejected call (read back by lq_last_error on this host thread).
void set_last_error(const char* fmt, ...);
// Validates a whitening descriptor against K (as lq_gemm does) and converts it.
lq_status whiten_from_desc(const lq_whiten_desc* T, int32_t K, Whiten* out);

// Raises the dynamic shared memory limit of `func` to `bytes` on the current device, once per
// (function, device) and only when a launch needs more than before (keeps launches capturable).
cudaError_t ensure_smem(const void* func, size_t bytes, int* cache_per_device);

// ---- launchers (host side); each returns cudaGetLastError() of its launch
cudaError_t launch_pack(const int8_t* b, int32_t N, int64_t L, int64_t words, uint32_t* packed,
                        cudaStream_t st);
cudaError_t launch_unpack(const uint32_t* packed, int32_t N, int64_t L, int64_t words,
                          int8_t* b, cudaStream_t st);
cudaError_t launch_whiten(const void* x, int xdt, int32_t batch, int32_t K, Whiten T,
                          float* xt, cudaStream_t st);
// Fused whiten + lift into fp32 z [batch][G*D]. If zero_words > 0, the launch also clears
// zero_ptr[0 .. zero_words) (the split-K counters of a following GEMV launch).
cudaError_t launch_lift_f32(const void* x, int xdt, int32_t batch, int32_t K, Whiten T,
                            const float* M, int32_t d, int32_t D, float* z, uint32_t* zero_ptr,
                            int32_t zero_words, cudaStream_t st);

// Plan of the int8 tensor-core GEMV (batch <= 8): a prep kernel per 512-bit chunk, then
// S K-slices x R row ranges, one CTA each.
struct G8Plan {
  bool ok;
  int nt;             // 8-column MMA tiles (2 tokens each)
  int nchunk;         // 512-bit chunks per row
  int sc;             // chunks per slice
  int S;              // slices
  int R;              // row ranges
  int nctas;          // S * R
  int xs_floats;      // whitening scratch per token (prep)
  size_t smem;        // gemv dynamic shared memory per CTA
  size_t prep_smem;   // prep dynamic shared memory per CTA
  size_t frag_bytes;  // scratch: B fragments
  size_t wtab_bytes;  // scratch: per-chunk column weights
  size_t csum_bytes;  // scratch: per-chunk sums of z
};
G8Plan plan_gemv_i8(int32_t batch, int64_t L, int32_t N, int32_t K, int32_t d, int32_t D,
                    int32_t Bh);
// scratch: frag_bytes + wtab_bytes + csum_bytes bytes (16-byte aligned); partials:
// [S][batch][N] floats and counters: [R] zeroed uint32 (both unused when S == 1)
cudaError_t launch_gemv_i8(const G8Plan& pl, const void* x, int xdt, int32_t batch, int32_t K,
                           Whiten T, const float* M, int32_t d, int32_t D, int64_t L,
                           const uint32_t* packed, int64_t row_bytes, int32_t N, const void* s,
                           int sdt, float* y, void* scratch, float* partials,
                           uint32_t* counters, cudaStream_t st);

// Plan of the tensor-core GEMM (always used from kTcMinBatch tokens, below that when it is
// expected to beat the int8 GEMV run per token group): a whiten + lift prologue writing fp16
// z with a per-token power-of-two scale, then a persistent tcgen05 kernel over 128-token x
// 256-row tiles.
constexpr int32_t kTcMinBatch = 64;
struct TcPlan {
  bool ok;
  int Lp;              // lifted length padded to the 64-coordinate stage
  int nks;             // stages per tile (Lp / 64)
  int tiles_n, tiles_m, tiles;
  int group_m;         // token tiles per raster group
  size_t smem;         // GEMM dynamic shared memory per CTA
  size_t pro_smem;     // prologue dynamic shared memory per CTA
  size_t z_bytes;      // scratch: fp16 z [batch][Lp]
  size_t scale_bytes;  // scratch: float 2^-e [batch], right after z
};
TcPlan plan_gemm_tc(int32_t batch, int64_t L, int32_t N, int32_t K, int32_t d);
// scratch: z_bytes + scale_bytes bytes, 256-byte aligned; status: the workspace status word
cudaError_t launch_gemm_tc(const TcPlan& pl, const void* x, int xdt, int32_t batch, int32_t K,
                           Whiten T, const float* M, int32_t d, int32_t D, int64_t L,
                           const uint32_t* packed, int64_t row_bytes, int32_t N, const void* s,
                           int sdt, float* y, void* scratch, uint32_t* status, cudaStream_t st);

// Plan of the staged int8 tensor-core GEMV (batch <= 8): a prep kernel, one CTA per 512-bit
// chunk, writes the activation fragments; the GEMV (S K-slices x R row ranges, one CTA per SM,
// programmatic dependent launch) streams the codes through shared memory with TMA.
struct BsPlan {
  bool ok;
  int nt;             // 8-column MMA tiles (2 tokens each)
  int nchunk;         // 512-bit chunks per row
  int sc;             // chunks per slice
  int S;              // slices
  int R;              // row ranges
  int rq, rrem;       // rows per range: rq + (range < rrem)
  int rows_max;       // rq + 1
  int rows_per_stage;  // 16 or 32
  int wch;            // chunks per stage window (odd)
  int stride;         // shared-memory row stride of a stage (64 * wch)
  int NS;             // ring stages
  int nctas;          // S * R
  int xs_floats;      // prep: whitened inputs of one chunk, per token
  size_t smem;        // GEMV dynamic shared memory per CTA
  size_t frag_smem;   // GEMV shared memory: the slice's fragments and a zero block
  size_t prep_smem;   // prep dynamic shared memory per CTA
  size_t frag_bytes;  // scratch: fragments [batch][nchunk][1536]
  size_t csum_bytes;  // scratch: per-chunk sums of z [nchunk][batch]
  size_t stok_bytes;  // scratch: per-token scales [batch]
  size_t gacc_bytes;  // scratch: int32 totals [batch][N][4] (S > 1), zero at rest
};
BsPlan plan_gemv_bs(int32_t batch, int64_t L, int32_t N, int32_t K, int32_t d, int32_t D,
                    int32_t Bh);
// Global scratch of one call: frags, csum and stok are rewritten by every call (16-byte
// aligned); gacc and counters [R] (used when S > 1) must be zero before the first call and are
// left zero by every call.
struct BsScratch {
  uint8_t* frags;
  float* csum;
  float* stok;
  int* gacc;
  uint32_t* counters;
  uint32_t* status;
};
cudaError_t launch_gemv_bs(const BsPlan& pl, const void* x, int xdt, int32_t batch, int32_t K,
                           Whiten T, const float* M, int32_t d, int32_t D, int64_t L,
                           const uint32_t* packed, int64_t row_bytes, int32_t N, const void* s,
                           int sdt, float* y, const BsScratch& ws, cudaStream_t st);

// Plan of the dequantise-once GEMM (large batches): W = blockwise M b in fp16 [N][Kw], fp16
// T(x) [batch][Kw] with a per-token power of two, then a persistent tcgen05 GEMM over
// 128-token x 256-row tiles.
struct DqPlan {
  bool ok;
  int G;               // blocks of d inputs per row
  int Kw;              // G*d padded to the 64-input stage
  int nks;             // stages per tile
  int tiles_n, tiles_m, tiles;
  size_t smem;         // GEMM dynamic shared memory per CTA
  size_t xt_smem;      // xt kernel dynamic shared memory
  size_t dq_smem;      // dequantisation kernel dynamic shared memory per CTA
  int dq_ctas_per_sm;  // dequantisation CTAs per SM
  size_t w_bytes;      // scratch: fp16 W [N][Kw]
  size_t x_bytes;      // scratch: fp16 xt [batch][Kw], after W
  size_t scale_bytes;  // scratch: float 2^-e [batch], after xt
};
DqPlan plan_gemm_dq(int32_t batch, int32_t N, int32_t K, int32_t d, int32_t D);
// scratch: w_bytes + x_bytes + scale_bytes bytes, 256-byte aligned; status: workspace word
cudaError_t launch_gemm_dq(const DqPlan& pl, const void* x, int xdt, int32_t batch, int32_t K,
                           Whiten T, const float* M, int32_t d, int32_t D,
                           const uint32_t* packed, int64_t row_bytes, int32_t N, const void* s,
                           int sdt, float* y, void* scratch, uint32_t* status, cudaStream_t st);

// cuTensorMapEncodeTiled through the runtime's driver entry point (nullptr if unavailable),
// and the SM count of the current device (0 on error); both cached.
typedef CUresult (*TensorMapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                      const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                      const cuuint32_t*, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);
TensorMapEncodeFn tensor_map_encode_fn();
int tc_sm_count();

// Nearest-codeword encoding, block by block: b [N][ceil(K/d)][D] +1/-1, err [N][G] or null.
// mode 0: all 2^D codewords; mode 1: first d coordinates solved, the rest enumerated.
cudaError_t launch_encode(const float* w, int64_t N, int32_t K, const float* M, int32_t d,
                          int32_t D, int32_t mode, int8_t* b, float* err, cudaStream_t st);

// One round of the codebook fit (see lq_codebook.cu): the encoder into b [S][D] and err [S],
// then the sums into the partials (codebook_partials(S) CTAs: pA [parts][d*D], pC
// [parts][D*D], pE [parts]) and the solve into M and *mse (mse may be null).
size_t codebook_partials(int64_t S);
cudaError_t launch_codebook_round(const float* w, int64_t S, float* M, int32_t d, int32_t D,
                                  int32_t mode, int8_t* b, float* err, double* pA, long long* pC,
                                  double* pE, double* mse, cudaStream_t st);

}  // namespace lq
