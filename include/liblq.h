/*
 * liblq.h -- C ABI of the B200 (sm_100a) LiftQuant decode library.
 *
 * The operator (LiftQuant: Continuous Bit-Width LLM Quantization via Dimensional
 * Lifting and Projection, sec. 3 intro and sec. 3.1; the romaanj.github.io review,
 * "Method"):
 *
 *     y[t][n] = s[n] * sum_k W[n][k] * T(x[t])[k]
 *     W[n][g*d + i] = sum_{j<D} M[i][j] * b[n][g][j],   b in {+1,-1}
 *
 * Each length-d block g of a weight row is stored as D sign bits b[n][g][.] and
 * decoded through the d x D mapping matrix M, so a row of K inputs costs
 * ceil(K/d) * D bits: the fractional bit-width D/d (24/10 = 2.4 bit). T is the
 * whitening transform: a random +-1 diagonal (and optional per-channel scale)
 * followed by the normalised Walsh-Hadamard transform on contiguous blocks.
 * The library evaluates the lifted form y = s . (b . z) with
 * z[t][g*D + j] = sum_i M[i][j] * T(x[t])[g*d + i], since b^T (M^T x) = (M b)^T x.
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers owned by the caller, row-major and
 *     dense. The library never allocates, frees, prints or exits.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls are
 *     asynchronous with respect to the host; results are ready when the stream is.
 *   - Arguments are checked on the host before anything is launched; a rejected
 *     call launches nothing and returns LQ_EINVAL or LQ_EUNSUPPORTED.
 *     lq_last_error() then holds a one-line reason (per host thread).
 *   - A failed launch returns LQ_ECUDA. Device-side failures are recorded in the
 *     workspace status word and read by lq_device_status().
 *   - Calls that share a workspace must be ordered on one stream.
 */
#ifndef LIBLQ_H
#define LIBLQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LQ_ABI_VERSION 1
/* Stored-code format. Row n, block g, lifted coordinate j is bit q = g*D + j of
 * the row; bit q is bit (q % 32) of 32-bit little-endian word q / 32 (equivalently
 * bit q % 8 of byte q / 8); a set bit means b = -1 (it is the sign bit that flips
 * z); each row is zero-padded to a multiple of 16 bytes. */
#define LQ_FORMAT_V1 1
/* Largest supported Hadamard block of T. */
#define LQ_MAX_HADAMARD 4096
/* Largest lifted dimension D per block (the pages' largest code is LQ-32/16). */
#define LQ_MAX_D 32

typedef enum lq_status {
  LQ_OK = 0,
  LQ_EINVAL = 1,        /* a null/misaligned pointer or an out-of-range size */
  LQ_EUNSUPPORTED = 2,  /* valid, but not implemented (e.g. Hadamard block > LQ_MAX_HADAMARD) */
  LQ_ECUDA = 3,         /* a CUDA launch or query failed */
  LQ_ETIMEOUT = 4,      /* a bounded device-side wait expired (status word) */
  LQ_EDEVICE = 5        /* a device-side check failed (status word) */
} lq_status;

typedef enum lq_dtype { LQ_F32 = 0, LQ_F16 = 1, LQ_BF16 = 2 } lq_dtype;

typedef void* lq_stream; /* a cudaStream_t */

#if defined(__GNUC__)
#define LQ_API __attribute__((visibility("default")))
#else
#define LQ_API
#endif

/* The whitening transform T: xt = H_Bh (sign . chan_scale . x) / sqrt(Bh) on each
 * contiguous block of Bh inputs, H in Sylvester (natural) order,
 * H[i][j] = (-1)^popcount(i & j). A NULL descriptor, or block == 0, is the identity. */
typedef struct lq_whiten_desc {
  const int8_t* sign;       /* [K] device, entries +1/-1; NULL = all +1 */
  const float* chan_scale;  /* [K] device; NULL = all 1 */
  int32_t block;            /* Bh: 0 (identity) or a power of two <= LQ_MAX_HADAMARD dividing K */
} lq_whiten_desc;

/* ABI version (LQ_ABI_VERSION) of the loaded library. */
LQ_API int32_t lq_abi_version(void);

/* Stored bits per row, ceil(K/d) * D (the paper's rate D/d when d divides K).
 * Returns -1 if K < 1, d < 1, D < d or D > LQ_MAX_D. */
LQ_API int64_t lq_lifted_bits(int32_t K, int32_t d, int32_t D);

/* Bytes per stored row: the lifted bits rounded up to a multiple of 16 bytes.
 * Returns -1 on invalid sizes (as lq_lifted_bits). */
LQ_API int64_t lq_row_stride_bytes(int32_t K, int32_t d, int32_t D);

/* Pack sign codes into LQ_FORMAT_V1 rows (offline step, paper sec. 3.1: w ~= M w_q).
 *   b_pm1  [N][ceil(K/d)*D] int8: entries < 0 are stored as -1, all others as +1.
 *   packed [N][lq_row_stride_bytes/4] uint32, 16-byte aligned; padding bits are written as 0.
 * Errors: LQ_EINVAL for null pointers, misalignment or invalid sizes (N >= 0; N = 0 is a no-op). */
LQ_API lq_status lq_pack(const int8_t* b_pm1, int32_t N, int32_t K, int32_t d, int32_t D,
                  uint32_t* packed, lq_stream stream);

/* Inverse of lq_pack: packed rows -> [N][ceil(K/d)*D] int8 of +1/-1. Padding is ignored. */
LQ_API lq_status lq_unpack(const uint32_t* packed, int32_t N, int32_t K, int32_t d, int32_t D,
                    int8_t* b_pm1, lq_stream stream);

/* Encoding searches of lq_encode. */
typedef enum lq_encode_mode {
  LQ_ENCODE_EXACT = 0,   /* all 2^D codewords, D <= 24 */
  LQ_ENCODE_SEEDED = 1   /* the first d coordinates solved, the other D - d enumerated */
} lq_encode_mode;

/* Nearest-codeword encoding of a weight matrix (paper sec. 3.1, the inner minimisation of
 * Eq. (1): every length-d block w of a row becomes the b in {+1,-1}^D that minimises
 * ||w - M b||^2; review "Method": the search in the lifted space, cut from 2^D to 2^(D-d)
 * candidates by a pseudo-inverse initialisation, practical up to D - d = 20 by its
 * "Limitations"). LQ_ENCODE_SEEDED reads that initialisation as: for every free part
 * b_F in {+1,-1}^(D-d) (coordinates d..D-1), u = M_S^-1 (w - M_F b_F) with M_S = M[:, 0..d),
 * b_i = +1 when u_i >= 0, else -1, for i < d. Either search keeps the candidate of smallest
 * distance, ties going to the smallest index (the codeword c with b_j = -1 exactly when bit j
 * of c is set, or the free part). Runs in fp32: candidates within fp32 rounding of each other
 * may be ordered differently than in exact arithmetic.
 *   w     [N][K] fp32 device, row-major; each row is zero-padded to ceil(K/d)*d.
 *   M     [d][D] fp32 device.
 *   b_pm1 [N][ceil(K/d)][D] int8 device, +1/-1: the codes in the layout lq_pack takes.
 *   err   [N][ceil(K/d)] fp32 device or NULL: ||w_block - M b||^2 of every block; NaN for
 *         LQ_ENCODE_SEEDED when M_S is singular.
 * Errors: LQ_EINVAL for null pointers (w, M, b_pm1), misaligned w/M/err, N < 0, K < 1, d < 1,
 * D < d, D > LQ_MAX_D or an unknown mode; LQ_EUNSUPPORTED for d > 16, exact with D > 24, or
 * seeded with D - d > 24; LQ_ECUDA for a failed launch. N = 0 is a no-op. Asynchronous on
 * `stream`. */
LQ_API lq_status lq_encode(const float* w, int32_t N, int32_t K, const float* M, int32_t d,
                           int32_t D, int32_t mode, int8_t* b_pm1, float* err, lq_stream stream);

/* Whitening alone: xt = T(x) (review, "Method": Hadamard mixing plus scalings).
 *   x  [batch][K] of dtype xdt;  xt [batch][K] float32.
 * Errors: LQ_EINVAL (null pointers, batch < 0, K < 1, bad block), LQ_EUNSUPPORTED
 * (block > LQ_MAX_HADAMARD). */
LQ_API lq_status lq_whiten(const void* x, lq_dtype xdt, int32_t batch, int32_t K,
                    const lq_whiten_desc* T, float* xt, lq_stream stream);

/* Whitening fused with the lift: z[t][g*D + j] = sum_{i<d} M[i][j] * T(x[t])[g*d + i],
 * with T(x) zero beyond K (review, "Method": T* = lift composed with T).
 *   M [d][D] float32 row-major; z [batch][ceil(K/d)*D] float32. */
LQ_API lq_status lq_lift(const void* x, lq_dtype xdt, int32_t batch, int32_t K,
                  const lq_whiten_desc* T, const float* M, int32_t d, int32_t D, float* z,
                  lq_stream stream);

/* Workspace bytes lq_gemm needs for this shape (0 on invalid sizes). */
LQ_API size_t lq_gemm_workspace_bytes(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D);

/* Number of kernels one lq_gemm call launches for this shape and Hadamard block (0 on invalid
 * sizes). Host-only, touches no device. No counterpart on the pages: it lets a caller account
 * for launches (graph sizing, profiling). */
LQ_API int32_t lq_gemm_launches(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D,
                                int32_t block);

/* Which kernels lq_gemm runs for this shape and Hadamard block (-1 on invalid sizes). Host-only,
 * touches no device. No counterpart on the pages: it lets tests and profiles name the path.
 *   LQ_ROUTE_GEMV_I8     int8 tensor-core GEMV over bit planes, prologue + contraction kernels
 *   LQ_ROUTE_NONE        no plan fits the shape: lq_gemm returns LQ_EUNSUPPORTED
 *   LQ_ROUTE_GEMM_TC     tcgen05 tensor-core GEMM over fp16 z (batch >= 64, or where cheaper)
 *   LQ_ROUTE_GEMV_GROUPS LQ_ROUTE_GEMV_I8 once per group of tokens
 *   LQ_ROUTE_GEMV_BULK   int8 tensor-core GEMV, prologue + contraction kernels, the codes
 *                        streamed through shared memory by TMA (batch <= 8 where its plan fits)
 *   LQ_ROUTE_GEMM_DQ     W = blockwise M b dequantised once to fp16 in the workspace, then a
 *                        dense tcgen05 GEMM of fp16 T(x) against W (large batches, where its
 *                        D/d-times smaller contraction outweighs writing and reading W) */
#define LQ_ROUTE_GEMV_I8 0
#define LQ_ROUTE_NONE 1
#define LQ_ROUTE_GEMM_TC 2
#define LQ_ROUTE_GEMV_GROUPS 3
#define LQ_ROUTE_GEMV_BULK 4
#define LQ_ROUTE_GEMM_DQ 5
LQ_API int32_t lq_gemm_route(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D,
                             int32_t block);

/* The decode operator, y = s . (W T(x)) (paper sec. 3 intro: o = diag(s) W (M T a);
 * review: diag(s) W_q (T* a)).
 *   x       [batch][K] of dtype xdt (f32, f16 or bf16)
 *   packed  [N][lq_row_stride_bytes/4] uint32 LQ_FORMAT_V1 rows, 16-byte aligned
 *   M       [d][D] float32;  s [N] of dtype sdt;  y [batch][N] float32 (overwritten)
 *   workspace: lq_gemm_workspace_bytes(...) bytes, 256-byte aligned, caller-owned.
 *     It must be zero-filled before its first use; every call leaves it ready for the next.
 * Accumulation is exact in int32 (the GEMV routes add integer products of int8 planes of z) or
 * fp32 in a fixed order (tensor-core GEMM): the result does not depend on timing.
 * Errors: LQ_EINVAL (null or misaligned pointers, batch < 1, N < 1, bad sizes,
 * workspace too small), LQ_EUNSUPPORTED (block > LQ_MAX_HADAMARD, or a shape that no kernel
 * plan fits: lq_gemm_route reports LQ_ROUTE_NONE), LQ_ECUDA. */
LQ_API lq_status lq_gemm(const void* x, lq_dtype xdt, int32_t batch, const lq_whiten_desc* T,
                  const uint32_t* packed, const float* M, const void* s, lq_dtype sdt,
                  int32_t d, int32_t D, int32_t K, int32_t N, float* y, void* workspace,
                  size_t workspace_bytes, lq_stream stream);

/* lq_gemm on a chosen route (LQ_ROUTE_GEMV_I8, _GEMM_TC, _GEMV_GROUPS, _GEMV_BULK or _GEMM_DQ)
 * instead of the one lq_gemm_route picks: the same operator and arguments, for comparing the
 * kernel families on one shape (both large-batch GEMMs, for instance). No counterpart on the
 * pages. The workspace must hold lq_gemm_route_workspace_bytes(..., route) bytes, zero-filled
 * before its first use. Errors: as lq_gemm, plus LQ_EINVAL for an unknown route and
 * LQ_EUNSUPPORTED when the route's plan does not fit the shape. */
LQ_API lq_status lq_gemm_on_route(const void* x, lq_dtype xdt, int32_t batch,
                                  const lq_whiten_desc* T, const uint32_t* packed,
                                  const float* M, const void* s, lq_dtype sdt, int32_t d,
                                  int32_t D, int32_t K, int32_t N, float* y, void* workspace,
                                  size_t workspace_bytes, int32_t route, lq_stream stream);

/* Workspace bytes of lq_gemm_on_route for this shape, Hadamard block and route; 0 on invalid
 * sizes or when the route's plan does not fit. */
LQ_API size_t lq_gemm_route_workspace_bytes(int32_t batch, int32_t K, int32_t N, int32_t d,
                                            int32_t D, int32_t block, int32_t route);

/* The plan of the TMA-staged GEMV (LQ_ROUTE_GEMV_BULK) for this shape and Hadamard block.
 * Host-only, touches no device; no counterpart on the pages: it lets tests check the plan's
 * coverage and bounds. out[0 .. LQ_STAGED_PLAN_FIELDS) receives: ok (0: no staged plan fits),
 * K-slices S, chunks per slice, row ranges R, rows per range (ranges 0 .. rrem-1 take one more),
 * rrem, rows per stage, chunks per window, ring stages, 512-coordinate chunks per row, dynamic
 * shared memory of the contraction kernel and of the prep kernel (bytes).
 * Errors: LQ_EINVAL on invalid sizes or a null out. */
#define LQ_STAGED_PLAN_FIELDS 12
LQ_API lq_status lq_gemv_staged_plan(int32_t batch, int32_t K, int32_t N, int32_t d, int32_t D,
                                     int32_t block, int64_t* out);

/* Bytes of the scratch array that lq_gemm_noalloc keeps on every device that loads the library. */
#define LQ_NOALLOC_SCRATCH_BYTES (8u << 20)

/* lq_gemm for callers that cannot allocate device memory. The paper has no counterpart: this is
 * a deployment entry point of this library, not a step of the method.
 * Some callers cannot hand the library a workspace: their device memory is owned by a host
 * framework or allocator they cannot call into (a plugin, an inference-server backend with a
 * fixed budget), or they run where allocating is not allowed. This entry point takes the same
 * arguments as lq_gemm except the workspace, allocates nothing (no cudaMalloc, no cudaFree, no
 * allocating library routine) and keeps its scratch in a fixed device array of
 * LQ_NOALLOC_SCRATCH_BYTES bytes that every GPU which loads the library holds until the process
 * exits. The array holds what lq_gemm keeps in its workspace on this path: the prologue's int8
 * activation fragments (most of it for large K), their per-chunk column weights and sums of z,
 * the split-K completion counters and the fp32 slice partials.
 *   - batch 1..8 (the small-batch GEMV); shapes whose scratch would exceed
 *     LQ_NOALLOC_SCRATCH_BYTES are rejected with LQ_EINVAL and a reason in lq_last_error().
 *   - The first call on a device sets that device up (finds the array's device address and
 *     clears its counters, synchronising the device): make that first call before any stream
 *     capture.
 *   - Every call on a device shares the one array and leaves it ready for the next call; calls
 *     that overlap on the GPU (different streams, or threads without ordering) race on it and
 *     must be serialised by the caller.
 * Errors: as lq_gemm, plus LQ_EINVAL for batch > 8 or a scratch need above the maximum, and
 * LQ_EUNSUPPORTED when no single-launch GEMV plan fits the shape (its K-slices cannot widen
 * enough for a CTA's rows to fit its warps' partial slots, e.g. 5..8 tokens of a 28672-row
 * layer); lq_gemm runs such batches as token groups. */
LQ_API lq_status lq_gemm_noalloc(const void* x, lq_dtype xdt, int32_t batch,
                                 const lq_whiten_desc* T, const uint32_t* packed, const float* M,
                                 const void* s, lq_dtype sdt, int32_t d, int32_t D, int32_t K,
                                 int32_t N, float* y, lq_stream stream);

/* Workspace bytes of lq_codebook_round for S samples (0 on invalid sizes). */
LQ_API size_t lq_codebook_workspace_bytes(int64_t S, int32_t d, int32_t D);

/* One round of the offline codebook fit (review "Method": M is fitted to a standard Gaussian;
 * paper sec. 3.1, Eq. (1): M* = argmin E ||w - M b*(w)||^2, its text cut before the gradient
 * path). Reading: alternating minimisation over samples w_s:
 *   (1) b_s = the nearest codeword of w_s under M (lq_encode's search, `mode` as there);
 *   (2) M = (sum_s w_s b_s^T)(sum_s b_s b_s^T)^-1, the least-squares fit with the codes fixed
 *       (where the straight-through gradient -2 sum_s (w_s - M b_s) b_s^T vanishes).
 *   w      [S][d] fp32 device (the samples, e.g. N(0, 1) draws).
 *   M      [d][D] fp32 device: read by step (1), overwritten by step (2) unless sum b b^T is
 *          singular, in which case it is left unchanged and *mse is -1.
 *   b_out  [S][D] int8 device (+1/-1 codes of step (1)) or NULL (the workspace holds them).
 *   mse    one fp64 on the device or NULL: sum_s ||w_s - M b_s||^2 / (S d) of step (1) (the
 *          encoder's fp32 distances added in fp64).
 *   workspace: lq_codebook_workspace_bytes(S, d, D) bytes, 256-byte aligned, caller-owned.
 * The sums run in fp64 (sum w b^T) and exactly in int64 (sum b b^T) in a fixed order, the solve
 * in fp64 with partial pivoting: the result does not depend on timing. Asynchronous on
 * `stream`. Errors: LQ_EINVAL (null or misaligned pointers, S < 1, bad sizes, unknown mode,
 * workspace too small), LQ_EUNSUPPORTED (as lq_encode), LQ_ECUDA. */
LQ_API lq_status lq_codebook_round(const float* w, int64_t S, float* M, int32_t d, int32_t D,
                                   int32_t mode, int8_t* b_out, double* mse, void* workspace,
                                   size_t workspace_bytes, lq_stream stream);

/* Synchronise `stream`, then read the workspace status word into *code (0 = no device-side
 * failure) and clear it. Returns LQ_OK, or the lq_status that the word records. */
LQ_API lq_status lq_device_status(void* workspace, int32_t* code, lq_stream stream);

/* Checks the device-side timeout path: launches one warp that waits on a barrier nothing ever
 * arrives on, with the bounded wait the kernels use (suspending try_wait plus a %globaltimer
 * deadline) cut to limit_ms (1..1000). When the deadline passes the warp records
 * LQ_ETIMEOUT in the workspace status word and returns; lq_device_status then reports it.
 * The context stays usable: the same workspace serves the next lq_gemm once the status has
 * been read. No counterpart on the pages. Errors: LQ_EINVAL (null or misaligned workspace,
 * limit out of range), LQ_ECUDA (launch). */
LQ_API lq_status lq_check_wait_timeout(void* workspace, int32_t limit_ms, lq_stream stream);

/* Static text for a status code. */
LQ_API const char* lq_status_string(lq_status status);

/* Reason for the last rejected call on this host thread ("" if none). */
LQ_API const char* lq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* LIBLQ_H */
