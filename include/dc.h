/*
 * dc.h -- C ABI of the B200 multi-tenant mixed-precision delta library.
 *
 * What it computes.  Delta-CoMe keeps the delta between a fine-tuned linear layer and its
 * backbone, Delta = W_ft - W_base, as SVD factors Delta ~= U diag(S) V^T whose singular vectors
 * are quantised at 8, 3 or 2 bits by singular-value rank, with the smallest ranks dropped (0 bit):
 *   - "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法" (paooo.com), section
 *     "Delta-CoMe的技术原理": SVD of the delta; more bits for the singular vectors of larger
 *     singular values; long-tail spectrum;
 *   - "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for Large Language
 *     Models" (atlas.scime.ai summary), section "Approach": 8/3/2-bit groups for successive
 *     singular vectors, the smallest ones 0-bit, at the size of a 1-bit delta; sections
 *     "Problem" and "Key results": many fine-tuned models served from one GPU.
 * At serving time every token k of a batch carries a tenant id tau(k) and gets
 *     y_k = W_base x_k + U_hat_tau (S_tau * (V_hat_tau^T x_k)),
 * with tenant id -1 meaning "backbone only".  Quantisation is round-to-nearest in groups of 128
 * consecutive elements of each singular vector with an fp16 scale and an fp16 zero point per
 * group: v_hat = (code - zero) * scale.
 *
 * Conventions.
 *   - Every entry point returns dc_status; DC_OK is 0.  No entry point aborts or traps.  The
 *     text of the last error of the calling thread is returned by dc_last_error().
 *   - The library never allocates device memory.  The caller allocates every device buffer
 *     (packed stores, tenant tables, workspaces, outputs) and passes raw device pointers and a
 *     cudaStream_t (as void*; NULL = legacy default stream).  Host pointers are borrowed for the
 *     duration of the call only.
 *   - Device entry points are asynchronous on the given stream unless stated otherwise.
 *   - Device pointers must be 16-byte aligned (DC_ERR_ALIGN otherwise).
 *   - d_out and d_in must be multiples of 128 (DC_ERR_SHAPE otherwise).
 *   - Bit widths must be 0, 2, 3 or 8 (DC_ERR_BITS otherwise).
 *   - Errors found by a kernel (a tenant id out of range) are written to a status word in the
 *     workspace and read back with dc_read_device_status(); the kernel skips the bad token.
 */
#ifndef DC_H
#define DC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t dc_status;
enum {
  DC_OK = 0,
  DC_ERR_INVALID_ARG = 1,  /* null pointer, negative size, non-finite factor, ...        */
  DC_ERR_SHAPE = 2,        /* dimension not a multiple of 128, rank above min(d_out,d_in) */
  DC_ERR_BITS = 3,         /* bit width not in {0, 2, 3, 8}                               */
  DC_ERR_ALIGN = 4,        /* device pointer not 16-byte aligned                          */
  DC_ERR_WORKSPACE = 5,    /* workspace or destination buffer too small                   */
  DC_ERR_TENANT = 6,       /* tenant id out of range (host check or device status word)    */
  DC_ERR_CUDA = 7,         /* a CUDA runtime call failed                                  */
  DC_ERR_UNSUPPORTED = 8   /* a valid request this build does not serve (see message)     */
};

/* DC_DTYPE_FP8 is a backbone weight format only (dc_linear.w_dtype): W_base then points at the
 * E4M3 codes row-major [d_out, d_in] followed directly by the fp32 row scales [d_out]
 * (dc_quantize_fp8_rows, dc_quantize_fp8_rows_device); the activations (bf16 or fp32) are
 * quantised per token inside the call.  With DC_BASE, either every linear of a call is fp8 or none
 * is (DC_ERR_UNSUPPORTED otherwise). */
enum { DC_DTYPE_F32 = 0, DC_DTYPE_BF16 = 1, DC_DTYPE_FP8 = 2 };

/* flags of dc_delta_linear_segmented / dc_layer_forward */
enum {
  DC_BASE = 1,          /* add W_base x                                                  */
  DC_DELTA = 2,         /* add U_hat (S * (V_hat^T x)) of the token's tenant             */
  DC_REUSE_ROUTING = 4, /* skip dc_build_segments: the workspace already holds the routing
                           of these tenant ids (e.g. every layer after the first)        */
  DC_DECODE_ONLY = 8    /* serve every segment with the decode kernels, also segments of 64
                           or more tokens that would take the tensor-core prefill path
                           (for comparisons and tests)                                   */
};

#define DC_MAX_BANDS 4
#define DC_GROUP 128

/* Rank bands of one tenant's linear, in descending singular-value order: band j holds rank[j]
 * consecutive ranks stored at bits[j] bits (8, 3, 2; 0 = dropped, stores nothing). */
typedef struct {
  int32_t d_out, d_in;
  int32_t n_bands;
  int32_t bits[DC_MAX_BANDS];
  int32_t rank[DC_MAX_BANDS];
} dc_factor_desc;

/* Where one tenant's packed delta lives.  Plain data: copy it by value, or into a device-side
 * tenant table (dc_tenant_table_upload).  dev_base == 0 means "this tenant has no delta for
 * this linear" (its tokens get the backbone only). */
typedef struct {
  uint64_t dev_base;   /* device address of the packed blob (256-byte aligned) */
  uint64_t bytes;      /* size of the blob                                      */
  dc_factor_desc desc;
  int32_t rank_total;  /* sum of the ranks of the non-zero bands                */
  int32_t reserved;
} dc_delta_handle;

/* One linear of the backbone plus the deltas of every tenant for it. */
typedef struct {
  const void* W_base;        /* device, row-major [d_out, d_in], dtype w_dtype (fp8: codes then
                                row scales, see DC_DTYPE_FP8)                                  */
  int32_t w_dtype;           /* DC_DTYPE_BF16 or DC_DTYPE_FP8 (tensor-core path), or
                                DC_DTYPE_F32                                                   */
  int32_t d_out, d_in;
  int32_t n_tenants;         /* tenant ids run over 0..n_tenants-1                            */
  int32_t max_rank;          /* upper bound of rank_total over the tenants (workspace sizing) */
  const dc_delta_handle* tenants_dev;  /* device array [n_tenants] (dc_tenant_table_upload)   */
} dc_linear;

/* Text of the last error raised on the calling thread ("" if none).
 * Passage: none (error reporting of this library; no counterpart in the pages). */
const char* dc_last_error(void);

/* Library version string.  Passage: none (no counterpart in the pages). */
const char* dc_version(void);

/* Passage: "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for Large Language
 * Models", section "Approach" (singular vectors kept at 8/3/2 bits by singular-value
 * rank, the smallest dropped at 0 bits); the byte layout itself is this library's.
 * Size in bytes of the packed blob of one tenant's linear.  Returns 0 for an invalid descriptor
 * (and sets dc_last_error).  The blob holds: S as fp32 [r]; V_hat^T codes as bit planes in
 * 16-rank tiles; U_hat codes as bit planes in 16-row tiles; fp16 scale and zero per group of
 * 128 for every kept singular vector. */
size_t dc_packed_size(const dc_factor_desc* desc);

/* Passage: "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", section "Delta-CoMe的技术原理"
 * (mixed-precision quantisation of the singular vectors: higher precision for larger singular
 * values); "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for Large Language
 * Models", section "Approach" (8/3/2-bit groups).  The
 * grid (round to nearest, groups of 128, fp16 scale and zero) is this library's reading of a point
 * the pages leave open.
 * Host round-to-nearest quantiser (deterministic, fp64 arithmetic), one rule for every group
 * of 128 elements of every kept singular vector:
 *   lo = min(0, min g), hi = max(0, max g), qmax = 2^b - 1,
 *   scale = fp16_rne((hi - lo) / qmax) (1 if it is 0), zero = clamp(rint(-lo / scale), 0, qmax),
 *   code = clamp(rint(v / scale) + zero, 0, qmax), rint = round half to even.
 * U:  fp32 column-major [d_out, r] (column i = u_i);  Vt: fp32 row-major [r, d_in] (row i = v_i)
 * where r = sum of the ranks of the non-zero bands, bands in order.
 * Outputs (host, caller-owned): codes_u uint8 [r, d_out] (row i = codes of u_i),
 * codes_v uint8 [r, d_in], sz_u uint16 [r, d_out/128, 2] and sz_v uint16 [r, d_in/128, 2]
 * holding the fp16 bit patterns of (scale, zero).  DC_ERR_INVALID_ARG on a non-finite input or
 * a scale that overflows fp16. */
dc_status dc_quantize_rtn(const dc_factor_desc* desc, const float* U, const float* Vt,
                          uint8_t* codes_u, uint8_t* codes_v, uint16_t* sz_u, uint16_t* sz_v);

/* Passage: "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for Large Language
 * Models", section "Approach" (the compressed delta of one
 * tenant); the serving layout is this library's.
 * Pack host codes into the serving layout and copy them to dev_dst (caller-owned, at least
 * dc_packed_size bytes, 256-byte aligned).  S: host fp32 [r].  Synchronises the stream before
 * returning so the host buffers may be freed.  Fills *out. */
dc_status dc_pack_upload(const dc_factor_desc* desc, const uint8_t* codes_u, const uint8_t* codes_v,
                         const uint16_t* sz_u, const uint16_t* sz_v, const float* S,
                         void* dev_dst, size_t dev_bytes, void* stream, dc_delta_handle* out);

/* Passage: as dc_quantize_rtn ("Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法",
 * "Delta-CoMe的技术原理"; "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for Large
 * Language Models", "Approach").
 * Device quantiser + packer: the same rule as dc_quantize_rtn, run on the GPU from device fp32
 * factors (U column-major [d_out, r], Vt row-major [r, d_in], S [r]) straight into the serving
 * layout at dev_dst.  Produces bit-identical codes to dc_quantize_rtn.  Asynchronous.
 * scratch: caller device buffer of dc_quantize_scratch_size(desc) bytes; its first int32 is a
 * status word set to DC_ERR_INVALID_ARG if a group held a non-finite value or its fp16 scale
 * overflowed (that group is stored with zero codes); read it with dc_read_device_status. */
dc_status dc_quantize_pack_device(const dc_factor_desc* desc, const float* U_dev, const float* Vt_dev,
                                  const float* S_dev, void* dev_dst, size_t dev_bytes, void* scratch,
                                  size_t scratch_bytes, void* stream, dc_delta_handle* out);

/* Passage: "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", section "Delta-CoMe的应用场景" (multi-tenant
 * serving: one backbone, a compressed delta per customer).
 * Copy n handles into a caller-owned device array (n * sizeof(dc_delta_handle) bytes).
 * Asynchronous; the host array must stay alive until the stream reaches the copy. */
dc_status dc_tenant_table_upload(const dc_delta_handle* handles, int32_t n, void* dev_dst,
                                 size_t dev_bytes, void* stream);

/* Passage: none (sizing of this library's scratch memory; no counterpart in the pages).
 * Bytes of workspace needed by dc_delta_linear_segmented / dc_layer_forward for a batch of at
 * most T tokens whose linears have ranks up to max_rank, d_in and d_out up to max_d_in and at
 * most max_tenants tenants (n_linears = 1 or 7).  The workspace holds the routing result, the
 * per-token activation limbs, the rank-reduction results and the device status word.  The same
 * arguments must be passed to the calls that use the workspace (through dc_linear.max_rank and
 * the batch size); a workspace smaller than this gives DC_ERR_WORKSPACE.  For T >= 64 it also
 * holds the prefill path's fp16 activation and t planes. */
size_t dc_workspace_size(int32_t T, int32_t max_rank, int32_t max_d_in, int32_t n_linears,
                         int32_t max_tenants);

/* Passage: none (scratch sizing; no counterpart in the pages).
 * Quantise on the device needs plain codes as scratch: bytes of scratch for one descriptor. */
size_t dc_quantize_scratch_size(const dc_factor_desc* desc);

/* Passage: "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", section "Delta-CoMe的应用场景" (multi-tenant
 * serving); "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for Large Language
 * Models", section "Problem" (serving many fine-tuned models
 * cheaply).  Every token of a batch goes to its own tenant's delta.
 * Token routing: stable counting sort of tenant ids (device int32 [T], -1 = backbone only, -1
 * first) into the workspace: permutation, inverse permutation and the segment list
 * {tenant, start, length} in ascending tenant order.  Resets the device status word.  Ids out
 * of range set DC_ERR_TENANT in the status word and are routed as -1. */
dc_status dc_build_segments(const int32_t* tenant_ids_dev, int32_t T, int32_t n_tenants,
                            void* ws, size_t ws_bytes, void* stream);

/* Passage: none (a check helper; no counterpart in the pages).
 * Copy the routing result out of the workspace (debug/test helper; device -> caller device
 * buffers): perm int32 [T], inv_perm int32 [T], segments int32 [T, 3] (first n_segments rows
 * valid), n_segments int32 [1]. */
dc_status dc_read_segments(const void* ws, int32_t T, int32_t* perm_dev, int32_t* inv_perm_dev,
                           int32_t* segments_dev, int32_t* n_segments_dev, void* stream);

/* Passage: "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for Large Language
 * Models", sections "Problem" and "Approach" (backbone plus
 * compressed delta per fine-tuned model); "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法",
 * sections "Delta-CoMe的技术原理" (low-rank decomposition of the delta) and "Delta-CoMe的应用场景"
 * (multi-tenant serving).
 * y[T, d_out] = (flags & DC_BASE ? W_base x : 0) + (flags & DC_DELTA ? U_hat (S * V_hat^T x) : 0)
 * for every token with its own tenant.  x: device [T, d_in] of dtype_in; y: device [T, d_out]
 * of dtype_out (F32 or BF16).  Runs dc_build_segments itself.  T >= 0 (T = 0 is a no-op).
 * Arithmetic of the delta: a tenant with 64 or more tokens in a batch of at least 128 tokens
 * takes the tensor-core prefill path, which needs BF16 activations.  It multiplies fp16
 * operands: U_hat and V_hat rounded to fp16, x and t scaled per token by a power of two, t
 * rounded to fp16.  That is about 3e-4 relative L2 error on the delta.  Every other token (and
 * every token with DC_DECODE_ONLY) is exact up to fp32: integer tensor-core products of the
 * codes, scales and zeros applied in fp32.  The backbone multiplies bf16 operands (or fp32 for
 * an F32 W_base) with fp32 accumulation. */
dc_status dc_delta_linear_segmented(const dc_linear* lin, const void* x, void* y,
                                    const int32_t* tenant_ids_dev, int32_t T, int32_t dtype_in,
                                    int32_t dtype_out, int32_t flags, void* ws, size_t ws_bytes,
                                    void* stream);

/* Allocation-free variant of dc_delta_linear_segmented.  The pages have no counterpart: this
 * is a serving-runtime convenience, not part of the method.
 *
 * Some callers cannot hand the library a workspace per call: a plain C host program with no
 * caching allocator (cudaMalloc and cudaFree synchronise the whole device, which would stall
 * every other stream once per call), or a serving runtime whose device memory plan is fixed at
 * start-up and forbids allocation on the request path.  This entry point serves them from one
 * workspace compiled into the library as a static device array of DC_STATIC_WORKSPACE_BYTES
 * (16 MiB) per device, enough for one linear at decode sizes (e.g. 11008 x 4096 at 1/16 with
 * T = 64 needs about 7 MB).  It allocates nothing and calls no allocating library.
 *
 * - Arguments, layouts and results are those of dc_delta_linear_segmented without ws/ws_bytes.
 *   flags may hold DC_BASE and DC_DELTA; DC_REUSE_ROUTING is rejected (DC_ERR_INVALID_ARG):
 *   the routing is rebuilt on every call.
 * - A request whose workspace (dc_workspace_size(T, lin->max_rank, max(d_in, d_out), 1,
 *   lin->n_tenants)) exceeds DC_STATIC_WORKSPACE_BYTES is rejected with DC_ERR_WORKSPACE before
 *   anything is launched.
 * - Nothing has to be zeroed by the caller: the array is zero when the library's device code is
 *   loaded, and every call resets the status word and the work counters it uses.
 * - The first call on each device looks up the array's device address (cudaGetSymbolAddress)
 *   and keeps it; make that first call on each device outside any stream capture.
 * - There is one array per device, shared by every caller in the process: two calls on the same
 *   device that can overlap (different streams, or different threads without ordering) race on
 *   it and give wrong results.  Serialise the calls on a device.
 * - host_status: NULL, or where to store the device status word of this call (then the call
 *   waits for the stream and clears the word, like dc_read_device_status).  With T = 0 nothing
 *   is launched and *host_status is set to 0. */
#define DC_STATIC_WORKSPACE_BYTES ((size_t)16 << 20)
dc_status dc_delta_linear_segmented_static(const dc_linear* lin, const void* x, void* y,
                                           const int32_t* tenant_ids_dev, int32_t T, int32_t dtype_in,
                                           int32_t dtype_out, int32_t flags, void* stream,
                                           int32_t* host_status);

/* Passage: as dc_delta_linear_segmented; the layer shapes are those of the Llama-2 backbones
 * that "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", section "Delta-CoMe的技术原理", names.
 * The seven projections of one Llama-style decoder layer in one call, sharing one routing:
 * lin[0..6] = q, k, v, o, gate, up, down.  q, k, v, gate and up read x_h [T, hidden]; o reads
 * x_o [T, hidden]; down reads x_f [T, ffn].  y[p] receives [T, lin[p].d_out]. */
dc_status dc_layer_forward(const dc_linear lin[7], const void* x_h, const void* x_o, const void* x_f,
                           void* const y[7], const int32_t* tenant_ids_dev, int32_t T,
                           int32_t dtype_in, int32_t dtype_out, int32_t flags, void* ws,
                           size_t ws_bytes, void* stream);

/* ---- fp8 backbone weights.
 * Passage: none (the pages fix no backbone precision; an optional serving precision of the shared
 * backbone: E4M3 of the OCP 8-bit floating point specification, 1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, subnormals m 2^-9, largest finite 448).
 * Per row r of W (host fp32 [rows, cols]): scales[r] = max|W[r]| / 448 in fp32 (1 for a zero row),
 * codes[r][c] = E4M3 round-to-nearest-even of the fp32 quotient W[r][c] / scales[r], saturating at
 * +-448.  Upload codes then scales contiguously (rows * cols bytes, then rows floats) as the W_base
 * of a linear with w_dtype DC_DTYPE_FP8.  Its backbone product is then sum_j (code_w s_row)
 * (code_x s_tok), the activations quantised per token by the same rule with the token's max|x|,
 * accumulated in fp32 on the tensor cores (kind::f8f6f4). */
dc_status dc_quantize_fp8_rows(const float* W, int32_t rows, int32_t cols, uint8_t* codes, float* scales);

/* The same rule on the device, with the rounding the call applies to the activations (an IEEE fp32
 * division, then one conversion to E4M3 with round-to-nearest-even and saturation).  W: device,
 * row-major [rows, cols], dtype DC_DTYPE_F32 or DC_DTYPE_BF16, 16-byte aligned, cols a multiple of
 * 16; codes: device [rows, cols]; scales: device [rows] fp32 (both caller-owned, 16-byte aligned;
 * codes then scales contiguously is a DC_DTYPE_FP8 W_base).  A value below half the smallest
 * subnormal may come out as the negative zero code 0x80 (value 0).  Rows must be finite: a row
 * holding an infinity or NaN gets a non-finite scale.  Asynchronous on `stream`. */
dc_status dc_quantize_fp8_rows_device(const void* W, int32_t dtype, int32_t rows, int32_t cols, uint8_t* codes,
                                      float* scales, void* stream);

/* ---- Device compressor: the SVD step.
 * Passage: "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", section "Delta-CoMe的技术原理"
 * (SVD of the parameter delta); "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for
 * Large Language Models", section "Approach".
 *
 * Top-r singular triplets of Delta = W_ft - W_base on the GPU, for dc_quantize_pack_device: a
 * randomized range finder (Gaussian test matrix of r + oversample columns from `seed`, power_iters
 * power iterations, each basis made orthonormal by CholeskyQR2 with fp64 Gram matrices) and a
 * one-sided Jacobi SVD of the projected matrix, in fp32 with fp64 Jacobi sums.  W_ft, W_base: device, row-major
 * [d_out, d_in], dtype DC_DTYPE_F32 or DC_DTYPE_BF16.  Outputs (device, caller-owned):
 * U_out [r, d_out] (row i = u_i), S_out [r] (descending), Vt_out [r, d_in] (row i = v_i), each pair
 * signed so that the largest-magnitude entry of v_i is positive (the lowest index on ties).  The
 * truncation error approaches the Eckart-Young optimum sqrt(sum_{i>r} sigma_i^2) as oversample and
 * power_iters grow (e.g. oversample = r/10 + 16, power_iters = 2).  ws: caller device memory of
 * dc_svd_workspace_size bytes (256-byte aligned).  Synchronises the stream (once per Jacobi sweep,
 * to test convergence, and once per basis, to check the Cholesky pivots: DC_ERR_INVALID_ARG if the
 * basis lost rank) and returns after the outputs are written; *sweeps_out (if not NULL)
 * receives the number of Jacobi sweeps run. */
size_t dc_svd_workspace_size(int32_t d_out, int32_t d_in, int32_t r, int32_t oversample);
dc_status dc_svd_device(const void* W_ft, const void* W_base, int32_t dtype, int32_t d_out, int32_t d_in, int32_t r,
                        int32_t oversample, int32_t power_iters, uint64_t seed, float* U_out, float* S_out,
                        float* Vt_out, void* ws, size_t ws_bytes, void* stream, int32_t* sweeps_out);

/* ---- PrinMix allocation variants (offline, host, fp64).
 * Passage: "Enhancing Delta Compression in LLMs via SVD-based Quantization Error Minimization",
 * sections 2.1 (eq. 5: the output error of quantising row i of V on calibration activations X is
 * about Sigma_ii^2 dV_i X X^T dV_i^T), 2.2 (bit allocation as a 0/1 integer linear program: one
 * width per row, a bit budget, candidate widths, at most K distinct widths) and 2.3
 * (reconstruction-target correction: U refit to the quantised V before U is quantised).
 * Widths are from {0, 2, 3, 8}; a width b costs b (d_out + d_in) code bits per rank; the budget is
 * ratio * 16 * d_out * d_in code bits.  X: host fp32 [n, d_in] calibration tokens (rows).  All host
 * arrays are caller-owned; nothing is allocated on the device.
 *
 * dc_prinmix_scores: scores[i * n_widths + j] = S_i^2 |dV_i(widths[j]) X^T|^2, dV_i = v_i minus its
 *   round-to-nearest image at that width (the dc_quantize_rtn rule), v_i itself for 0 bits.
 *   Vt: [r, d_in] rows v_i.
 * dc_prinmix_allocate: the exact optimum of the ILP over those scores (widths must include 0; a
 *   dynamic program over the budget per allowed set of nonzero widths); width_out[r]; *objective =
 *   the summed error of the optimum.
 * dc_prinmix_rtc: U_out = U M with M = H G^-1, G = A A^T, H = B A^T, A = Sigma V_hat X^T,
 *   B = Sigma V X^T (the least-squares refit), by a Cholesky factorisation of G in fp64 (with a
 *   1e-12 relative ridge).  U, U_out: column-major [d_out, k] (row i of the buffer = u_i); Vt_hat:
 *   the dequantised V rows [k, d_in].  DC_ERR_INVALID_ARG if G is not positive definite.
 * dc_prinmix_compress: scores, allocation, then the kept ranks grouped into bands by width, widest
 *   first (8, 3, 2), singular-value order inside a band: desc_out (the plan), perm_out[r] (source
 *   rank of kept rank i; -1 past the kept ones), U_out [k, d_out] / S_out [k] / Vt_out [k, d_in] of
 *   the kept ranks in that order, U refit by RTC when rtc != 0.  Quantise and pack the outputs with
 *   dc_quantize_rtn and dc_pack_upload (or dc_quantize_pack_device). */
dc_status dc_prinmix_scores(const float* Vt, const float* S, int32_t r, int32_t d_in, const float* X, int32_t n,
                            const int32_t* widths, int32_t n_widths, double* scores);
dc_status dc_prinmix_allocate(const double* scores, int32_t r, const int32_t* widths, int32_t n_widths, int32_t d_out,
                              int32_t d_in, double ratio, int32_t max_kinds, int32_t* width_out, double* objective);
dc_status dc_prinmix_rtc(const float* U, const float* S, const float* Vt, const float* Vt_hat, int32_t k,
                         int32_t d_out, int32_t d_in, const float* X, int32_t n, float* U_out);
dc_status dc_prinmix_compress(const float* U, const float* S, const float* Vt, int32_t r, int32_t d_out, int32_t d_in,
                              const float* X, int32_t n, double ratio, const int32_t* widths, int32_t n_widths,
                              int32_t max_kinds, int32_t rtc, dc_factor_desc* desc_out, int32_t* perm_out,
                              float* U_out, float* S_out, float* Vt_out, double* objective);

/* ---- Tenant paging.
 * Passage: "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法", FAQ "多模型同机部署最该关注什么？"
 * (keep the frequently used models resident, load the long-tail ones on demand).
 *
 * A pager keeps at most n_slots tenants resident in a caller-owned device arena of n_slots slots of
 * slot_bytes each.  Every tenant's packed deltas for all of its linears form one host image (pinned
 * host memory, caller-owned, alive while the pager uses it); blob_offsets[i] is where the blob of
 * table i lies in the image (256-byte aligned; -1: the tenant has no delta for that linear).  The
 * pager keeps n_tables device tenant tables (the tenants_dev arrays of the linears, caller-owned,
 * already filled with every tenant's handles) pointing at the right slots: a handle's dev_base is the
 * blob's device address while the tenant is resident and 0 otherwise (its tokens then get the
 * backbone only).  Start with dev_base = 0 for every paged tenant.
 *
 * Per batch: dc_pager_prepare(ids) on the host, then enqueue the batch's kernels on compute_stream,
 * then dc_pager_commit(compute_stream).  prepare picks slots for the batch's missing tenants (least
 * recently used first, never a tenant of the batch) and, on copy_stream, waits for the last batch
 * that read each victim slot, copies the images (one cudaMemcpyAsync each) and patches the tables;
 * compute_stream is made to wait for that work.  Copies for the next batch overlap the kernels of the
 * current one when prepare is called before those kernels finish.  prepare fails with
 * DC_ERR_UNSUPPORTED (changing nothing) if a batch holds more distinct tenants than slots, and with
 * DC_ERR_TENANT on an id >= n_tenants; ids < 0 are backbone-only tokens.  scratch: caller device
 * memory of dc_pager_scratch_size bytes (16-byte aligned) for the table patches.  The pager
 * allocates no device memory; it owns CUDA events and host bookkeeping only.  One pager per device
 * and thread; its calls are not thread-safe. */
typedef struct dc_pager dc_pager;
typedef struct {
  int32_t n_tenants;    /* tenant ids 0 .. n_tenants - 1                          */
  int32_t n_slots;      /* tenants resident at once                               */
  uint64_t slot_bytes;  /* bytes of one slot (multiple of 256, >= every image)     */
  int32_t n_tables;     /* tenant tables kept current (one per linear)            */
  int32_t reserved;
} dc_pager_desc;
typedef struct {
  int64_t hits;          /* batch tenants found resident                          */
  int64_t misses;        /* batch tenants loaded                                  */
  int64_t evictions;     /* loads that displaced a resident tenant                */
  int64_t bytes_loaded;  /* host -> device image bytes                            */
  int64_t batches;       /* prepared batches                                      */
} dc_pager_stats;
size_t dc_pager_scratch_size(const dc_pager_desc* desc);
dc_status dc_pager_create(const dc_pager_desc* desc, void* arena_dev, size_t arena_bytes, void* const* tables_dev,
                          void* scratch_dev, size_t scratch_bytes, dc_pager** out);
dc_status dc_pager_set_tenant(dc_pager* pager, int32_t tenant, const void* image_host, uint64_t image_bytes,
                              const int64_t* blob_offsets);
dc_status dc_pager_prepare(dc_pager* pager, const int32_t* tenant_ids_host, int32_t T, void* copy_stream,
                           void* compute_stream);
dc_status dc_pager_commit(dc_pager* pager, void* compute_stream);
dc_status dc_pager_get_stats(const dc_pager* pager, dc_pager_stats* out);
/* Slot of a resident tenant, -1 otherwise (a check helper). */
int32_t dc_pager_slot_of(const dc_pager* pager, int32_t tenant);
/* Release the pager's events and bookkeeping (after its streams are idle). */
dc_status dc_pager_destroy(dc_pager* pager);

/* Passage: none (a check helper; no counterpart in the pages).
 * Decode the integer codes of one tenant's linear back out of the packed layout, with the same
 * device decode functions the serving kernels use.  which = 0: U codes as uint8 [r, d_out]
 * (row i = codes of u_i); which = 1: V codes as uint8 [r, d_in].  out_dev: caller device
 * buffer. */
dc_status dc_unpack_codes_debug(const dc_delta_handle* h, int32_t which, uint8_t* out_dev,
                                void* stream);

/* Passage: none (profiling; no counterpart in the pages).
 * Per-kernel timing: after dc_profile_begin(capacity) every kernel launched by the serving entry
 * points on this thread is bracketed by two CUDA events recorded on its stream (at most
 * `capacity` launches).  dc_profile_end synchronises those events, writes each launch's duration
 * in milliseconds and its kernel kind (0 routing, 1 activation prep, 2 rank reduction, 3 delta
 * output, 4 backbone output)
 * to the caller's host arrays, destroys the events and returns the number of launches recorded
 * (negative on error).  Events recorded during stream capture become graph nodes; profile eager
 * calls only. */
dc_status dc_profile_begin(int32_t capacity);
int32_t dc_profile_end(float* ms_out, int32_t* kind_out, int32_t capacity);

/* Passage: none (error reporting; no counterpart in the pages).
 * Read (and then clear) the device status word of a workspace; synchronises the stream. */
dc_status dc_read_device_status(void* ws, void* stream, int32_t* host_status);

#ifdef __cplusplus
}
#endif
#endif /* DC_H */
