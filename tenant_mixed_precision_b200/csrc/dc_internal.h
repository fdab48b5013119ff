// Declarations shared by the host and CUDA translation units of the library.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "dc.h"
#include "dc_layout.h"

#include <nvtx3/nvToolsExt.h>

// An NVTX range named after the entry point for the duration of the call (header-only NVTX v3: a
// no-op unless a profiler or tracer is attached to the process).
struct DcNvtxRange {
  explicit DcNvtxRange(const char* name) { nvtxRangePushA(name); }
  ~DcNvtxRange() { nvtxRangePop(); }
  DcNvtxRange(const DcNvtxRange&) = delete;
  DcNvtxRange& operator=(const DcNvtxRange&) = delete;
};
#define DC_NVTX(name) DcNvtxRange dc_nvtx_range_(name)

dc_status dc_fail(dc_status st, const char* fmt, ...);
dc_status dc_cuda_check(cudaError_t e, const char* what);
void dc_clear_error();
dc_status dc_check_desc(const dc_factor_desc* d, DcLayout* L);
void dc_fill_handle(const dc_factor_desc* desc, const DcLayout& L, void* dev, dc_delta_handle* out);
uint16_t dc_f64_to_f16(double x);
double dc_f16_to_f64(uint16_t h);
// One group of round-to-nearest quantisation (the rule of dc_quantize_rtn): n values at stride
// `stride` -> codes at stride `cstride`, sz = fp16 bits of (scale, zero).  False on a non-finite
// value or an fp16 scale overflow.
bool dc_rtn_group(const float* v, int64_t stride, int n, int bits, uint8_t* codes, int64_t cstride, uint16_t* sz);

// Limits of this build.
#define DC_MAX_TENANTS 8192     // routing histogram lives in shared memory
#define DC_TOK_BLOCK 64         // tokens per output block of the decode output kernel
#define DC_V_NT 2               // 16-rank tiles per V work item
#define DC_V_TOKS 4             // tokens per V/U pass (two pairs)
#define DC_XBLK 1616            // per (token, 512-column block): 3 limb rows of 512 B, 4 x 4 fp32 limb sums, pad

// Status word slots at the start of the workspace.
enum {
  DC_WS_STATUS = 0,
  DC_WS_NSEG = 1,
  DC_WS_VCOUNTER = 2,
  DC_WS_NITEMS = 3,
  DC_WS_UCOUNTER = 4,
  DC_WS_BCOUNTER = 5,
  DC_WS_SLOTS = 64
};

// One V work item, self-contained (written by the prep kernel, read with one 64-byte load):
// a band's tiles tile0 .. tile0+ntiles-1 of one tenant's linear for one 4-token pass.
// 16-byte aligned: it is moved with 16-byte vector loads and stores.
struct alignas(16) DcVItem {
  int64_t vbase;       // device address of the tile group's first block
  int64_t sbase;       // device address of S[rank0]
  int32_t f4;          // bytes of one full 512-column block of the group (distance between blocks)
  int32_t bits;
  int32_t rows_left;   // ranks of the band from tile0 on (rows of tile i = min(16, rows_left - 16 i))
  int32_t ntiles;
  int32_t nkb, tail_groups;
  int32_t p, m;        // linear, input
  int32_t tok0, ntok;  // sorted token positions of the pass
  int32_t rank0;       // rank of row 0 of tile0
  int32_t pad;
};

// One (linear, segment) record for the output kernel, self-contained.
struct DcUBand {
  int32_t bits, rank, r0;
  int32_t quads, steps, last;  // U geometry of the band (dc_layout.h)
  int32_t nblk, full;          // blocks per 128-row group and bytes of a full block
  int32_t boff;                // offset of the band inside a run
  int32_t pad[3];
};
struct alignas(16) DcURec {  // moved with 16-byte vector loads and stores
  int64_t blob;
  int64_t u_off;  // start of the 128-row group runs (blob-relative)
  int32_t valid, tenant, st, len, r, n_bands, u_unit;
  float umax;     // bound on the U scales of the 2/3-bit bands
  DcUBand band[DC_MAX_BANDS];
};

// Workspace layout (byte offsets from the workspace base).
struct DcWs {
  int32_t T, max_rank, max_d_in, n_lin, n_in, r_stride, max_items, max_tenants, nkb, pad;
  int32_t bt_nb;     // token block of the tensor-core backbone (multiple of 16, <= 256)
  int32_t bt_units;  // upper bound on its (linear, 128-row tile, token block) units
  int32_t tcols;     // columns of the fp16 t plane: every band starts on a multiple of 64
  int32_t pad2;
  int64_t status, perm, inv, segs, items, urecs, xl, xsort, xe, tws, yd, dflag, tmax, bt_part, bt_cnt;
  int64_t tseg;      // per tenant-sorted token: its segment
  int64_t t16;       // fp16 t / 2^E(token): [n_lin][T][tcols] (prefill path)
  int64_t xs16;      // fp16 x * 2^(14 - E(token)), tenant-sorted: [n_in][T][max_d_in] (prefill path)
  int64_t x8;        // E4M3 codes of x / s(token), tenant-sorted: [n_in][T][max_d_in] (fp8 backbone)
  int64_t sx8;       // s(token) = max|x| / 448: [n_in][T] fp32 (fp8 backbone)
  int64_t total;
};

// Segments of at least DC_PF_MIN tokens take the tensor-core (prefill) delta path when the batch
// has at least twice that many tokens (a build may set another threshold with -DDC_PF_MIN=n; the
// workspace size follows it).
#ifndef DC_PF_MIN
#define DC_PF_MIN 64
#endif

// Tensor-core backbone: CTAs of the persistent grid (at most; 148 SMs on B200) and the partial
// tiles they may leave for split units (two per CTA: its first and its last unit).
#define DC_BT_MAX_CTAS 148

DcWs dc_ws_layout(int32_t T, int32_t max_rank, int32_t max_d_in, int32_t n_lin, int32_t max_tenants);
