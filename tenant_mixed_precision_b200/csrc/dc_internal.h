// Declarations shared by the host and CUDA translation units of the library.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "dc.h"
#include "dc_layout.h"

dc_status dc_fail(dc_status st, const char* fmt, ...);
dc_status dc_cuda_check(cudaError_t e, const char* what);
void dc_clear_error();
dc_status dc_check_desc(const dc_factor_desc* d, DcLayout* L);
void dc_fill_handle(const dc_factor_desc* desc, const DcLayout& L, void* dev, dc_delta_handle* out);
uint16_t dc_f64_to_f16(double x);
double dc_f16_to_f64(uint16_t h);

// Limits of this build.
#define DC_MAX_TENANTS 8192     // routing histogram lives in shared memory
#define DC_TOK_BLOCK 64         // tokens per output block of the decode output kernel
#define DC_V_NT 2               // 16-rank tiles per V work item
#define DC_V_TOKS 4             // tokens per V/U pass (two pairs)

// Status word slots at the start of the workspace.
enum { DC_WS_STATUS = 0, DC_WS_VCOUNTER = 1, DC_WS_NITEMS = 2, DC_WS_NSEG = 3, DC_WS_SLOTS = 64 };

// One V work item: projection p, segment seg, token pass, band, first tile, tile count.
struct DcVItem {
  int16_t p, band;
  int32_t seg;
  int32_t tile0;
  int16_t ntiles, pass;
};

// Workspace layout (byte offsets from the workspace base).
struct DcWs {
  int32_t T, max_rank, max_d_in, n_lin, n_in, r_stride, max_items, max_tenants;
  int64_t status, perm, inv, segs, items, layouts, xl, xs, xe, tws, total;
};

DcWs dc_ws_layout(int32_t T, int32_t max_rank, int32_t max_d_in, int32_t n_lin, int32_t max_tenants);
