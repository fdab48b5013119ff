// Serving kernels for multi-tenant mixed-precision deltas on B200 (sm_100a).
//
// Per batch (one call of dc_delta_linear_segmented / dc_layer_forward):
//   k_segments  token routing: stable counting sort of tenant ids into segments.
//   k_prep      per sorted token: the activation as a 24-bit fixed-point integer split into three
//               signed 8-bit limbs (so u8 x s8 tensor-core MMAs reproduce x exactly to 2^-22 of
//               the token's largest entry), limb sums per group of 128; extra blocks write one
//               self-contained record per (linear, segment) and the V work list.
//   k_vstage    rank reduction t = S * (V_hat^T x) per (linear, segment): 2/3/8-bit codes are
//               unpacked in registers into u8 MMA operands (mma.m16n8k32), the zero point and
//               the per-group fp16 scale are applied in an fp32 epilogue per group of 128.
//   k_ustage    y = W_base x (bf16 mma.m16n8k16, fp32 accumulation) plus, for every segment,
//               U_hat (S * t): B = scale * t is re-expressed per (128-row group, token) as a
//               24-bit fixed-point integer in three s8 limbs and multiplied with the u8 codes of
//               U_hat; written once per output element, in the token's original position.
//
// The method: "Delta-CoMe – 清华联合 OpenBMB 等高校开源的新型增量压缩算法" (paooo.com),
// "Delta-CoMe的技术原理" and "Delta-CoMe的应用场景"; "Delta-CoMe: Training-Free
// Delta-Compression with Mixed-Precision for Large Language Models", "Approach".
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "dc.h"
#include "dc_btsched.h"
#include "dc_devstate.h"
#include "dc_internal.h"
#include "dc_layout.h"
#include "dc_pack.h"
#include "dc_tma.h"
#include "dc_umma.h"

#define FULLMASK 0xffffffffu

// ---------------------------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint4 ldg128(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ uint2 ldg64(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ldg32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ldg16(const void* p) {
  unsigned short r;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return (uint32_t)r;
}
__device__ __forceinline__ uint32_t wsel(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// D += A(u8, 16x32, row) * B(s8, 32x8, col), int32 accumulate.
__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// D += A(bf16, 16x16, row) * B(bf16, 16x8, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void set_status(int* st, int code) { atomicCAS(st + DC_WS_STATUS, 0, code); }

// Two fp32 values to E4M3 (round to nearest even, saturating at +-448): lo in bits 0-7, hi in 8-15.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return (uint32_t)r;
}

// ---- register extraction from packed words (shared by the serving kernels and the debug unpacker)
// V, 2-bit mask layout: word 2s+hh of the lane-row, group p -> 4 codes weighted by 4^p.
__device__ __forceinline__ uint32_t v_reg_mask2(uint32_t w, int p) { return w & (0x03030303u << (2 * p)); }
// V/U shift layout 2-bit: 4 codes at position q of the word.
__device__ __forceinline__ uint32_t reg_shift2(uint32_t w, int q) { return (w >> (2 * q)) & 0x03030303u; }
// V 3-bit high plane: bit 8b + 2s + hh -> bit 2 of byte b.
__device__ __forceinline__ uint32_t v_reg_hi3(uint32_t w1, int s, int hh) {
  return ((w1 >> (2 * s + hh)) & 0x01010101u) << 2;
}
// U 3-bit high plane: bit 4j + b of a 16-bit lane value -> bit 2 of byte b.
__device__ __forceinline__ uint32_t u_reg_hi3(uint32_t h16, int j) {
  return (((h16 >> (4 * j)) & 0xFu) * 0x00810204u) & 0x04040404u;
}
// U mask layout: word j, step p -> 4 codes weighted by 4^p.
__device__ __forceinline__ uint32_t u_reg_mask2(uint32_t w, int p) { return w & (0x03030303u << (2 * p)); }

// ---------------------------------------------------------------------------------------------
// workspace
// ---------------------------------------------------------------------------------------------
DcWs dc_ws_layout(int32_t T, int32_t max_rank, int32_t max_d_in, int32_t n_lin, int32_t max_tenants) {
  DcWs W;
  std::memset(&W, 0, sizeof(W));
  W.T = T;
  W.max_rank = max_rank;
  W.max_d_in = (int32_t)dc_align(max_d_in, 128);
  W.n_lin = n_lin;
  W.n_in = n_lin == 7 ? 3 : 1;
  W.r_stride = (int32_t)dc_align(max_rank > 0 ? max_rank : 1, 4);
  W.max_tenants = max_tenants;
  const int64_t tiles = (max_rank + 15) / 16;
  const int64_t per_pass = tiles / DC_V_NT + DC_MAX_BANDS + 1;
  const int64_t passes = (int64_t)T / DC_V_TOKS + T + 1;
  W.max_items = (int32_t)std::min<int64_t>((int64_t)n_lin * passes * per_pass + 16, (int64_t)1 << 30);
  int64_t off = 0;
  auto take = [&](int64_t bytes) {
    int64_t o = off;
    off = dc_align(off + bytes, 256);
    return o;
  };
  W.status = take(DC_WS_SLOTS * 4);
  W.perm = take((int64_t)T * 4);
  W.inv = take((int64_t)T * 4);
  W.segs = take((int64_t)T * 12);
  W.items = take((int64_t)W.max_items * sizeof(DcVItem));
  W.urecs = take((int64_t)n_lin * (T > 0 ? T : 1) * sizeof(DcURec));
  W.nkb = (W.max_d_in + 511) / 512;
  W.xl = take((int64_t)W.n_in * T * W.nkb * DC_XBLK);
  W.xsort = take((int64_t)W.n_in * T * W.max_d_in * 2);
  W.xe = take((int64_t)W.n_in * T * 4);
  W.tws = take((int64_t)n_lin * T * W.r_stride * 4);
  W.yd = take((int64_t)n_lin * T * W.max_d_in * 4);
  // per-call state: delta flags (written for every token by k_prep), output bounds and backbone
  // unit counters (zeroed by k_prep)
  W.bt_nb = T <= 256 ? (int32_t)dc_align(T > 0 ? T : 1, 16) : 256;
  W.bt_units = n_lin * (W.max_d_in / 128) * (int32_t)((T + W.bt_nb - 1) / W.bt_nb);
  W.dflag = take((int64_t)n_lin * T);
  W.tmax = take((int64_t)n_lin * T * 4);
  W.bt_cnt = take((int64_t)W.bt_units * 4);
  W.bt_part = take((int64_t)2 * DC_BT_MAX_CTAS * 128 * W.bt_nb * 4);
  W.tseg = take((int64_t)T * 4);
  W.tcols = (int32_t)dc_align(max_rank > 0 ? max_rank : 1, 64) + 64 * (DC_MAX_BANDS - 1);
  W.t16 = T >= DC_PF_MIN ? take((int64_t)n_lin * T * W.tcols * 2) : take(0);
  W.xs16 = T >= DC_PF_MIN ? take((int64_t)W.n_in * T * W.max_d_in * 2) : take(0);
  W.x8 = take((int64_t)W.n_in * T * W.max_d_in);
  W.sx8 = take((int64_t)W.n_in * T * 4);
  W.total = off;
  return W;
}

extern "C" size_t dc_workspace_size(int32_t T, int32_t max_rank, int32_t max_d_in, int32_t n_linears,
                                    int32_t max_tenants) {
  DC_NVTX("dc_workspace_size");
  if (T < 0 || max_rank < 0 || max_d_in < 0 || (n_linears != 1 && n_linears != 7) || max_tenants < 0) return 0;
  return (size_t)dc_ws_layout(T, max_rank, max_d_in, n_linears, max_tenants).total;
}

struct DcLinDev {
  const void* W;
  const dc_delta_handle* tenants;
  void* y;
  int32_t d_out, d_in, n_tenants, w_dtype, input, pad;
};

struct DcFwd {
  CUtensorMap wmap[7];     // backbone weights, box 64 columns x 128 rows, 128-byte swizzle
  CUtensorMap xmap[3];     // tenant-sorted bf16 activations, box 64 columns x 64 tokens
  DcLinDev lin[7];
  const void* x[3];
  int32_t dx[3];
  int32_t n_lin, T, dtype_in, dtype_out, flags, pad;
  int32_t order[7];        // launch order of the linears in the U kernel (largest first)
  int32_t tile_prefix[8];  // cumulative 128-row output tiles in that order
  int64_t bt_chunk_prefix[8];  // tensor-core backbone: cumulative 128-byte chunks of all units, same order
                               // (with teams: of one token block's units)
  int64_t bt_total;            // total chunks
  int64_t bt_ctb;              // with teams: chunks of one token block
  int32_t bt_ntb, bt_ns, bt_grid, bt_team;  // token blocks, pipeline stages, CTAs, team size (0: no teams)
  int32_t bt_gtiles[8];        // per linear (same order): row tiles per group of the unit order
  CUtensorMap tmap;            // prefill path: fp16 t plane [n_lin T rows x tcols], box 64 x 256
  CUtensorMap xpf[3];          // prefill path: fp16 scaled tenant-sorted activations, box 64 x pf_box
  int32_t fp8;                 // the backbone weights are E4M3 codes with fp32 row scales
  int32_t pf;                  // segments of >= DC_PF_MIN tokens take the prefill delta path
  int32_t pf_box;              // min(256, T)
  DcWs ws;
};

struct WsPtr {
  int* st;
  int* perm;
  int* inv;
  int* segs;
  DcVItem* items;
  DcURec* urecs;
  uint8_t* xl;
  uint8_t* xsort;
  int* xe;
  float* tws;
  float* yd;
  uint8_t* dflag;
  int* tmax;  // per (linear, sorted token): max |t| over the 2/3-bit ranks, as fp32 bits
  int* tseg;  // per sorted token: its segment
  __half* t16;    // prefill path: t / 2^E per token as fp16
  __half* xs16;   // prefill path: x * 2^(14 - E) per token as fp16
  uint8_t* x8;    // fp8 backbone: E4M3 codes of x / s(token)
  float* sx8;     // fp8 backbone: s(token)
};
__device__ __forceinline__ WsPtr ws_ptr(const DcWs& W, uint8_t* ws) {
  WsPtr p;
  p.st = (int*)(ws + W.status);
  p.perm = (int*)(ws + W.perm);
  p.inv = (int*)(ws + W.inv);
  p.segs = (int*)(ws + W.segs);
  p.items = (DcVItem*)(ws + W.items);
  p.urecs = (DcURec*)(ws + W.urecs);
  p.xl = ws + W.xl;
  p.xsort = ws + W.xsort;
  p.xe = (int*)(ws + W.xe);
  p.tws = (float*)(ws + W.tws);
  p.yd = (float*)(ws + W.yd);
  p.dflag = ws + W.dflag;
  p.tmax = (int*)(ws + W.tmax);
  p.tseg = (int*)(ws + W.tseg);
  p.t16 = (__half*)(ws + W.t16);
  p.xs16 = (__half*)(ws + W.xs16);
  p.x8 = ws + W.x8;
  p.sx8 = (float*)(ws + W.sx8);
  return p;
}

// ---------------------------------------------------------------------------------------------
// k_segments: stable counting sort of tenant ids (-1 first).  One block; warp 0 scans.
// ---------------------------------------------------------------------------------------------
__global__ void k_segments(const int32_t* __restrict__ ids, int T, int n, uint8_t* ws, DcWs W) {
  extern __shared__ int sm_seg[];
  int* cnt = sm_seg;
  int* start = sm_seg + (n + 1);
  WsPtr P = ws_ptr(W, ws);
  const int tid = threadIdx.x, lane = tid & 31;
  for (int i = tid; i < DC_WS_SLOTS; i += blockDim.x) P.st[i] = 0;
  for (int i = tid; i <= n; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  for (int i = tid; i < T; i += blockDim.x) {
    const int id = ids[i];
    const bool ok = id >= -1 && id < n;
    if (!ok) atomicCAS(P.st + DC_WS_STATUS, 0, DC_ERR_TENANT);
    atomicAdd(&cnt[ok ? id + 1 : 0], 1);
  }
  __syncthreads();
  if (tid < 32) {
    int carry = 0, segc = 0;
    for (int base = 0; base <= n; base += 32) {
      const int i = base + lane;
      const int c = i <= n ? cnt[i] : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(FULLMASK, incl, o);
        if (lane >= o) incl += v;
      }
      if (i <= n) start[i] = carry + incl - c;
      const bool f = i >= 1 && i <= n && c > 0;
      const unsigned m = __ballot_sync(FULLMASK, f);
      const int pos = segc + __popc(m & ((1u << lane) - 1u));
      if (f) {
        P.segs[3 * pos] = i - 1;
        P.segs[3 * pos + 1] = carry + incl - c;
        P.segs[3 * pos + 2] = c;
      }
      segc += __popc(m);
      carry += __shfl_sync(FULLMASK, incl, 31);
    }
    if (lane == 0) P.st[DC_WS_NSEG] = segc;
    __syncwarp();
    for (int base = 0; base < T; base += 32) {
      const int i = base + lane;
      const bool v = i < T;
      int key = n + 1;  // sentinel for idle lanes
      if (v) {
        const int id = ids[i];
        key = (id >= -1 && id < n) ? id + 1 : 0;
      }
      const unsigned peers = __match_any_sync(FULLMASK, key);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      int pos = 0;
      if (v) pos = start[key] + rank;
      __syncwarp();
      if (v) {
        P.perm[pos] = i;
        P.inv[i] = pos;
        if (rank == 0) start[key] += __popc(peers);
      }
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------------------------------------
// k_prep: activation limbs, limb sums, exponents; extra blocks write the (linear, segment)
// records and the V work list.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ int sext8(int v) { return (int)(int8_t)(v & 0xff); }

__device__ void build_records_for(const DcFwd& F, const WsPtr& P, int p, int s) {
  const DcWs& W = F.ws;
  const int tau = P.segs[3 * s], st = P.segs[3 * s + 1], len = P.segs[3 * s + 2];
  DcURec R;
  R.blob = 0;
  R.valid = 0;
  R.tenant = tau;
  R.st = st;
  R.len = len;
  R.r = R.n_bands = R.u_unit = 0;
  R.umax = 0.f;
  R.u_off = 0;
  for (int b = 0; b < DC_MAX_BANDS; ++b) {
    DcUBand& U = R.band[b];
    U.bits = U.rank = U.r0 = U.quads = U.steps = U.last = U.nblk = U.full = U.boff = 0;
    U.pad[0] = U.pad[1] = U.pad[2] = 0;
  }
  DcLayout L;
  L.valid = 0;
  if (tau < F.lin[p].n_tenants) {
    const dc_delta_handle* h = F.lin[p].tenants + tau;
    if (h->dev_base != 0) {
      L = dc_layout(h->desc);
      if (!L.valid || L.d_out != F.lin[p].d_out || L.d_in != F.lin[p].d_in || L.r > W.r_stride) {
        L.valid = 0;
        set_status(P.st, DC_ERR_SHAPE);
      }
    }
    if (L.valid) {
      R.blob = (int64_t)h->dev_base;
      R.valid = 1;
      R.r = L.r;
      R.n_bands = L.n_bands;
      R.u_off = L.u_off;
      R.u_unit = (int32_t)L.u_unit;
      R.umax = *reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(h->dev_base) + L.umax_off);
      for (int b = 0; b < L.n_bands; ++b) {
        DcUBand& U = R.band[b];
        const DcBand& B = L.band[b];
        U.bits = B.bits;
        U.rank = B.rank;
        U.r0 = B.r0;
        U.quads = B.u_quads;
        U.steps = B.u_steps;
        U.last = B.u_last;
        U.nblk = B.u_nblk;
        U.full = B.u_full;
        U.boff = (int32_t)B.u_boff;
      }
    }
  }
  P.urecs[(int64_t)p * W.T + s] = R;
  for (int k = 0; k < len; ++k) P.dflag[(int64_t)p * W.T + st + k] = (uint8_t)R.valid;
  if (p == 0)
    for (int k = 0; k < len; ++k) P.tseg[st + k] = s;
  if (!R.valid || !(F.flags & DC_DELTA)) return;
  if (F.pf && len >= DC_PF_MIN) return;  // k_vpre computes t for this segment
  const int passes = (len + DC_V_TOKS - 1) / DC_V_TOKS;
  int per_pass = 0;
  for (int b = 0; b < L.n_bands; ++b) per_pass += (L.band[b].v_tiles + L.band[b].v_group - 1) / L.band[b].v_group;
  const int count = passes * per_pass;
  const int base = atomicAdd(P.st + DC_WS_NITEMS, count);
  if (base + count > W.max_items) {
    set_status(P.st, DC_ERR_WORKSPACE);
    return;
  }
  int k = base;
  for (int ps = 0; ps < passes; ++ps)
    for (int b = 0; b < L.n_bands; ++b) {
      const DcBand& B = L.band[b];
      const int tpi = B.v_group;
      for (int t0 = 0; t0 < B.v_tiles; t0 += tpi) {
        DcVItem it;
        it.vbase = R.blob + B.v_off + dc_v_group_block_off(B, L, t0 / tpi, 0);
        it.sbase = R.blob + 4 * (int64_t)(B.r0 + 16 * t0);
        it.f4 = (int32_t)dc_v_group_block_bytes(B, t0 / tpi, 4);
        it.bits = B.bits;
        it.rows_left = B.rank - 16 * t0;
        it.ntiles = min(tpi, B.v_tiles - t0);
        it.nkb = L.nkb;
        it.tail_groups = L.tail_groups;
        it.p = p;
        it.m = F.lin[p].input;
        it.tok0 = st + DC_V_TOKS * ps;
        it.ntok = min(DC_V_TOKS, len - DC_V_TOKS * ps);
        it.rank0 = B.r0 + 16 * t0;
        it.pad = 0;
        P.items[k++] = it;
      }
    }
}

__global__ void __launch_bounds__(256) k_prep(const __grid_constant__ DcFwd F, uint8_t* ws) {
  const DcWs& W = F.ws;
  WsPtr P = ws_ptr(W, ws);
  if (blockIdx.x >= (unsigned)W.T) {
    // record blocks: block (T + i, y) handles (linear y, segments i, i + #record blocks, ...)
    const int nseg = P.st[DC_WS_NSEG];
    const int p = blockIdx.y;
    if (p >= F.n_lin) return;
    for (int s = (blockIdx.x - W.T) * blockDim.x + threadIdx.x; s < nseg; s += (gridDim.x - W.T) * blockDim.x)
      build_records_for(F, P, p, s);
    return;
  }
  if (blockIdx.y == 0) {  // this call's output bounds and backbone unit counters start from zero
    int* cnt = reinterpret_cast<int*>(ws + W.bt_cnt);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < W.n_lin * W.T; i += W.T * blockDim.x) P.tmax[i] = 0;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < W.bt_units; i += W.T * blockDim.x) cnt[i] = 0;
  }
  if (blockIdx.y >= (unsigned)W.n_in) return;
  const int j = blockIdx.x, m = blockIdx.y;
  const int d = F.dx[m];
  const int T = W.T, maxd = W.max_d_in;
  const int i = P.perm[j];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  auto load4 = [&](int k, float (&v)[4]) {
    if (F.dtype_in == DC_DTYPE_F32) {
      const float4 q = *reinterpret_cast<const float4*>((const float*)F.x[m] + (int64_t)i * d + k);
      v[0] = q.x, v[1] = q.y, v[2] = q.z, v[3] = q.w;
    } else {
      const uint2 q = *reinterpret_cast<const uint2*>((const __nv_bfloat16*)F.x[m] + (int64_t)i * d + k);
      v[0] = __uint_as_float(q.x << 16), v[1] = __uint_as_float(q.x & 0xffff0000u);
      v[2] = __uint_as_float(q.y << 16), v[3] = __uint_as_float(q.y & 0xffff0000u);
    }
  };
  float mx = 0.f;
  for (int k = tid * 4; k < d; k += 1024) {
    float v[4];
    load4(k, v);
#pragma unroll
    for (int q = 0; q < 4; ++q) mx = fmaxf(mx, fabsf(v[q]));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(FULLMASK, mx, o));
  __shared__ float red[8];
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) mx = fmaxf(mx, red[w]);
  int e = 0;
  if (mx > 0.f) {
    int E;
    frexpf(mx, &E);  // mx < 2^E
    e = 22 - E;      // |x| * 2^e < 2^22
  }
  uint8_t* xcol = P.xl + ((int64_t)m * W.nkb * T + j) * DC_XBLK;  // block kb at + kb * T * DC_XBLK
  // prefill operand: x * 2^(e - 8) = x * 2^(14 - E), below 2^14 in magnitude; a bf16 value
  // (8 significant bits) is exact in fp16 unless it is below 2^-31 max|x|
  const float sx16 = ldexpf(1.f, e - 8);
  // fp8 backbone operand: E4M3 codes of x / s, s = max|x| / 448 (1 for a zero token), the quotient
  // rounded once in fp32 (IEEE division) and then to nearest even E4M3, saturating
  float s8 = __fdiv_rn(mx, 448.f);
  if (s8 == 0.f) s8 = 1.f;
  for (int k = tid * 4; k < d; k += 1024) {
    float v[4];
    load4(k, v);
    if (F.dtype_in == DC_DTYPE_BF16)  // tenant-sorted copy for the backbone tiles
      *reinterpret_cast<uint2*>(P.xsort + ((int64_t)(m * T + j) * maxd + k) * 2) =
          *reinterpret_cast<const uint2*>((const __nv_bfloat16*)F.x[m] + (int64_t)i * d + k);
    if (F.fp8) {
      const uint32_t c01 = e4m3x2(__fdiv_rn(v[0], s8), __fdiv_rn(v[1], s8));
      const uint32_t c23 = e4m3x2(__fdiv_rn(v[2], s8), __fdiv_rn(v[3], s8));
      *reinterpret_cast<uint32_t*>(P.x8 + (int64_t)(m * T + j) * maxd + k) = c01 | (c23 << 16);
    }
    if (F.pf) {
      const __half2 h01 = __floats2half2_rn(v[0] * sx16, v[1] * sx16);
      const __half2 h23 = __floats2half2_rn(v[2] * sx16, v[3] * sx16);
      *reinterpret_cast<uint2*>(P.xs16 + (int64_t)(m * T + j) * maxd + k) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
    }
    uint32_t w0 = 0, w1 = 0, w2 = 0;
    int s0 = 0, s1 = 0, s2 = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int xi = __float2int_rn(ldexpf(v[q], e));
      const int l0 = sext8(xi);
      const int x1 = (xi - l0) >> 8;
      const int l1 = sext8(x1);
      const int l2 = (x1 - l1) >> 8;
      w0 |= (uint32_t)(l0 & 0xff) << (8 * q);
      w1 |= (uint32_t)(l1 & 0xff) << (8 * q);
      w2 |= (uint32_t)(l2 & 0xff) << (8 * q);
      s0 += l0, s1 += l1, s2 += l2;
    }
    // [kb][limb 0 | limb 1 | limb 2 | limb sums of the block's 4 groups]
    uint8_t* blk = xcol + (int64_t)(k >> 9) * T * DC_XBLK;
    const int within = k & 511;
    *reinterpret_cast<uint32_t*>(blk + within) = w0;
    *reinterpret_cast<uint32_t*>(blk + 512 + within) = w1;
    *reinterpret_cast<uint32_t*>(blk + 1024 + within) = w2;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      s0 += __shfl_xor_sync(FULLMASK, s0, o);
      s1 += __shfl_xor_sync(FULLMASK, s1, o);
      s2 += __shfl_xor_sync(FULLMASK, s2, o);
    }
    if (lane == 0) {  // limb sums of the group (|sum| <= 128 * 128: exact in fp32)
      float* xs = reinterpret_cast<float*>(blk + 1536 + 16 * (within >> 7));
      xs[0] = (float)s0, xs[1] = (float)s1, xs[2] = (float)s2, xs[3] = 0.f;
    }
  }
  if (tid == 0) {
    P.xe[m * T + j] = e;
    if (F.fp8) P.sx8[m * T + j] = s8;
  }
}

// ---------------------------------------------------------------------------------------------
// k_vstage: t = S * (V_hat^T x).  Persistent CTAs of 8 consumer warps + 1 producer warp.  The
// producer takes one work item at a time (prefetching the next item's record), and streams the
// item's 512-column blocks -- codes and meta of every tile, the activation limbs and limb sums of
// the pass's tokens -- into a ring of shared-memory stages with bulk copies; consumer warp w
// decodes tile w from shared memory into u8 MMA operands.  With the item's last block the producer
// also stages S of the item's ranks and the tokens' activation exponents for the epilogue.
// ---------------------------------------------------------------------------------------------
#define V_STAGES 4
#define V_CTAS_PER_SM 2  // two CTAs per SM: twice the warps to hide the consumers' latencies
#define V_A_BYTES 18432   // one block of the item's tiles: 8 x 2304 (2-bit), 5 x 3328 (3-bit), 2 x 8448 (8-bit)
#define V_XTOK DC_XBLK    // one token's limb block in shared memory (1616: offsets tokens by 20 banks)
#define V_X_BYTES (4 * V_XTOK)
#define V_S_BYTES 512     // the item's S (at most 128 ranks), staged with its last block
#define V_STAGE_BYTES (V_A_BYTES + V_X_BYTES + V_S_BYTES)
#define V_CONSUMERS 8
#define V_THREADS (32 * (V_CONSUMERS + 1))

struct VDesc {
  int kind;  // 0 block, 1 end
  int bits, rows_left, ntiles, tok0, ntok, m, p, kb, ngrp, first, last, rank0, pad;
  int64_t sbase;
  int e[DC_V_TOKS];  // activation exponents of the pass tokens (set with the item's last block)
};

struct VSmemTail {
  VDesc desc[V_STAGES];
  uint64_t full[V_STAGES];
  uint64_t empty[V_STAGES];
  DcVItem rec[2];  // producer: current and next item
};
// two CTAs per SM: 228 KB of shared memory per SM, 1 KB of it reserved per CTA; 16-byte staged rows
static_assert(V_STAGES * V_STAGE_BYTES + sizeof(VSmemTail) + 1024 <= 233472 / V_CTAS_PER_SM &&
                  (V_A_BYTES + V_X_BYTES) % 16 == 0 && V_STAGE_BYTES % 16 == 0,
              "rank-reduction shared memory");

// acc[q] += s_row * (C[q] - z_row * xs_tok).  C entries: q = 0 (row g, pair token 0), 1 (row g,
// token 1), 2 (row g+8, token 0), 3 (row g+8, token 1).  Tokens past the pass have zero limbs and
// zero limb sums, so their entries stay zero.
__device__ __forceinline__ void v_epi(float (&acc)[4], const int (&C)[4], float sA, float zA, float sB, float zB,
                                      float x0, float x1) {
  acc[0] = fmaf(sA, fmaf(-zA, x0, (float)C[0]), acc[0]);
  acc[2] = fmaf(sB, fmaf(-zB, x0, (float)C[2]), acc[2]);
  acc[1] = fmaf(sA, fmaf(-zA, x1, (float)C[1]), acc[1]);
  acc[3] = fmaf(sB, fmaf(-zB, x1, (float)C[3]), acc[3]);
}

// One 512-column block of one 16-rank tile for ntok <= 2 NPAIR tokens, all loops unrolled.
// FULL: the block holds 4 groups (2-bit codes then use the mask layout); otherwise ngrp < 4.
template <int BITS, int NPAIR, bool FULL>
__device__ __forceinline__ void v_block(int ntok, int rows, int ngrp_rt, const uint8_t* A, const uint8_t* X,
                                        float (&acc)[2][4], int lane) {
  const int ngrp = FULL ? 4 : ngrp_rt;
  const int g = lane >> 2, t = lane & 3;
  const int nh0 = min(rows, 8), nh1 = max(0, rows - 8);
  const bool ok0 = g < nh0, ok1 = g < nh1;
  const uint8_t* meta = A + dc_v_block_code_bytes(BITS, rows, ngrp);
  // B operand: lane g < 6 supplies limb g>>1 of pass token 2 pr + (g&1); limb sums of lane t's limb
  const int limb = g >> 1;
  const uint8_t* xrow[NPAIR];
  bool xval[NPAIR];
#pragma unroll
  for (int pr = 0; pr < NPAIR; ++pr) {
    const int tk = 2 * pr + (g & 1);
    xval[pr] = (g < 6) && (tk < ntok);
    xrow[pr] = X + (xval[pr] ? tk * V_XTOK + 512 * limb : 0) + 32 * t;
  }
  const float* xsum = reinterpret_cast<const float*>(X + 1536 + 4 * (t < 3 ? t : 0));
  uint4 wm0a = make_uint4(0, 0, 0, 0), wm0b = wm0a, wm1a = wm0a, wm1b = wm0a;
  if (BITS == 2 && FULL) {
    if (ok0) {
      wm0a = *reinterpret_cast<const uint4*>(A + dc_v_mask_off(4 * nh0, lane, 0));
      wm0b = *reinterpret_cast<const uint4*>(A + dc_v_mask_off(4 * nh0, lane, 1));
    }
    if (ok1) {
      const uint8_t* h1 = A + dc_v_half_off(2, rows, 4, 1);
      wm1a = *reinterpret_cast<const uint4*>(h1 + dc_v_mask_off(4 * nh1, lane, 0));
      wm1b = *reinterpret_cast<const uint4*>(h1 + dc_v_mask_off(4 * nh1, lane, 1));
    }
  }
#pragma unroll
  for (int grp = 0; grp < 4; ++grp) {
    if (!FULL && grp >= ngrp) break;
    // activation limbs of this group (B fragments of the 4 steps) and limb sums
    uint32_t bw[NPAIR][8];
#pragma unroll
    for (int pr = 0; pr < NPAIR; ++pr) {
      uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0;
      if (xval[pr]) {
        q0 = *reinterpret_cast<const uint4*>(xrow[pr] + grp * 128);
        q1 = *reinterpret_cast<const uint4*>(xrow[pr] + grp * 128 + 16);
      }
      bw[pr][0] = q0.x, bw[pr][1] = q0.y, bw[pr][2] = q0.z, bw[pr][3] = q0.w;
      bw[pr][4] = q1.x, bw[pr][5] = q1.y, bw[pr][6] = q1.z, bw[pr][7] = q1.w;
    }
    float xs[2 * NPAIR];
#pragma unroll
    for (int k = 0; k < 2 * NPAIR; ++k) xs[k] = (t < 3 && k < ntok) ? xsum[k * (V_XTOK / 4) + grp * 4] : 0.f;
    const uint2 mt = *reinterpret_cast<const uint2*>(meta + (grp * 8 + g) * 8);
    uint32_t a[4][4];  // [step][reg]
    if (BITS == 2 && FULL) {
      const uint32_t msk = 0x03030303u << (2 * grp);
      a[0][0] = wm0a.x & msk, a[0][1] = wm1a.x & msk, a[0][2] = wm0a.y & msk, a[0][3] = wm1a.y & msk;
      a[1][0] = wm0a.z & msk, a[1][1] = wm1a.z & msk, a[1][2] = wm0a.w & msk, a[1][3] = wm1a.w & msk;
      a[2][0] = wm0b.x & msk, a[2][1] = wm1b.x & msk, a[2][2] = wm0b.y & msk, a[2][3] = wm1b.y & msk;
      a[3][0] = wm0b.z & msk, a[3][1] = wm1b.z & msk, a[3][2] = wm0b.w & msk, a[3][3] = wm1b.w & msk;
    } else {
      const int p0 = dc_v_plane0_bytes(BITS, ngrp);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const bool ok = h ? ok1 : ok0;
        const int nh = h ? nh1 : nh0;
        const uint8_t* hb = A + dc_v_half_off(BITS, rows, ngrp, h);
        if (BITS == 8) {
          uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0;
          if (ok) {
            q0 = *reinterpret_cast<const uint4*>(hb + lane * p0 + 32 * grp);
            q1 = *reinterpret_cast<const uint4*>(hb + lane * p0 + 32 * grp + 16);
          }
          a[0][h] = q0.x, a[0][h + 2] = q0.y, a[1][h] = q0.z, a[1][h + 2] = q0.w;
          a[2][h] = q1.x, a[2][h + 2] = q1.y, a[3][h] = q1.z, a[3][h + 2] = q1.w;
        } else {
          uint2 w2 = make_uint2(0, 0);
          uint32_t w1 = 0;
          if (ok) {
            w2 = *reinterpret_cast<const uint2*>(hb + lane * p0 + 8 * grp);
            if (BITS == 3) w1 = *reinterpret_cast<const uint32_t*>(hb + 4 * nh * p0 + lane * (4 * ngrp) + 4 * grp);
          }
#pragma unroll
          for (int s = 0; s < 4; ++s)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t r = reg_shift2((s >> 1) ? w2.y : w2.x, 2 * (s & 1) + hh);
              if (BITS == 3) r |= v_reg_hi3(w1, s, hh);
              a[s][h + 2 * hh] = r;
            }
        }
      }
    }
    int C[NPAIR][4];
#pragma unroll
    for (int pr = 0; pr < NPAIR; ++pr) {
      C[pr][0] = C[pr][1] = C[pr][2] = C[pr][3] = 0;
#pragma unroll
      for (int s = 0; s < 4; ++s) mma_u8s8(C[pr], a[s][0], a[s][1], a[s][2], a[s][3], bw[pr][2 * s], bw[pr][2 * s + 1]);
    }
    // per-group scale and zero of rows g and g+8; 2-bit full blocks carry the weight 4^grp
    const float w = (BITS == 2 && FULL) ? (float)(1 << (2 * grp)) : 1.f;
    const __half2 m0 = *reinterpret_cast<const __half2*>(&mt.x);
    const __half2 m1 = *reinterpret_cast<const __half2*>(&mt.y);
    const float sA = __low2float(m0) * (1.f / w), zA = __high2float(m0) * w;
    const float sB = __low2float(m1) * (1.f / w), zB = __high2float(m1) * w;
    v_epi(acc[0], C[0], sA, zA, sB, zB, xs[0], xs[1]);
    if (NPAIR > 1) v_epi(acc[1], C[NPAIR - 1], sA, zA, sB, zB, xs[2 * NPAIR - 2], xs[2 * NPAIR - 1]);
  }
}

// Code copies: per bit width one or two token pairs; only 2-bit codes have a separate layout for
// full blocks (3/8-bit blocks take the group count at run time).  Few copies keep the consumer
// loop small in the instruction cache.
template <int BITS, int NPAIR>
__device__ __forceinline__ void v_block_dispatch_ngrp(int ntok, bool full, int rows, int ngrp, const uint8_t* A,
                                                      const uint8_t* X, float (&acc)[2][4], int lane) {
  if (BITS == 2 && full)
    v_block<BITS, NPAIR, true>(ntok, rows, 4, A, X, acc, lane);
  else
    v_block<BITS, NPAIR, false>(ntok, rows, ngrp, A, X, acc, lane);
}

template <int BITS>
__device__ __forceinline__ void v_block_dispatch(int ntok, bool full, int rows, int ngrp, const uint8_t* A,
                                                 const uint8_t* X, float (&acc)[2][4], int lane) {
  if (ntok <= 2)
    v_block_dispatch_ngrp<BITS, 1>(ntok, full, rows, ngrp, A, X, acc, lane);
  else
    v_block_dispatch_ngrp<BITS, 2>(ntok, full, rows, ngrp, A, X, acc, lane);
}

__device__ __forceinline__ uint4 ldg128_item(const DcVItem* it, int lane) {
  return ldg128(reinterpret_cast<const uint8_t*>(it) + 16 * lane);
}

__global__ void __launch_bounds__(V_THREADS, V_CTAS_PER_SM) k_vstage(const __grid_constant__ DcFwd F, uint8_t* ws) {
  extern __shared__ __align__(128) uint8_t vsm[];
  VSmemTail* tail = reinterpret_cast<VSmemTail*>(vsm + V_STAGES * V_STAGE_BYTES);
  WsPtr P = ws_ptr(F.ws, ws);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < V_STAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], V_CONSUMERS);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const int T = F.ws.T;
  if (warp == V_CONSUMERS) {
    // ---------------- producer warp
    const int nitems = P.st[DC_WS_NITEMS];
    uint32_t seq = 0;
    int it = 0;
    if (lane == 0) it = atomicAdd(P.st + DC_WS_VCOUNTER, 1);
    it = __shfl_sync(FULLMASK, it, 0);
    uint4 pf = make_uint4(0, 0, 0, 0);
    if (it < nitems && lane < 4) pf = ldg128_item(P.items + it, lane);
    for (;;) {
      // current record <- prefetched one; start fetching the next
      __syncwarp();
      if (lane < 4) reinterpret_cast<uint4*>(&tail->rec[0])[lane] = pf;
      __syncwarp();
      const bool end = it >= nitems;
      int nx = 0;
      if (!end) {
        if (lane == 0) nx = atomicAdd(P.st + DC_WS_VCOUNTER, 1);
        nx = __shfl_sync(FULLMASK, nx, 0);
        if (nx < nitems && lane < 4) pf = ldg128_item(P.items + nx, lane);
      }
      const DcVItem& I = tail->rec[0];
      const int nkb = end ? 1 : I.nkb;
      // the epilogue's operands, fetched now and staged with the item's last block: S of the item's
      // ranks (lane l: ranks 4 l .. 4 l + 3) and the pass tokens' activation exponents
      float sv[4] = {0.f, 0.f, 0.f, 0.f};
      int ev = 0;
      if (!end) {
        const float* S = reinterpret_cast<const float*>(I.sbase);
        const int nr = min(16 * I.ntiles, I.rows_left);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (4 * lane + j < nr) sv[j] = S[4 * lane + j];
        if (lane < I.ntok) ev = P.xe[I.m * T + I.tok0 + lane];
      }
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = seq % V_STAGES;
        if (seq >= V_STAGES && !mbar_wait(&tail->empty[s], ((seq / V_STAGES) - 1) & 1)) {
          set_status(P.st, DC_ERR_CUDA);
          return;
        }
        
        uint8_t* stage = vsm + (size_t)s * V_STAGE_BYTES;
        if (end) {
          if (lane == 0) {
            tail->desc[s].kind = 1;
            mbar_arrive(&tail->full[s]);
          }
          return;
        }
        const int ngrp = (kb == I.nkb - 1) ? I.tail_groups : 4;
        const int last_rows = min(16, I.rows_left - 16 * (I.ntiles - 1));
        const uint32_t code_bytes = (uint32_t)((I.ntiles - 1) * dc_v_block_bytes(I.bits, 16, ngrp) +
                                               dc_v_block_bytes(I.bits, last_rows, ngrp));
        const uint32_t total = code_bytes + (uint32_t)(I.ntok * DC_XBLK);
        if (kb == I.nkb - 1) {  // ordered before the stage's arrive by the warp barrier below
          *reinterpret_cast<float4*>(stage + V_A_BYTES + V_X_BYTES + 16 * lane) = make_float4(sv[0], sv[1], sv[2], sv[3]);
          if (lane < DC_V_TOKS) tail->desc[s].e[lane] = ev;
        }
        __syncwarp();
        if (lane == 0) {
          VDesc& d = tail->desc[s];
          d.kind = 0;
          d.bits = I.bits;
          d.rows_left = I.rows_left;
          d.ntiles = I.ntiles;
          d.tok0 = I.tok0;
          d.ntok = I.ntok;
          d.m = I.m;
          d.p = I.p;
          d.kb = kb;
          d.ngrp = ngrp;
          d.first = kb == 0;
          d.last = kb == I.nkb - 1;
          d.rank0 = I.rank0;
          d.sbase = I.sbase;
          mbar_arrive_expect_tx(&tail->full[s], total);
        }
        __syncwarp();
        if (lane == 0) {
          bulk_g2s(stage, reinterpret_cast<const uint8_t*>(I.vbase) + (int64_t)kb * I.f4, code_bytes, &tail->full[s]);
        } else if (lane == 1) {
          const uint8_t* src = P.xl + (((int64_t)I.m * F.ws.nkb + kb) * T + I.tok0) * DC_XBLK;
          bulk_g2s(stage + V_A_BYTES, src, (uint32_t)(I.ntok * DC_XBLK), &tail->full[s]);
        }
        ++seq;
      }
      it = nx;
    }
  }
  // ---------------- consumer warps
  uint32_t seq = 0;
  float acc[2][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[a][q] = 0.f;
  const int g = lane >> 2, t = lane & 3;
  for (;;) {
    const int s = seq % V_STAGES;
    if (!mbar_wait(&tail->full[s], (seq / V_STAGES) & 1)) {
      set_status(P.st, DC_ERR_CUDA);
      return;
    }
    const VDesc& d = tail->desc[s];  // read only before the stage is handed back
    if (d.kind == 1) return;
    const uint8_t* stage = vsm + (size_t)s * V_STAGE_BYTES;
    if (warp < d.ntiles) {
      if (d.first) {
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[a][q] = 0.f;
      }
      const int rows = min(16, d.rows_left - 16 * warp);
      const uint8_t* A = stage + warp * dc_v_block_bytes(d.bits, 16, d.ngrp);
      const uint8_t* X = stage + V_A_BYTES;
      const bool full = d.ngrp == 4;
      if (d.bits == 2)
        v_block_dispatch<2>(d.ntok, full, rows, d.ngrp, A, X, acc, lane);
      else if (d.bits == 3)
        v_block_dispatch<3>(d.ntok, full, rows, d.ngrp, A, X, acc, lane);
      else
        v_block_dispatch<8>(d.ntok, full, rows, d.ngrp, A, X, acc, lane);
      if (d.last) {
        // combine the three limbs (lane t holds limb t), scale by 2^-e and S, store t
        const float lw = (float)(1 << (8 * min(t, 2)));
        const float* S = reinterpret_cast<const float*>(stage + V_A_BYTES + V_X_BYTES);  // staged S
        float tmx[DC_V_TOKS] = {0.f, 0.f, 0.f, 0.f};  // max |t| per pass token over this warp's rows
#pragma unroll
        for (int pr = 0; pr < 2; ++pr)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v = t < 3 ? acc[pr][q] * lw : 0.f;
            v += __shfl_xor_sync(FULLMASK, v, 1);
            v += __shfl_xor_sync(FULLMASK, v, 2);
            const int row = g + 8 * (q >> 1);
            const int tk = 2 * pr + (q & 1);
            if (t == 0 && row < rows && tk < d.ntok) {
              const int rl = 16 * warp + row;  // row within the item
              const int tok = d.tok0 + tk;
              const float tv = ldexpf(v, -d.e[tk]) * S[rl];
              P.tws[((int64_t)d.p * T + tok) * F.ws.r_stride + d.rank0 + rl] = tv;
              tmx[tk] = fmaxf(tmx[tk], fabsf(tv));
            }
          }
        if (d.bits != 8) {  // bound for the output kernel's fixed-point exponent (2/3-bit ranks)
#pragma unroll
          for (int tk = 0; tk < DC_V_TOKS; ++tk) {
            float m = tmx[tk];
            m = fmaxf(m, __shfl_xor_sync(FULLMASK, m, 4));
            m = fmaxf(m, __shfl_xor_sync(FULLMASK, m, 8));
            m = fmaxf(m, __shfl_xor_sync(FULLMASK, m, 16));
            if (lane == 0 && tk < d.ntok && m > 0.f)
              atomicMax(P.tmax + d.p * T + d.tok0 + tk, __float_as_int(m));
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&tail->empty[s]);
    ++seq;
  }
}

// ---------------------------------------------------------------------------------------------
// k_udelta: ydelta[token, row] = (U_hat (scale * t))[row] for every token of every segment with a
// delta.  Work is taken from a global counter in chunks of (linear, segment, up to U_CHUNK
// consecutive 128-row output groups).  For each pass of <= 4 tokens and each pair of groups of
// the chunk the producer warp streams the groups' U blocks in batches of consecutive blocks
// (codes of the eight 16-row tiles and the meta of the blocks' ranks: one bulk copy per group),
// together with the pass's t values of the batch's ranks (one copy per token, shared by the two
// groups), through a ring of shared-memory stages.  One CTA per SM: consumer warp w works on
// group w / 8 of the stage and owns its rows 16 (w % 8) .. 16 (w % 8) + 15.
//
// Arithmetic of a (group, pass) unit: B = scale * t is written, per token, as the fixed-point
// integer rint(B * 2^e) with e fixed by the bound umax * max|t| (so |B * 2^e| < 2^21): one fp32
// FMA with the constant 1.5 * 2^23 leaves rint(B * 2^e) + 2^22 in the low 23 bits of the result,
// whose three low bytes are the unsigned limbs of the operand.  The tensor cores multiply the u8
// codes by those u8 limbs exactly (mma m16n8k32 u8.u8 -> s32); B column 6 is all ones, giving
// the codes' row sums, which remove the 2^22 bias.  The zero points are removed in fp32
// (sum over ranks of zero * scale * t), then the exponent.  8-bit bands are summed in fp32
// during the limb phase, one output row per thread.
// ---------------------------------------------------------------------------------------------
#define U_GSTAGE 2           // 128-row output groups per stage (same tenant, linear and pass)
#define U_STAGES 4
#define U_STAGE_BYTES 45056  // a batch of blocks (codes + meta) for each group, then the t windows
#define U_CTAS_PER_SM 1
#define U_MAXSUB 8           // blocks per batch
#define U_MAXBLK 64          // blocks per (linear, tenant) U run of one group
#define U_CHUNK 4            // 128-row output groups per chunk of work
#define U_LROW 544           // row stride of a limb matrix = rank slots per stage (rows 8 banks apart)
#define U_LBUF (16 * U_LROW) // one limb matrix: rows 6 pr + 2 limb + token-in-pair, then constant rows
#define U_CONSUMERS 16       // 8 warps per group of the stage: warp w owns rows 16 (w % 8) .. + 15
#define U_THREADS (32 * (U_CONSUMERS + 1))
#define U_MAGIC 12582912.0f  // 1.5 * 2^23

struct UDesc {
  int kind;              // 1 batch, 2 end
  int p, go, tok0, ntok;
  int ng;                // groups go, go + 1, ... in the stage (1 .. U_GSTAGE)
  int nsub;              // blocks in the batch
  int code_bytes;        // bytes of the batch's blocks of one group (group g at g * code_bytes; the t
                         // windows at U_GSTAGE * code_bytes)
  int tfl;               // floats per token t window
  int t_shift;           // position of the batch's first rank inside the t window
  int ufirst, ulast;     // the batch opens / closes its (group, pass) unit
  int error;
  alignas(16) int sub[U_MAXSUB][4];  // per block: bits | nq << 4 | ns << 8 | last << 16; nr | tile_bytes << 16;
                         // stage offset of the codes | limb slot << 16; stage offset of the meta |
                         // offset of the first rank in the t windows << 16
  float pe[DC_V_TOKS];   // 2^e per pass token
  float ie[DC_V_TOKS];   // 2^-e
};

struct UBlkE {  // producer-side table of a run's blocks
  int off, bytes, p0, p1, nr, r0;
};

struct USmemTail {
  UDesc desc[U_STAGES];
  uint64_t full[U_STAGES];
  uint64_t empty[U_STAGES];
  alignas(16) DcURec rec;        // producer: record of the current chunk
  UBlkE tbl[U_MAXBLK];           // producer: blocks of the current chunk's runs
  alignas(16) int bsub[U_MAXBLK][4];  // producer: per block of the pass, its UDesc.sub entry
  int4 bat[U_MAXBLK];                 // producer: per batch, first block | blocks << 8 | t shift << 16,
                                      // code bytes, t window floats, first t column
  int nbatch;
  alignas(16) float zpart[2][U_GSTAGE][DC_V_TOKS][8];  // per-warp zero-point sums of a stage's units (two in flight)
  float s8[U_GSTAGE][128][DC_V_TOKS + 1];  // 8-bit band sums of a unit: [row][token] (padded: no bank conflicts)
};

// D += A(u8, 16x32, row) * B(u8, 32x8, col), int32 accumulate.
__device__ __forceinline__ void mma_u8u8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// chunk u -> (linear p, segment sg, first group go0, groups ngo); linears in F.order
__device__ __forceinline__ bool ud_chunk(const DcFwd& F, int nseg, int u, int& p, int& sg, int& go0, int& ngo) {
  for (int i = 0; i < F.n_lin; ++i) {
    const int q = F.order[i];
    const int G = F.lin[q].d_out / 128;
    const int nc = (G + U_CHUNK - 1) / U_CHUNK;
    const int cnt = nseg * nc;
    if (u < cnt) {
      p = q;
      sg = u / nc;
      go0 = (u % nc) * U_CHUNK;
      ngo = min(U_CHUNK, G - go0);
      return true;
    }
    u -= cnt;
  }
  return false;
}

// Exponent e of a pass token from the bound umax * max|t|: |scale * t * 2^e| < 2^21.
__device__ __forceinline__ int ud_exponent(float umax, int tmax_bits) {
  const float bound = umax * __int_as_float(tmax_bits);
  if (!(bound > 0.f)) return 0;
  int E;
  frexpf(bound, &E);
  return max(-120, min(120, 21 - E));
}

// Limb-matrix row of B column g (0..7) for token pair pr: columns 0..5 are the limbs of the pair's
// tokens (rows 6 pr + g), column 6 a row of ones (the codes' row sums), column 7 a row of zeros.
// The constant rows are 14/15 for pair 0 and 12/13 for pair 1: with rows 8 banks apart, the rows
// one 16-lane half of a warp reads lie on four different groups of 8 banks.
__device__ __forceinline__ int ud_brow(int g, int pr) { return g < 6 ? 6 * pr + g : (pr ? 12 : 14) + (g - 6); }

// Shift-layout steps of one 16-row tile, the first of them being MMA step k0 of the block.  Every
// step but a partial last one stores all 32 lanes: lane l's 2-bit word at 4 l, its 3-bit high
// plane at 128 + 2 l.  A partial last step stores nl = 8 ceil(last / 8) lanes, row g's words
// at g * nl / 8 + t.
template <int BITS, int NPAIR>
__device__ __forceinline__ void ud_steps(const uint8_t* sb, int k0, int ns, int last, const uint8_t* brow,
                                         int pstride, int (&C)[2][4][4], int lane) {
  constexpr int SB = BITS == 3 ? 192 : 128;  // bytes of a full step (both planes)
  const int g = lane >> 2, t = lane & 3;
  const int nfull = last == 32 ? ns : ns - 1;
#pragma unroll 2
  for (int si = 0; si < nfull; ++si) {
    const uint8_t* p = sb + si * SB;
    const uint32_t wv = reinterpret_cast<const uint32_t*>(p)[lane];
    uint32_t hv = 0;
    if (BITS == 3) hv = reinterpret_cast<const uint16_t*>(p + 128)[lane];
    uint32_t a[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      a[j] = reg_shift2(wv, j);
      if (BITS == 3) a[j] |= u_reg_hi3(hv, j);
    }
#pragma unroll
    for (int pr = 0; pr < NPAIR; ++pr) {
      const uint2 bb = *reinterpret_cast<const uint2*>(brow + pr * pstride + 32 * (k0 + si));
      mma_u8u8(C[pr][0], a[0], a[1], a[2], a[3], bb.x, bb.y);
    }
  }
  if (nfull == ns) return;
  const uint8_t* p = sb + nfull * SB;
  const int nl = dc_u_step_lanes(last);
  const int ntv = nl / 8;
  uint32_t wv = 0, hv = 0;
  if (t < ntv) {
    wv = *reinterpret_cast<const uint32_t*>(p + 4 * (g * ntv + t));
    if (BITS == 3) hv = *reinterpret_cast<const uint16_t*>(p + 4 * nl + 2 * (g * ntv + t));
  }
  uint32_t a[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    a[j] = reg_shift2(wv, j);
    if (BITS == 3) a[j] |= u_reg_hi3(hv, j);
  }
#pragma unroll
  for (int pr = 0; pr < NPAIR; ++pr) {
    const uint2 bb = *reinterpret_cast<const uint2*>(brow + pr * pstride + 32 * (k0 + nfull));
    mma_u8u8(C[pr][0], a[0], a[1], a[2], a[3], bb.x, bb.y);
  }
}

// MMA over one block for this warp's 16-row tile.  `lb` is the block's slot in the limb matrix.
// C[pair][position][reg].
template <int NPAIR>
__device__ __forceinline__ void ud_mma(const uint8_t* blk, int bits, int nq, int ns, int last, int tile_bytes,
                                       const uint8_t* lb, int (&C)[2][4][4], int warp, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const uint8_t* ub = blk + warp * tile_bytes;
  const uint8_t* brow = lb + ud_brow(g, 0) * U_LROW + 8 * t;
  const int pstride = (ud_brow(g, 1) - ud_brow(g, 0)) * U_LROW;
  if (nq == 2 && ns == 0) {  // full 2-bit block: two quads in straight-line code
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 wq = *reinterpret_cast<const uint4*>(ub + 512 * q + 16 * lane);
      uint2 bq[NPAIR][4];
#pragma unroll
      for (int pr = 0; pr < NPAIR; ++pr)
#pragma unroll
        for (int ps = 0; ps < 4; ++ps)
          bq[pr][ps] = *reinterpret_cast<const uint2*>(brow + pr * pstride + 32 * (4 * q + ps));
#pragma unroll
      for (int ps = 0; ps < 4; ++ps) {
        const uint32_t msk = 0x03030303u << (2 * ps);
#pragma unroll
        for (int pr = 0; pr < NPAIR; ++pr)
          mma_u8u8(C[pr][ps], wq.x & msk, wq.y & msk, wq.z & msk, wq.w & msk, bq[pr][ps].x, bq[pr][ps].y);
      }
    }
    return;
  }
#pragma unroll 1
  for (int q = 0; q < nq; ++q) {
    const uint4 wq = *reinterpret_cast<const uint4*>(ub + 512 * q + 16 * lane);
#pragma unroll
    for (int ps = 0; ps < 4; ++ps) {
      const int step = 4 * q + ps;
      const uint32_t msk = 0x03030303u << (2 * ps);
      const uint32_t a0 = wq.x & msk, a1 = wq.y & msk, a2 = wq.z & msk, a3 = wq.w & msk;
#pragma unroll
      for (int pr = 0; pr < NPAIR; ++pr) {
        const uint2 bb = *reinterpret_cast<const uint2*>(brow + pr * pstride + 32 * step);
        mma_u8u8(C[pr][ps], a0, a1, a2, a3, bb.x, bb.y);
      }
    }
  }
  if (ns == 0) return;
  if (bits == 3)
    ud_steps<3, NPAIR>(ub + 512 * nq, 4 * nq, ns, last, brow, pstride, C, lane);
  else
    ud_steps<2, NPAIR>(ub + 512 * nq, 4 * nq, ns, last, brow, pstride, C, lane);
}

// fields read with 16-byte vector loads
static_assert(offsetof(USmemTail, zpart) % 16 == 0 && offsetof(USmemTail, rec) % 16 == 0 &&
                  offsetof(USmemTail, bsub) % 16 == 0 && offsetof(USmemTail, bat) % 16 == 0 &&
                  offsetof(UDesc, sub) % 16 == 0 && sizeof(UDesc) % 16 == 0 && (U_STAGES * U_STAGE_BYTES) % 16 == 0 &&
                  U_LBUF % 16 == 0,
              "delta-output shared-memory alignment");
// two CTAs per SM: 228 KB of shared memory per SM, 1 KB of it reserved per CTA
static_assert(U_STAGES * U_STAGE_BYTES + 2 * U_GSTAGE * U_LBUF + sizeof(USmemTail) + 1024 <= 233472 / U_CTAS_PER_SM &&
                  U_STAGES * U_STAGE_BYTES + 2 * U_GSTAGE * U_LBUF + sizeof(USmemTail) <= 232448,
              "delta-output shared memory exceeds the per-CTA share");

// One group of one stage of the delta-output consumers for a pass of ntok <= NTOK tokens (limb
// columns of tokens ntok .. NTOK - 1 keep stale bytes; their outputs are never formed).  The group's
// 256 threads (tid) and 8 warps (warp) work on its blocks at `stage`; `tw` are the t windows both
// groups share.  Phase A: the limb matrix of scale * t for every 2/3-bit block of the batch (one rank
// per thread, each block in its own slot); 8-bit blocks are summed in fp32 by threads 128..255, one
// output row each.  One barrier of all consumer warps.  Phase B: this warp's MMAs over every
// 2/3-bit block.  `lb` is the group's limb matrix of this stage.  A group slot the stage does not
// use (active false) only takes part in the barrier.
template <int NTOK>
__device__ __forceinline__ void ud_stage(const UDesc& d, const uint8_t* stage, const float* tw, bool active,
                                         uint8_t* lb, int (&C)[2][4][4], float (&zc)[DC_V_TOKS],
                                         float (&s8)[DC_V_TOKS], int ntok, int tid, int warp, int lane,
                                         int bar) {
  const int tfl = d.tfl, nsub = active ? d.nsub : 0;
  float pe[NTOK];
#pragma unroll
  for (int q = 0; q < NTOK; ++q) pe[q] = d.pe[q];
  for (int i = 0; i < nsub; ++i) {
    const int4 sd = *reinterpret_cast<const int4*>(d.sub[i]);
    const int nr = sd.y & 0xffff;
    if ((sd.x & 15) == 8) {  // row tid - 128: sum over the block's ranks of (c - z) * s * t
      const int row = tid - 128;
      if (row >= 0) {
        const uint8_t* cr = stage + (sd.z & 0xffff) + row * nr;
        const uint8_t* meta = stage + (sd.w & 0xffff);
        const float* tr = tw + (sd.w >> 16);
        for (int k = 0; k < nr; ++k) {
          const __half2 mz = *reinterpret_cast<const __half2*>(meta + 4 * k);
          const float f = ((float)cr[k] - __high2float(mz)) * __low2float(mz);
#pragma unroll
          for (int q = 0; q < NTOK; ++q)
            if (q < ntok) s8[q] = fmaf(f, tr[q * tfl + k], s8[q]);
        }
      }
      continue;
    }
    if (tid >= nr) continue;
    const int slot = sd.z >> 16, moff = sd.w & 0xffff, ro = sd.w >> 16;
    const __half2 mz = *reinterpret_cast<const __half2*>(stage + moff + 4 * tid);
    const float sc = __low2float(mz), zs = sc * __high2float(mz);
    uint8_t* col = lb + slot + tid;
#pragma unroll
    for (int q = 0; q < NTOK; ++q) {
      if (q >= ntok) break;
      const float tq = tw[q * tfl + ro + tid];
      const uint32_t v = __float_as_uint(fmaf(sc, tq * pe[q], U_MAGIC));
      uint8_t* c = col + (6 * (q >> 1) + (q & 1)) * U_LROW;
      c[0] = (uint8_t)v;
      c[2 * U_LROW] = (uint8_t)(v >> 8);
      c[4 * U_LROW] = (uint8_t)(v >> 16);
      zc[q] = fmaf(zs, tq, zc[q]);
    }
  }
  named_bar(bar, 256);
  for (int i = 0; i < nsub; ++i) {
    const int4 sd = *reinterpret_cast<const int4*>(d.sub[i]);
    const int bits = sd.x & 15;
    if (bits == 8) continue;
    const int nq = (sd.x >> 4) & 15, ns = (sd.x >> 8) & 255, last = sd.x >> 16;
    ud_mma<(NTOK + 1) / 2>(stage + (sd.z & 0xffff), bits, nq, ns, last, sd.y >> 16, lb + (sd.z >> 16), C, warp,
                           lane);
  }
}

__global__ void __launch_bounds__(U_THREADS, U_CTAS_PER_SM) k_udelta(const __grid_constant__ DcFwd F, uint8_t* ws) {
  extern __shared__ __align__(128) uint8_t usm[];
  uint8_t* lbuf = usm + U_STAGES * U_STAGE_BYTES;  // limb matrices [stage parity][group of the stage]
  USmemTail* tail = reinterpret_cast<USmemTail*>(lbuf + 2 * U_GSTAGE * U_LBUF);
  WsPtr P = ws_ptr(F.ws, ws);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = F.ws.T;
  if (threadIdx.x == 0) {
    for (int s = 0; s < U_STAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], U_CONSUMERS);
    }
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 2 * U_GSTAGE * U_LROW; i += blockDim.x) {  // constant rows 12..15 of every matrix
    const int b = i / U_LROW, w = i % U_LROW, row = 12 + w / (U_LROW / 4);
    reinterpret_cast<uint32_t*>(lbuf + b * U_LBUF + 12 * U_LROW)[w] = (row == 12 || row == 14) ? 0x01010101u : 0u;
  }
  __syncthreads();
  if (warp == U_CONSUMERS) {
    // ---------------- producer warp
    const int nseg = P.st[DC_WS_NSEG];
    constexpr int REC_VEC = sizeof(DcURec) / 16;
    uint32_t seq = 0;
    auto acquire = [&](int& s) -> bool {
      s = seq % U_STAGES;
      if (seq >= U_STAGES && !mbar_wait(&tail->empty[s], ((seq / U_STAGES) - 1) & 1)) {
        set_status(P.st, DC_ERR_CUDA);
        return false;
      }
      
      return true;
    };
    // next chunk: index, its record (lanes 0..14) and the tmax words of its first pass (lanes 0..3)
    auto grab = [&](int& p, int& sg, int& go0, int& ngo, uint4& rv, int& tm) -> bool {
      int u = 0;
      if (lane == 0) u = atomicAdd(P.st + DC_WS_UCOUNTER, 1);
      u = __shfl_sync(FULLMASK, u, 0);
      if (nseg == 0 || !ud_chunk(F, nseg, u, p, sg, go0, ngo)) return false;
      rv = lane < REC_VEC ? ldg128(reinterpret_cast<const uint8_t*>(P.urecs + (int64_t)p * T + sg) + 16 * lane)
                          : make_uint4(0, 0, 0, 0);
      const int st0 = P.segs[3 * sg + 1], len = P.segs[3 * sg + 2];
      tm = lane < min(DC_V_TOKS, len) ? P.tmax[p * T + st0 + lane] : 0;
      return true;
    };
    int p = 0, sg = 0, go0 = 0, ngo = 0, tm = 0;
    uint4 rv = make_uint4(0, 0, 0, 0);
    bool have = grab(p, sg, go0, ngo, rv, tm);
    while (have) {
      __syncwarp();
      if (lane < REC_VEC) reinterpret_cast<uint4*>(&tail->rec)[lane] = rv;
      __syncwarp();
      const int cp = p, cgo0 = go0, cngo = ngo;
      int ctm = tm;
      int np = 0, nsg = 0, ngo0 = 0, nngo = 0, ntm = 0;
      uint4 nrv = make_uint4(0, 0, 0, 0);
      const bool nhave = grab(np, nsg, ngo0, nngo, nrv, ntm);
      const DcURec& R = tail->rec;
      int NB = 0;
      for (int b = 0; b < R.n_bands; ++b) NB += R.band[b].nblk;
      if (NB > U_MAXBLK) {
        set_status(P.st, DC_ERR_UNSUPPORTED);
      } else if (R.valid && !(F.pf && R.len >= DC_PF_MIN)) {  // long segments: k_upre
        // block table of the run, one lane per block
        for (int i = lane; i < NB; i += 32) {
          int b = 0, k = i;
          while (k >= R.band[b].nblk) k -= R.band[b++].nblk;
          const DcUBand& UB = R.band[b];
          DcBand B;
          B.bits = UB.bits, B.rank = UB.rank, B.r0 = UB.r0;
          B.u_quads = UB.quads, B.u_steps = UB.steps, B.u_last = UB.last;
          const DcUBlk K = dc_u_block(B, k);
          UBlkE& E = tail->tbl[i];
          E.off = UB.boff + k * UB.full;
          E.bytes = K.bytes;
          E.p0 = UB.bits | (K.nq << 4) | (K.ns << 8) | (K.last << 16);
          E.p1 = K.nr | (K.tile_bytes << 16);
          E.nr = K.nr;
          E.r0 = UB.r0 + K.rr0;
        }
        __syncwarp();
        const uint8_t* runs = reinterpret_cast<const uint8_t*>(R.blob) + R.u_off;
        for (int pt0 = R.st; pt0 < R.st + R.len; pt0 += DC_V_TOKS) {
          const int ntok = min(DC_V_TOKS, R.st + R.len - pt0);
          if (pt0 != R.st) ctm = lane < ntok ? P.tmax[cp * T + pt0 + lane] : 0;
          const int e = ud_exponent(R.umax, ctm);  // lane q: token q
          const float pe = ldexpf(1.f, e), ie = ldexpf(1.f, -e);
          if (lane == 0) {
            // batches of consecutive blocks that fit a stage with this pass's t windows and the
            // limb matrix; per block, its stage offsets, limb slot and t offset (the same for every
            // group of the chunk)
            int nbt = 0, i = 0;
            while (i < NB) {
              const UBlkE& Ei = tail->tbl[i];
              const int w0 = Ei.r0 & ~3;
              int cb = 0, sl = 0, tfl = 0, j = i;
              while (j < NB && j - i < U_MAXSUB) {
                const UBlkE& Ej = tail->tbl[j];
                const int tj = (int)dc_align(Ej.r0 + Ej.nr, 4) - w0;
                const int sj = (Ej.p0 & 15) == 8 ? 0 : (int)dc_align(Ej.nr, 32);
                if (j > i && (U_GSTAGE * (cb + Ej.bytes) + ntok * 4 * tj > U_STAGE_BYTES || sl + sj > U_LROW)) break;
                const int off = Ej.off - Ei.off;
                *reinterpret_cast<int4*>(tail->bsub[j]) =
                    make_int4(Ej.p0, Ej.p1, off | (sl << 16),
                              (off + Ej.bytes - (int)dc_align((int64_t)4 * Ej.nr, 16)) | ((Ej.r0 - w0) << 16));
                cb = off + Ej.bytes;
                sl += sj;
                tfl = tj;
                ++j;
              }
              tail->bat[nbt++] = make_int4(i | ((j - i) << 8) | ((Ei.r0 - w0) << 16), cb, tfl, w0);
              i = j;
            }
            tail->nbatch = nbt;
          }
          __syncwarp();
          const int nbatch = tail->nbatch;
          for (int go = cgo0; go < cgo0 + cngo; go += U_GSTAGE) {
            const int ng = min(U_GSTAGE, cgo0 + cngo - go);  // groups of this stage
            for (int j = 0; j < nbatch; ++j) {
              const int4 B = tail->bat[j];
              const int f = B.x & 0xff, nsub = (B.x >> 8) & 0xff, code_bytes = B.y, tfl = B.z, w0 = B.w;
              const bool fits = U_GSTAGE * code_bytes + ntok * 4 * tfl <= U_STAGE_BYTES;
              int s;
              if (!acquire(s)) return;
              uint8_t* stage = usm + (size_t)s * U_STAGE_BYTES;
              UDesc& d = tail->desc[s];
              if (lane < 4 * nsub) d.sub[lane >> 2][lane & 3] = tail->bsub[f + (lane >> 2)][lane & 3];
              if (lane < DC_V_TOKS) {
                d.pe[lane] = pe;
                d.ie[lane] = ie;
              }
              if (lane == 0) {
                d.kind = 1;
                d.p = cp, d.go = go, d.tok0 = pt0, d.ntok = ntok, d.ng = ng;
                d.nsub = nsub, d.code_bytes = code_bytes, d.tfl = tfl, d.t_shift = B.x >> 16;
                d.ufirst = j == 0, d.ulast = j == nbatch - 1;
                d.error = fits ? 0 : 1;
                if (fits) {
                  mbar_arrive_expect_tx(&tail->full[s], (uint32_t)(ng * code_bytes + ntok * 4 * tfl));
                } else {
                  set_status(P.st, DC_ERR_UNSUPPORTED);
                  mbar_arrive(&tail->full[s]);
                }
              }
              __syncwarp();
              if (fits) {
                if (lane < ng) {  // group go + lane's blocks
                  bulk_g2s(stage + lane * code_bytes, runs + (int64_t)(go + lane) * R.u_unit + tail->tbl[f].off,
                           (uint32_t)code_bytes, &tail->full[s]);
                } else if (lane >= U_GSTAGE && lane < U_GSTAGE + ntok) {
                  const int q = lane - U_GSTAGE;
                  const float* src = P.tws + ((int64_t)cp * T + pt0 + q) * F.ws.r_stride + w0;
                  bulk_g2s(stage + U_GSTAGE * code_bytes + q * 4 * tfl, src, (uint32_t)(4 * tfl), &tail->full[s]);
                }
              }
              __syncwarp();
              ++seq;
            }
          }
        }
      }
      p = np, sg = nsg, go0 = ngo0, ngo = nngo, rv = nrv, tm = ntm;
      have = nhave;
    }
    int s;
    if (!acquire(s)) return;
    if (lane == 0) {
      tail->desc[s].kind = 2;
      mbar_arrive(&tail->full[s]);
    }
    return;
  }
  // ---------------- consumer warps
  const int gs = warp >> 3, w8 = warp & 7;  // group slot of the stage, tile of the group
  const int tid = threadIdx.x & 255;        // thread of the group slot
  const int t = lane & 3;
  int C[2][4][4];
  float zc[DC_V_TOKS];
  float s8[DC_V_TOKS];
  uint32_t seq = 0, unit = 0;
  for (;;) {
    const int s = seq % U_STAGES;
    // every consumer warp waits for the stage itself; the vote makes the warps of a group slot
    // leave together when any of their waits ran out, so none is left at a named barrier.  The two
    // slots have their own barriers (a slot may run up to the ring's depth ahead of the other)
    const bool okw = mbar_wait(&tail->full[s], (seq / U_STAGES) & 1);
    if (!bar_and(3 + gs, 256, okw)) {
      if (!okw) set_status(P.st, DC_ERR_CUDA);
      return;
    }
    const UDesc& d = tail->desc[s];
    if (d.kind == 2) return;
    const uint8_t* stage = usm + (size_t)s * U_STAGE_BYTES;
    const int ntok = d.ntok;
    const bool active = gs < d.ng;  // this slot's group is part of the stage
    if (d.ufirst) {
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
          for (int q = 0; q < 4; ++q) C[a][b][q] = 0;
#pragma unroll
      for (int q = 0; q < DC_V_TOKS; ++q) zc[q] = s8[q] = 0.f;
    }
    // the limb matrices alternate by stage: a warp writes matrix (seq & 1) only after every warp
    // has passed the previous stage's barrier, i.e. finished its MMAs on the matrix of two stages ago
    uint8_t* lb = lbuf + ((seq & 1) * U_GSTAGE + gs) * U_LBUF;
    if (!d.error) {
      const uint8_t* blocks = stage + gs * d.code_bytes;
      const float* tw = reinterpret_cast<const float*>(stage + U_GSTAGE * d.code_bytes);
      // two code copies (one or two token pairs) keep the loop body small
      if (ntok <= 2)
        ud_stage<2>(d, blocks, tw, active, lb, C, zc, s8, ntok, tid, w8, lane, 1 + gs);
      else
        ud_stage<4>(d, blocks, tw, active, lb, C, zc, s8, ntok, tid, w8, lane, 1 + gs);
    } else {
      named_bar(1 + gs, 256);  // keep the stage's barrier count uniform
    }
    const bool ulast = d.ulast;
    int p = 0, go = 0, tok0 = 0;
    float ie[DC_V_TOKS] = {0.f, 0.f, 0.f, 0.f};
    if (ulast) {  // read before the stage (and its descriptor) is handed back
      p = d.p, go = d.go + gs, tok0 = d.tok0;
#pragma unroll
      for (int q = 0; q < DC_V_TOKS; ++q) ie[q] = d.ie[q];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&tail->empty[s]);
    ++seq;
    if (!ulast) continue;
    // ---- epilogue of the stage's (group, pass) units.  The zero-point sums are per token (the same
    // for every row of a group): each warp's share goes to shared memory, one barrier, and every
    // warp then finishes its own 16 rows.  Sums run in a fixed order (deterministic).  A slot whose
    // group the stage did not hold writes nothing.
    const int ub = unit & 1;
    {  // warp sums of the zero-point terms, reduced and scattered: lane 8 q ends with token q's sum
      const bool hi = lane & 16, b3 = lane & 8;
      float k0 = hi ? zc[2] : zc[0], k1 = hi ? zc[3] : zc[1];
      k0 += __shfl_xor_sync(FULLMASK, hi ? zc[0] : zc[2], 16);
      k1 += __shfl_xor_sync(FULLMASK, hi ? zc[1] : zc[3], 16);
      float v = b3 ? k1 : k0;
      v += __shfl_xor_sync(FULLMASK, b3 ? k0 : k1, 8);
#pragma unroll
      for (int o = 4; o; o >>= 1) v += __shfl_xor_sync(FULLMASK, v, o);
      if ((lane & 7) == 0) tail->zpart[ub][gs][lane >> 3][w8] = v;
    }
    if (tid >= 128) {  // 8-bit sums of row tid - 128
#pragma unroll
      for (int q = 0; q < DC_V_TOKS; ++q) tail->s8[gs][tid - 128][q] = s8[q];
    }
    named_bar(5 + gs, 256);
    // lane t of quad g holds columns 2t, 2t+1 of rows g and g+8 (regs 0, 1 and 2, 3).  Column 7 is
    // zero: lane 3 replaces it by column 6 (the row sum), then a 4x4 transpose inside the quad
    // leaves lane t with register t of every lane of its quad, i.e. output (row g + 8 (t >> 1),
    // token-in-pair t & 1): w[0] limb 0, w[1] limb 1, w[2] limb 2, w[3] the row sum.
    const int orow = 16 * w8 + (lane >> 2) + 8 * (t >> 1);
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      if (2 * pr >= ntok || !active) continue;
      int w[4];
#pragma unroll
      for (int r = 0; r < 4; ++r)
        w[r] = C[pr][0][r] + (C[pr][1][r] >> 2) + (C[pr][2][r] >> 4) + (C[pr][3][r] >> 6);
      if (t == 3) {
        w[1] = w[0];
        w[3] = w[2];
      }
      // transpose: round 1 swaps with lane t ^ 1 the registers whose bit 0 differs from t's,
      // round 2 with lane t ^ 2 those whose bit 1 differs
      {
        const bool o = t & 1;
        const int a = __shfl_xor_sync(FULLMASK, o ? w[0] : w[1], 1);
        const int b = __shfl_xor_sync(FULLMASK, o ? w[2] : w[3], 1);
        if (o) { w[0] = a; w[2] = b; } else { w[1] = a; w[3] = b; }
      }
      {
        const bool o = (t >> 1) & 1;
        const int a = __shfl_xor_sync(FULLMASK, o ? w[0] : w[2], 2);
        const int b = __shfl_xor_sync(FULLMASK, o ? w[1] : w[3], 2);
        if (o) { w[0] = a; w[1] = b; } else { w[2] = a; w[3] = b; }
      }
      const int q = 2 * pr + (t & 1);
      const float ieq = (t & 1) ? ie[2 * pr + 1] : ie[2 * pr];
      if (q < ntok) {
        const float4 z0 = *reinterpret_cast<const float4*>(&tail->zpart[ub][gs][q][0]);
        const float4 z1 = *reinterpret_cast<const float4*>(&tail->zpart[ub][gs][q][4]);
        const float zs = ((z0.x + z0.y) + (z0.z + z0.w)) + ((z1.x + z1.y) + (z1.z + z1.w));
        const float v = (float)(w[2] - 64 * w[3]) * 65536.f + (float)w[1] * 256.f + (float)w[0];
        const float y = fmaf(v, ieq, -zs) + tail->s8[gs][orow][q];
        P.yd[((int64_t)p * T + tok0 + q) * F.ws.max_d_in + 128 * go + orow] = y;
      }
    }
    ++unit;
  }
}

// ---------------------------------------------------------------------------------------------
// k_base: y = W_base x + ydelta, persistent CTAs of 8 consumer warps + 1 producer warp over units
// (linear, 128-row output tile, 64-token block), largest linears first.  The producer streams
// 128 x 128 tiles of W_base and 64 x 128 tiles of the tenant-sorted activations with 2-D tensor
// copies (128-byte swizzle); consumer warp w owns rows 16w..16w+15 and writes the unit's outputs,
// plus the delta of k_udelta, in the tokens' original order.
// ---------------------------------------------------------------------------------------------
#define B_STAGES 8
#define B_STAGE_BYTES (24 * 1024)  // a multiple of 1024 (128-byte-swizzled tensor tiles)
#define B_KC 64                    // backbone columns per stage: one 64-column box
#define B_WBOX 16384               // 128 rows x 64 bf16
#define B_XBOX 8192                // 64 tokens x 64 bf16

struct BDesc {
  int kind;  // 0 backbone chunk (bf16), 2 end, 3 backbone fp32 (read in place), 4 unit without backbone
  int first, last;
  int p, ot, tb, Tb;
};

struct BSmemTail {
  BDesc desc[B_STAGES];
  uint64_t full[B_STAGES];
  uint64_t empty[B_STAGES];
};

__device__ __forceinline__ void b_unit_coords(const DcFwd& F, int u, int nTB, int& p, int& ot, int& tb) {
  int slot = 0;
  while (slot + 1 < F.n_lin && u >= F.tile_prefix[slot + 1] * nTB) ++slot;
  p = F.order[slot];
  const int local = u - F.tile_prefix[slot] * nTB;
  ot = local / nTB;
  tb = (local % nTB) * DC_TOK_BLOCK;
}

// fp32 backbone (small fp32 layers): plain FFMA from global memory in the MMA fragment layout.
__device__ void b_base_f32(const DcFwd& F, const DcLinDev& lin, const int* perm, int ot, int tb, int Tb, int w,
                           int lane, float (&acc)[8][4]) {
  const int g = lane >> 2, t = lane & 3;
  const int d_in = lin.d_in;
  const float* Wm = (const float*)lin.W;
  const int r0 = ot * 128 + 16 * w + g;
  const float* w0 = Wm + (int64_t)r0 * d_in;
  const float* w1 = w0 + (int64_t)8 * d_in;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int tok = 8 * nt + 2 * t + q;
      if (tok >= Tb) continue;
      const int src = perm[tb + tok];
      float s0 = 0.f, s1 = 0.f;
      if (F.dtype_in == DC_DTYPE_F32) {
        const float* xr = (const float*)F.x[lin.input] + (int64_t)src * d_in;
        for (int k = 0; k < d_in; ++k) {
          s0 = fmaf(w0[k], xr[k], s0);
          s1 = fmaf(w1[k], xr[k], s1);
        }
      } else {
        const __nv_bfloat16* xr = (const __nv_bfloat16*)F.x[lin.input] + (int64_t)src * d_in;
        for (int k = 0; k < d_in; ++k) {
          const float xv = __bfloat162float(xr[k]);
          s0 = fmaf(w0[k], xv, s0);
          s1 = fmaf(w1[k], xv, s1);
        }
      }
      acc[nt][q] += s0;
      acc[nt][2 + q] += s1;
    }
  }
}

#define KB_CONSUMERS 8  // consumer warps of k_base (warp w: rows 16 w .. 16 w + 15 of the tile)
#define KB_THREADS (32 * (KB_CONSUMERS + 1))
__global__ void __launch_bounds__(KB_THREADS, 1) k_base(const __grid_constant__ DcFwd F, uint8_t* ws) {
  extern __shared__ __align__(1024) uint8_t bsm_raw[];
  uint8_t* sm = bsm_raw + ((1024 - (smem_u32(bsm_raw) & 1023)) & 1023);  // 1024-aligned for swizzled tiles
  BSmemTail* tail = reinterpret_cast<BSmemTail*>(sm + B_STAGES * B_STAGE_BYTES);
  WsPtr P = ws_ptr(F.ws, ws);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = F.ws.T;
  const int nTB = (T + DC_TOK_BLOCK - 1) / DC_TOK_BLOCK;
  if (threadIdx.x == 0) {
    for (int s = 0; s < B_STAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], KB_CONSUMERS);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == KB_CONSUMERS) {
    // ---------------- producer warp
    const int n_units = F.tile_prefix[F.n_lin] * nTB;
    uint32_t seq = 0;
    auto acquire = [&](int& s) -> bool {
      s = seq % B_STAGES;
      if (seq >= B_STAGES && !mbar_wait(&tail->empty[s], ((seq / B_STAGES) - 1) & 1)) {
        set_status(P.st, DC_ERR_CUDA);
        return false;
      }
      fence_proxy_async();
      return true;
    };
    for (;;) {
      int u = 0;
      if (lane == 0) u = atomicAdd(P.st + DC_WS_BCOUNTER, 1);
      u = __shfl_sync(FULLMASK, u, 0);
      if (u >= n_units) {
        int s;
        if (!acquire(s)) return;
        if (lane == 0) {
          tail->desc[s].kind = 2;
          mbar_arrive(&tail->full[s]);
        }
        return;
      }
      int p, ot, tb;
      b_unit_coords(F, u, nTB, p, ot, tb);
      const DcLinDev& lin = F.lin[p];
      const int Tb = min(DC_TOK_BLOCK, T - tb);
      const bool base = (F.flags & DC_BASE) != 0;
      const bool bf16 = lin.w_dtype == DC_DTYPE_BF16;
      const int nkc = base ? (bf16 ? lin.d_in / B_KC : 1) : 1;
      for (int kc = 0; kc < nkc; ++kc) {
        int s;
        if (!acquire(s)) return;
        uint8_t* stage = sm + (size_t)s * B_STAGE_BYTES;
        if (lane == 0) {
          BDesc& d = tail->desc[s];
          d.kind = base ? (bf16 ? 0 : 3) : 4, d.first = kc == 0, d.last = kc == nkc - 1;
          d.p = p, d.ot = ot, d.tb = tb, d.Tb = Tb;
          if (base && bf16)
            mbar_arrive_expect_tx(&tail->full[s], (uint32_t)(B_WBOX + 128 * min(64, T)));
          else
            mbar_arrive(&tail->full[s]);
          if (base && bf16) {
            tma_load_2d(stage, &F.wmap[p], kc * B_KC, ot * 128, &tail->full[s]);
            tma_load_2d(stage + B_WBOX, &F.xmap[lin.input], kc * B_KC, tb, &tail->full[s]);
          }
        }
        __syncwarp();
        ++seq;
      }
    }
  }
  // ---------------- consumer warps
  const int g = lane >> 2, t = lane & 3;
  float acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[a][q] = 0.f;
  uint32_t seq = 0;
  for (;;) {
    const int s = seq % B_STAGES;
    if (!mbar_wait(&tail->full[s], (seq / B_STAGES) & 1)) {
      set_status(P.st, DC_ERR_CUDA);
      return;
    }
    const BDesc d = tail->desc[s];
    if (d.kind == 2) return;
    const uint8_t* stage = sm + (size_t)s * B_STAGE_BYTES;
    if (d.first) {
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[a][q] = 0.f;
    }
    if (d.kind == 0) {
      // rows 16w.. of W and the block's tokens, 64 columns, stored with the 128-byte swizzle
      // (16-byte chunk c of row r at chunk c ^ (r & 7))
      const int ntv = (d.Tb + 7) >> 3;
      const int r0 = 16 * warp + g, r1 = r0 + 8;
      uint4 wa[2], wb[2];
#pragma unroll
      for (int k32 = 0; k32 < 2; ++k32) {
        const int c = 4 * k32 + t;
        wa[k32] = *reinterpret_cast<const uint4*>(stage + r0 * 128 + ((c ^ (r0 & 7)) << 4));
        wb[k32] = *reinterpret_cast<const uint4*>(stage + r1 * 128 + ((c ^ (r1 & 7)) << 4));
      }
      // each 64-column chunk is summed in a fresh MMA chain, then added with an IEEE fp32 add
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        if (nt < ntv) {
          const int xr = 8 * nt + g;
          float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int k32 = 0; k32 < 2; ++k32) {
            const int c = 4 * k32 + t;
            const uint4 xv = *reinterpret_cast<const uint4*>(stage + B_WBOX + xr * 128 + ((c ^ (xr & 7)) << 4));
            mma_bf16(part, wa[k32].x, wb[k32].x, wa[k32].y, wb[k32].y, xv.x, xv.y);
            mma_bf16(part, wa[k32].z, wb[k32].z, wa[k32].w, wb[k32].w, xv.z, xv.w);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[nt][q] += part[q];
        }
      }
    } else if (d.kind == 3) {
      b_base_f32(F, F.lin[d.p], P.perm, d.ot, d.tb, d.Tb, warp, lane, acc);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&tail->empty[s]);
    if (d.last) {
      // ---- output (+ delta) in the tokens' original order
      const DcLinDev& lin = F.lin[d.p];
      const float* yd = P.yd + (int64_t)d.p * T * F.ws.max_d_in;
      const uint8_t* hasd = P.dflag + (int64_t)d.p * T;
      const bool delta = (F.flags & DC_DELTA) != 0;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int tok = 8 * nt + 2 * t + (q & 1);
          const int row = d.ot * 128 + 16 * warp + g + 8 * (q >> 1);
          if (tok < d.Tb) {
            float v = acc[nt][q];
            if (delta && hasd[d.tb + tok]) v += yd[(int64_t)(d.tb + tok) * F.ws.max_d_in + row];
            const int64_t o = (int64_t)P.perm[d.tb + tok] * lin.d_out + row;
            if (F.dtype_out == DC_DTYPE_F32)
              reinterpret_cast<float*>(lin.y)[o] = v;
            else
              reinterpret_cast<__nv_bfloat16*>(lin.y)[o] = __float2bfloat16_rn(v);
          }
        }
    }
    ++seq;
  }
}

// ---------------------------------------------------------------------------------------------
// k_base_tc: y = W_base x (+ ydelta) on the tcgen05 tensor cores, for bf16 backbones (kind::f16)
// and E4M3 backbones (kind::f8f6f4, activations quantised per token by k_prep).
// A unit is (linear p, 128-row output tile ot, block of NB tenant-sorted tokens); its K is cut
// into chunks of 128 bytes of a row (64 bf16 or 128 E4M3 columns).  With one token block the
// units' chunks (ordered inside a linear by group of tiles, token block, tile), largest-K linears
// first, form one sequence split evenly over the persistent CTAs (stream-K), so every CTA moves
// the same number of bytes whatever the tile count; with several token blocks the CTAs form teams
// of one CTA per block that split one block's sequence (see bt_range).  Per CTA: warp 0 loads each
// chunk's W slice (128 rows) and activation slice (NB rows) with 2-D TMA into a ring of stages;
// warp 1 owns two NB-column fp32 accumulators in Tensor Memory and, from one thread, issues 4 MMAs
// (M 128, N NB, 32 bytes of K each) per chunk, releasing the stage with a commit; warps 2-9 (two
// warpgroups, one TMEM lane quarter per warp, lane = output row) drain a finished accumulator.
// A unit shared by several CTAs leaves fp32 partial tiles; the last contributor to arrive (a
// counter per unit) adds them in k order, so the result does not depend on timing.  The epilogue
// applies the E4M3 scales, adds the delta and writes y in the tokens' original order.
// ---------------------------------------------------------------------------------------------
#define BT_THREADS 320
#define BT_MAX_STAGES 8
#define BT_A_BYTES 16384  // 128 rows x 64 bf16
#define BT_MAX_SEGS 64

struct BtTail {
  uint64_t full[BT_MAX_STAGES];
  uint64_t empty[BT_MAX_STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  int abort;
  int last_flag;
  int perm[256];    // epilogue: original position of each token of the unit's block (-1: none)
  uint8_t dfl[256]; // epilogue: the token has a delta
  float sxs[256];   // epilogue, fp8 backbone: the token's activation scale
  int nseg;         // segments of this CTA's chunk range (-1: more than BT_MAX_SEGS)
  int64_t sg[BT_MAX_SEGS];  // their first chunks, in processing order
};

// The chunk bookkeeping of both schedules (stream-K, teams) is in dc_btsched.h.

__device__ __forceinline__ bool bt_aborted(BtTail* tail) { return *reinterpret_cast<volatile int*>(&tail->abort) != 0; }

__device__ __forceinline__ bool bt_wait(uint64_t* bar, uint32_t parity, BtTail* tail, int* st) {
  if (bt_aborted(tail)) return false;
  if (mbar_wait(bar, parity)) return true;
  tail->abort = 1;
  set_status(st, DC_ERR_CUDA);
  return false;
}

__global__ void __launch_bounds__(BT_THREADS, 1) k_base_tc(const __grid_constant__ DcFwd F, uint8_t* ws) {
  extern __shared__ __align__(1024) uint8_t bt_raw[];
  uint8_t* sm = bt_raw + ((1024 - (smem_u32(bt_raw) & 1023)) & 1023);  // 1024-aligned (swizzled tiles)
  const int NB = F.ws.bt_nb, NS = F.bt_ns;
  const int stage_bytes = BT_A_BYTES + NB * 128;
  BtTail* tail = reinterpret_cast<BtTail*>(sm + (size_t)NS * stage_bytes);
  WsPtr P = ws_ptr(F.ws, ws);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = F.ws.T;
  const int c = blockIdx.x;
  int64_t g0, g1;
  bt_range(F, c, g0, g1);
  uint32_t ncols = 32;
  while (ncols < (uint32_t)(2 * NB)) ncols <<= 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tail->acc_full[b], 1);
      mbar_init(&tail->acc_empty[b], 8);
    }
    tail->abort = 0;
    // Segment order: the range's last segment, then its first, then the rest.  Both ends are
    // usually units shared with the neighbouring CTAs; doing them first lets the last contributor
    // finish those units while streaming continues, instead of in the range's tail.
    int n = 0;
    for (int64_t g = g0; g < g1; ++n) {
      if (n < BT_MAX_SEGS) tail->sg[n] = g;
      const BtSeg S = bt_seg_at(F, g, g1);
      g = S.ustart + S.k1;
    }
    if (n <= BT_MAX_SEGS) {
      if (n >= 2) {
        const int64_t last = tail->sg[n - 1];
        for (int i = n - 1; i > 0; --i) tail->sg[i] = tail->sg[i - 1];
        tail->sg[0] = last;
      }
      tail->nseg = n;
    } else {
      tail->nseg = -1;  // natural order
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tail->tmem_base), ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tail->tmem_base;
  if (warp == 0) {
    // ---------------- TMA producer
    uint32_t seq = 0;
    const int nseg = tail->nseg;
    const int kc = F.fp8 ? 128 : 64;  // elements per 128-byte chunk
    int64_t g = g0;
    for (int si = 0; (nseg >= 0 ? si < nseg : g < g1) && !bt_aborted(tail); ++si) {
      const BtSeg S = bt_seg_at(F, nseg >= 0 ? tail->sg[si] : g, g1);
      const int p = F.order[S.slot];
      const int m = F.lin[p].input;
      for (int k = S.k0; k < S.k1; ++k, ++seq) {
        const int s = seq % NS;
        if (seq >= (uint32_t)NS && !bt_wait(&tail->empty[s], ((seq / NS) - 1) & 1, tail, P.st)) break;
        if (lane == 0) {
          uint8_t* st = sm + (size_t)s * stage_bytes;
          mbar_arrive_expect_tx(&tail->full[s], (uint32_t)stage_bytes);
          tma_load_2d(st, &F.wmap[p], k * kc, S.ot * 128, &tail->full[s]);
          tma_load_2d(st + BT_A_BYTES, &F.xmap[m], k * kc, S.tb * NB, &tail->full[s]);
        }
        __syncwarp();
      }
      g = S.ustart + S.k1;
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread)
    const bool fp8 = F.fp8 != 0;
    const uint32_t idesc = fp8 ? umma_idesc_e4m3(128, NB) : umma_idesc_bf16(128, NB);
    uint32_t seq = 0, segi = 0;
    const int nseg = tail->nseg;
    int64_t g = g0;
    for (int si = 0; (nseg >= 0 ? si < nseg : g < g1) && !bt_aborted(tail); ++si, ++segi) {
      const BtSeg S = bt_seg_at(F, nseg >= 0 ? tail->sg[si] : g, g1);
      const int b = segi & 1;
      if (segi >= 2 && !bt_wait(&tail->acc_empty[b], ((segi >> 1) - 1) & 1, tail, P.st)) break;
      tc_fence_after();
      const uint32_t dt = tbase + (uint32_t)(b * NB);
      bool ok = true;
      for (int k = S.k0; k < S.k1; ++k, ++seq) {
        const int s = seq % NS;
        if (!bt_wait(&tail->full[s], (seq / NS) & 1, tail, P.st)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sm + (size_t)s * stage_bytes);
          const uint64_t ad = umma_desc_sw128(a0), bd = umma_desc_sw128(a0 + BT_A_BYTES);
          // 32 bytes of each row per MMA (K = 16 bf16 or K = 32 E4M3): 2 x 16 further inside the atom
          if (fp8) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f8(dt, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, (k > S.k0 || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f16(dt, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, (k > S.k0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(&tail->empty[s]));  // the stage is free once these MMAs have read it
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) umma_commit(smem_u32(&tail->acc_full[b]));  // accumulator complete
      __syncwarp();
      g = S.ustart + S.k1;
    }
  } else {
    // ---------------- epilogue: two warpgroups (warps 2-5, 6-9), TMEM lane quarter warp % 4;
    // warpgroup wg drains the 16-column blocks 2 i + wg of the accumulator
    const int q4 = warp & 3, wg = (warp - 2) >> 2;
    const int row = 32 * q4 + lane;  // output row inside the tile
    const bool delta = (F.flags & DC_DELTA) != 0;
    float* part_base = reinterpret_cast<float*>(ws + F.ws.bt_part);
    int* cnt = reinterpret_cast<int*>(ws + F.ws.bt_cnt);
    uint32_t segi = 0;
    // The eight warps leave the loop together: the outcome of every wait is agreed through a
    // reducing named barrier, so no warp is left waiting at a barrier the others skipped.
    const int nseg = tail->nseg;
    int64_t g = g0;
    for (int si = 0; nseg >= 0 ? si < nseg : g < g1; ++si, ++segi) {
      const BtSeg S = bt_seg_at(F, nseg >= 0 ? tail->sg[si] : g, g1);
      const int b = segi & 1;
      const bool okw = bt_wait(&tail->acc_full[b], (segi >> 1) & 1, tail, P.st);
      if (!bar_and(1, 256, okw)) break;
      tc_fence_after();
      const int p = F.order[S.slot];
      const DcLinDev& lin = F.lin[p];
      const bool whole = S.k0 == 0 && S.k1 == S.K;
      const int my_slot = S.ustart <= bt_g0(F, c) ? 0 : 1;  // 0: the CTA's first unit, 1: its last
      float* mypart = part_base + ((int64_t)(2 * c + my_slot) * NB) * 128;
      const uint32_t ta = tbase + ((uint32_t)(32 * q4) << 16) + (uint32_t)(b * NB);
      const int orow = S.ot * 128 + row;
      const int et = threadIdx.x - 64;  // 0..255
      // destinations of the block's tokens, staged once per unit
      for (int col = et; col < NB; col += 256) {
        const int ts = S.tb * NB + col;
        tail->perm[col] = ts < T ? P.perm[ts] : -1;
        tail->dfl[col] = (delta && ts < T) ? P.dflag[(int64_t)p * T + ts] : 0;
        if (F.fp8) tail->sxs[col] = ts < T ? P.sx8[(int64_t)lin.input * T + ts] : 0.f;
      }
      // fp8 backbone: the accumulator holds sum code_w code_x; the output row's weight scale and
      // (per column) the token's activation scale turn it into W_hat x_hat
      const float sw = F.fp8 ? reinterpret_cast<const float*>(static_cast<const uint8_t*>(lin.W) +
                                                              (int64_t)lin.d_out * lin.d_in)[orow]
                             : 1.f;
      named_bar(1, 256);
      const float* ydp = P.yd + (int64_t)p * T * F.ws.max_d_in + orow;
      for (int cb = 16 * wg; cb < NB; cb += 32) {
        uint32_t r[16];
        tmem_ld16(ta + cb, r);
        tmem_ld_wait();
        if (whole) {
          float yv[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = cb + j;
            yv[j] = __uint_as_float(r[j]);
            if (F.fp8) yv[j] = yv[j] * sw * tail->sxs[col];
            if (tail->dfl[col]) yv[j] += ydp[(int64_t)(S.tb * NB + col) * F.ws.max_d_in];
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int dst = tail->perm[cb + j];
            if (dst >= 0) {
              const int64_t o = (int64_t)dst * lin.d_out + orow;
              if (F.dtype_out == DC_DTYPE_F32)
                reinterpret_cast<float*>(lin.y)[o] = yv[j];
              else
                reinterpret_cast<__nv_bfloat16*>(lin.y)[o] = __float2bfloat16_rn(yv[j]);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) mypart[(cb + j) * 128 + row] = __uint_as_float(r[j]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->acc_empty[b]);  // the accumulator may be overwritten
      if (!whole) {
        // hand the partial over; the last contributor of the unit finishes it
        __threadfence();
        named_bar(1, 256);
        // the unit's contributors: CTAs c0, c0 + cs, ..., c1 (cs = 1, or the team size)
        const int c0 = bt_cta_of(F, S.ustart), c1 = bt_cta_of(F, S.ustart + S.K - 1);
        const int cs = F.bt_team ? F.bt_team : 1;
        if (et == 0) {
          const int old = atomicAdd(cnt + S.u, 1);
          tail->last_flag = old == (c1 - c0) / cs;
          __threadfence();
        }
        named_bar(1, 256);
        if (tail->last_flag) {
          for (int cb = 16 * wg; cb < NB; cb += 32) {
            float yv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) yv[j] = 0.f;
            for (int cc = c0; cc <= c1; cc += cs) {  // k order
              const int sl = S.ustart <= bt_g0(F, cc) ? 0 : 1;
              const float* pp = part_base + ((int64_t)(2 * cc + sl) * NB + cb) * 128 + row;
              float pv[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) pv[j] = __ldcg(pp + j * 128);
#pragma unroll
              for (int j = 0; j < 16; ++j) yv[j] += pv[j];
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int col = cb + j;
              if (F.fp8) yv[j] = yv[j] * sw * tail->sxs[col];
              if (tail->dfl[col]) yv[j] += ydp[(int64_t)(S.tb * NB + col) * F.ws.max_d_in];
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int dst = tail->perm[cb + j];
              if (dst >= 0) {
                const int64_t o = (int64_t)dst * lin.d_out + orow;
                if (F.dtype_out == DC_DTYPE_F32)
                  reinterpret_cast<float*>(lin.y)[o] = yv[j];
                else
                  reinterpret_cast<__nv_bfloat16*>(lin.y)[o] = __float2bfloat16_rn(yv[j]);
              }
            }
          }
        }
      }
      g = S.ustart + S.k1;
    }
  }
  // every role has left its loop (all waits are bounded); release Tensor Memory
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, ncols);
  }
}

// ---------------------------------------------------------------------------------------------
// Prefill delta path (segments of at least DC_PF_MIN tokens), tcgen05 tensor cores.
//
// k_vpre computes t and writes it as one fp16 plane, t / 2^E per token (2^E > max |x| of the
// token), in the layout k_upre loads with TMA: [linear][token][tcols], band b of the tenant
// starting at column sum_{b' < b} align(rank_b', 64), zeros in the padding.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ int pf_band_col(const DcURec& R, int b) {
  int c = 0;
  for (int i = 0; i < b; ++i) c += (R.band[i].rank + 63) & ~63;
  return c;
}

// One 16-byte chunk (8 consecutive K columns) of a 128-byte-swizzled K-major 16-bit tile row.
__device__ __forceinline__ void sw128_store(uint8_t* tile, int row, int chunk, uint4 v) {
  *reinterpret_cast<uint4*>(tile + row * 128 + ((chunk ^ (row & 7)) << 4)) = v;
}

// fp16 (c - z) * s for 8 codes (4 bytes of r0, then 4 of r1); pair k covers codes 2k and 2k + 1,
// zb[k] holds 1024 + z and s[k] the scale of each.  A byte c placed under the fp16 exponent of 1024
// reads as 1024 + c, so one subtraction of 1024 + z gives c - z exactly (z is an integer code, both
// terms are integers below 2048); the product is then the one rounding, to nearest even.
__device__ __forceinline__ uint4 pf_deq16(uint32_t r0, uint32_t r1, const __half2 (&s)[4], const __half2 (&zb)[4]) {
  const uint32_t c[4] = {__byte_perm(r0, 0x64646464u, 0x5140), __byte_perm(r0, 0x64646464u, 0x7362),
                         __byte_perm(r1, 0x64646464u, 0x5140), __byte_perm(r1, 0x64646464u, 0x7362)};
  uint32_t h[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __half2 v = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&c[k]), zb[k]), s[k]);
    h[k] = *reinterpret_cast<const uint32_t*>(&v);
  }
  return make_uint4(h[0], h[1], h[2], h[3]);
}

// (1024 + z, scale) of a stored (scale, zero) pair, both halves of each result the same.
__device__ __forceinline__ void pf_meta_bcast(__half2 mz, __half2& s2, __half2& zb2) {
  s2 = __low2half2(mz);
  zb2 = __hadd2(__high2half2(mz), __float2half2_rn(1024.f));
}

// ---------------------------------------------------------------------------------------------
// k_upre: ydelta = U_hat t for segments of at least DC_PF_MIN tokens, on tcgen05.
// Unit = (linear p, long segment, 128-row output group go); the segment's tokens are taken in
// tiles of up to 256 (the MMA N).  K = the tenant's ranks, band by band, in chunks of 64.
// Both operands are fp16: U_hat as the fp16 rounding of (c - z) * scale, and t scaled per token
// by 2^-E (2^E > max |x| of the token), which the epilogue undoes.
//   warp 0     TMA: per chunk the t plane tile (256 tokens x 64 ranks); per U block the block's
//              bytes (codes of the eight 16-row tiles + meta) into a two-slot ring
//   warps 1-16 expansion, two sets of eight taking alternate chunks (one 16-row tile per warp):
//              (c - z) * scale of the chunk's 128 x 64 codes as fp16 (a 128-byte-swizzled
//              K-major tile), from the staged block
//   warp 17    TMEM owner and MMA issuer: D[row][token] += U_hat t (M 128, N tokens, K 16 per
//              instruction), two accumulators
//   warps 18-21 epilogue: TMEM lane quarter = warp % 4, writes ydelta = D * 2^E
// Units are claimed dynamically (a global counter, posted to every warp through a shared-memory
// ring); every wait is bounded.
// ---------------------------------------------------------------------------------------------
#define UP_EXP_WARPS 16
#define UP_MMA_WARP (1 + UP_EXP_WARPS)
#define UP_THREADS (32 * (UP_MMA_WARP + 5))
#define UP_A_BYTES 16384                  // 128 rows x 64 fp16
#define UP_B_BYTES 32768                  // 256 tokens x 64 fp16
#define UP_STAGE_BYTES (UP_A_BYTES + UP_B_BYTES)
#define UP_STAGES 4
#define UP_BLK_BYTES 13312                // largest U block (3-bit, 8 steps, with meta)
#define UP_MAX_LONG 256

#define UP_UQ 4                          // slots of the unit ring
#define UP_COUNTER_SLOT 7                // status word: next unit to claim (zeroed per call)
#define UP_TAKERS (UP_THREADS / 32 - 1)  // warps that read the unit ring

struct UpTail {
  uint64_t full_b[UP_STAGES], full_a[UP_STAGES], empty[UP_STAGES];
  uint64_t blk_full[2], blk_empty[2];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t uq_full[UP_UQ], uq_empty[UP_UQ];
  int uq[UP_UQ];  // units claimed by the producer, in order
  uint32_t tmem_base;
  int abort;
  int nlong;
  int lseg[UP_MAX_LONG];
  DcURec rec[UP_THREADS / 32];  // each warp's copy of its current unit's record
};

static_assert(1024 + UP_STAGES * UP_STAGE_BYTES + 2 * UP_BLK_BYTES + sizeof(UpTail) <= 232448,
              "k_upre shared memory exceeds the 227 KB a block may use");

struct UpChunk {
  int b, c0;   // band, first band-relative rank of the chunk
  int k;       // U block of the band holding it
};

// Chunk i of a record (band by band, 64 ranks each); false past the last one.
__device__ __forceinline__ bool up_chunk(const DcURec& R, int i, UpChunk& C) {
  for (int b = 0; b < R.n_bands; ++b) {
    const int n = (R.band[b].rank + 63) / 64;
    if (i < n) {
      const DcUBand& UB = R.band[b];
      C.b = b;
      C.c0 = 64 * i;
      if (UB.bits == 8 || UB.bits == 3) {
        C.k = C.c0 / (UB.bits == 8 ? 64 : 256);
      } else {
        const int qi = C.c0 / 128;
        C.k = (C.c0 < 128 * UB.quads && qi < 2 * (UB.quads / 2)) ? qi / 2 : UB.nblk - 1;
      }
      return true;
    }
    i -= n;
  }
  return false;
}

__device__ __forceinline__ DcBand up_band(const DcUBand& UB) {
  DcBand B;
  B.bits = UB.bits, B.rank = UB.rank, B.r0 = UB.r0;
  B.u_quads = UB.quads, B.u_steps = UB.steps, B.u_last = UB.last;
  return B;
}

// Unit u -> (linear p, long segment index, group go); false past the last unit.
__device__ __forceinline__ bool up_unit(const DcFwd& F, int nlong, int u, int& p, int& j, int& go) {
  for (int i = 0; i < F.n_lin; ++i) {
    const int q = F.order[i];
    const int G = F.lin[q].d_out / 128;
    const int cnt = nlong * G;
    if (u < cnt) {
      p = q;
      j = u / G;
      go = u % G;
      return true;
    }
    u -= cnt;
  }
  return false;
}

// Expand ranks [c0, c0 + 64) of band UB for the 16-row tile `tile` of the staged block `blk`
// (geometry K) into the fp16 tile `at` (rows 16 tile + g and + g + 8).  Only the band's last shift
// step can be short, and it is the last step of its block, so every step of a block before it
// starts a whole step's bytes after the previous one.
__device__ __forceinline__ void up_expand_tile(const uint8_t* blk, const DcUBand& UB, const DcUBlk& K, int c0,
                                               int tile, int lane, uint8_t* at) {
  const int g = lane >> 2, t = lane & 3;
  const uint8_t* tb = blk + tile * K.tile_bytes;
  const uint8_t* meta = blk + K.code_bytes;
  uint32_t a[2][4];
#pragma unroll
  for (int s = 0; s < 2; ++s)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) a[s][jj] = 0u;
  if (UB.bits == 2 && c0 < 128 * UB.quads) {  // both steps in one mask-layout quad
    const uint4 wq = *reinterpret_cast<const uint4*>(tb + 512 * (c0 / 128 - K.q0) + 16 * lane);
    const int ps = (c0 & 127) >> 5;  // 0 or 2
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) a[s][jj] = (wsel(wq, jj) >> (2 * (ps + s))) & 0x03030303u;
  } else if (UB.bits == 8) {
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int i = c0 + 32 * s + 8 * t + 4 * (jj >> 1) + b;
          const int row = 16 * tile + g + 8 * (jj & 1);
          const uint32_t c = i < UB.rank ? blk[row * K.nr + (i - K.rr0)] : 0u;
          a[s][jj] |= c << (8 * b);
        }
  } else {  // shift-layout steps
    const int full_step = (int)dc_u_step_bytes(UB.bits, 32);
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int rs = c0 + 32 * s;
      if (rs < UB.rank) {
        const int si = (rs - 128 * UB.quads) >> 5;  // shift-layout step of the band
        const uint8_t* sb = tb + 512 * K.nq + (si - K.s0) * full_step;
        const int valid = si == UB.steps - 1 ? UB.last : 32;
        const int nl = dc_u_step_lanes(valid), ntv = nl / 8;
        uint32_t wv = 0, hv = 0;
        if (t < ntv) {
          wv = *reinterpret_cast<const uint32_t*>(sb + 4 * (g * ntv + t));
          if (UB.bits == 3) hv = *reinterpret_cast<const uint16_t*>(sb + dc_align((int64_t)nl * 4, 16) + 2 * (g * ntv + t));
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          a[s][jj] = reg_shift2(wv, jj);
          if (UB.bits == 3) a[s][jj] |= u_reg_hi3(hv, jj);
        }
      }
    }
  }
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int r8 = c0 + 32 * s + 8 * t;  // band-relative rank of this lane's first column
    uint32_t mw[8];  // (scale, zero) of ranks r8 .. r8 + 7; zero past the band
    if (r8 + 8 <= UB.rank) {
      const uint4 m0 = *reinterpret_cast<const uint4*>(meta + 4 * (r8 - K.rr0));
      const uint4 m1 = *reinterpret_cast<const uint4*>(meta + 4 * (r8 - K.rr0) + 16);
      mw[0] = m0.x, mw[1] = m0.y, mw[2] = m0.z, mw[3] = m0.w, mw[4] = m1.x, mw[5] = m1.y, mw[6] = m1.z, mw[7] = m1.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) mw[e] = r8 + e < UB.rank ? *reinterpret_cast<const uint32_t*>(meta + 4 * (r8 + e - K.rr0)) : 0u;
    }
    __half2 s2[4], zb2[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t sp = __byte_perm(mw[2 * q], mw[2 * q + 1], 0x5410);  // the two scales
      const uint32_t zp = __byte_perm(mw[2 * q], mw[2 * q + 1], 0x7632);  // the two zeros
      s2[q] = *reinterpret_cast<const __half2*>(&sp);
      zb2[q] = __hadd2(*reinterpret_cast<const __half2*>(&zp), __float2half2_rn(1024.f));
    }
    sw128_store(at, 16 * tile + g, 4 * s + t, pf_deq16(a[s][0], a[s][2], s2, zb2));      // row g: ranks 8t .. 8t + 7
    sw128_store(at, 16 * tile + g + 8, 4 * s + t, pf_deq16(a[s][1], a[s][3], s2, zb2));  // row g + 8
  }
}

__device__ __forceinline__ bool up_aborted(UpTail* tail) { return *reinterpret_cast<volatile int*>(&tail->abort) != 0; }

__device__ __forceinline__ bool up_wait(uint64_t* bar, uint32_t parity, UpTail* tail, int* st) {
  if (up_aborted(tail)) return false;
  if (mbar_wait(bar, parity)) return true;
  tail->abort = 1;
  set_status(st, DC_ERR_CUDA);
  return false;
}

// Next (unit, token tile) of this CTA's sequence; the same for every role.
struct UpIter {
  int u, tt;    // current unit (-1 before the first) and token tile
  uint32_t kq;  // units taken from the ring so far
};
// The unit's record is copied into the calling warp's slot in shared memory (R points there).
__device__ __forceinline__ void up_load_rec(const DcURec* src, DcURec* dst) {
  constexpr int NV = sizeof(DcURec) / 16;
  const int lane = threadIdx.x & 31;
  __syncwarp();
  if (lane < NV) reinterpret_cast<uint4*>(dst)[lane] = ldg128(reinterpret_cast<const uint8_t*>(src) + 16 * lane);
  __syncwarp();
}

// Units are claimed dynamically: the producer warp takes the next unit index from a global counter
// and posts it in a ring; the other warps take the same sequence from the ring.  A failed wait
// gives an index past the last unit.
__device__ __forceinline__ int up_unit_index(const WsPtr& P, UpTail* tail, uint32_t& k) {
  const int slot = k % UP_UQ;
  int u = 1 << 30;
  if (threadIdx.x < 32) {  // producer warp: claim
    if (k >= UP_UQ && !up_wait(&tail->uq_empty[slot], ((k / UP_UQ) - 1) & 1, tail, P.st)) return u;
    if (threadIdx.x == 0) {
      u = atomicAdd(P.st + UP_COUNTER_SLOT, 1);
      tail->uq[slot] = u;
      mbar_arrive(&tail->uq_full[slot]);
    }
    u = __shfl_sync(FULLMASK, u, 0);
  } else {
    if (!up_wait(&tail->uq_full[slot], (k / UP_UQ) & 1, tail, P.st)) return u;
    u = *reinterpret_cast<volatile int*>(&tail->uq[slot]);
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&tail->uq_empty[slot]);
  }
  ++k;
  return u;
}

__device__ __forceinline__ bool up_next(const DcFwd& F, const WsPtr& P, UpTail* tail, UpIter& it, int& p,
                                        int& go, const DcURec*& R, int& tok0, int& ntok) {
  const int T = F.ws.T;
  DcURec* mine = &tail->rec[threadIdx.x >> 5];
  for (;;) {
    if (it.u >= 0) {
      R = mine;  // still the current unit's record
      if (R->valid && 256 * (it.tt + 1) < R->len) {
        ++it.tt;
        tok0 = R->st + 256 * it.tt;
        ntok = min(256, R->st + R->len - tok0);
        return true;
      }
    }
    it.u = up_unit_index(P, tail, it.kq);
    it.tt = 0;
    int j;
    if (!up_unit(F, tail->nlong, it.u, p, j, go)) return false;
    up_load_rec(P.urecs + (int64_t)p * T + tail->lseg[j], mine);
    R = mine;
    if (!R->valid) {
      it.tt = 1 << 20;  // skip: the next call moves to the next unit
      continue;
    }
    tok0 = R->st;
    ntok = min(256, R->len);
    return true;
  }
}

__global__ void __launch_bounds__(UP_THREADS, 1) k_upre(const __grid_constant__ DcFwd F, uint8_t* ws) {
  extern __shared__ __align__(1024) uint8_t up_raw[];
  uint8_t* sm = up_raw + ((1024 - (smem_u32(up_raw) & 1023)) & 1023);
  uint8_t* blkring = sm + UP_STAGES * UP_STAGE_BYTES;
  UpTail* tail = reinterpret_cast<UpTail*>(blkring + 2 * UP_BLK_BYTES);
  WsPtr P = ws_ptr(F.ws, ws);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = F.ws.T;
  if (threadIdx.x == 0) {
    for (int s = 0; s < UP_STAGES; ++s) {
      mbar_init(&tail->full_b[s], 1);
      mbar_init(&tail->full_a[s], 8);
      mbar_init(&tail->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tail->blk_full[b], 1);
      mbar_init(&tail->blk_empty[b], UP_EXP_WARPS);
      mbar_init(&tail->acc_full[b], 1);
      mbar_init(&tail->acc_empty[b], 4);
    }
    for (int q = 0; q < UP_UQ; ++q) {
      mbar_init(&tail->uq_full[q], 1);
      mbar_init(&tail->uq_empty[q], UP_TAKERS);
    }
    tail->abort = 0;
    const int nseg = P.st[DC_WS_NSEG];  // long segments, in segment order
    int n = 0;
    for (int sg = 0; sg < nseg && n < UP_MAX_LONG; ++sg)
      if (P.segs[3 * sg] >= 0 && P.segs[3 * sg + 2] >= DC_PF_MIN) tail->lseg[n++] = sg;
    tail->nlong = n;
    fence_mbar_init();
  }
  if (warp == UP_MMA_WARP) {
    tmem_alloc(smem_u32(&tail->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tail->tmem_base;
  UpIter it{-1, 0, 0u};
  int p = 0, go = 0, tok0 = 0, ntok = 0;
  const DcURec* R = nullptr;
  if (warp == 0) {
    // ---------------- TMA producer: t plane tiles per chunk, U blocks into the ring
    uint32_t seq = 0, bseq = 0;
    while (!up_aborted(tail) && up_next(F, P, tail, it, p, go, R, tok0, ntok)) {
      const uint8_t* run = reinterpret_cast<const uint8_t*>(R->blob) + R->u_off + (int64_t)go * R->u_unit;
      int lb = -1, lk = -1;
      UpChunk C;
      for (int ci = 0; up_chunk(*R, ci, C); ++ci, ++seq) {
        if (C.b != lb || C.k != lk) {  // a new U block
          lb = C.b, lk = C.k;
          const int bs = bseq & 1;
          if (bseq >= 2 && !up_wait(&tail->blk_empty[bs], ((bseq >> 1) - 1) & 1, tail, P.st)) break;
          const DcUBand& UB = R->band[C.b];
          const int bytes = dc_u_block(up_band(UB), C.k).bytes;
          if (lane == 0) {
            mbar_arrive_expect_tx(&tail->blk_full[bs], (uint32_t)bytes);
            bulk_g2s(blkring + bs * UP_BLK_BYTES, run + UB.boff + (int64_t)C.k * UB.full, (uint32_t)bytes,
                     &tail->blk_full[bs]);
          }
          __syncwarp();
          ++bseq;
        }
        const int s = seq % UP_STAGES;
        if (seq >= UP_STAGES && !up_wait(&tail->empty[s], ((seq / UP_STAGES) - 1) & 1, tail, P.st)) break;
        if (lane == 0) {
          uint8_t* st = sm + (size_t)s * UP_STAGE_BYTES + UP_A_BYTES;
          const int col = pf_band_col(*R, C.b) + C.c0;
          mbar_arrive_expect_tx(&tail->full_b[s], (uint32_t)UP_B_BYTES);
          tma_load_2d(st, &F.tmap, col, p * T + tok0, &tail->full_b[s]);
        }
        __syncwarp();
      }
    }
  } else if (warp <= UP_EXP_WARPS) {
    // ---------------- expansion warps: warp w expands the 16-row tile (w - 1) % 8 of the chunks
    // whose sequence number has the parity (w - 1) / 8; every warp takes every block
    const int e = (warp - 1) & 7, set = (warp - 1) >> 3;
    uint32_t seq = 0, bseq = 0;
    while (!up_aborted(tail) && up_next(F, P, tail, it, p, go, R, tok0, ntok)) {
      int lb = -1, lk = -1;
      UpChunk C;
      DcUBlk K;
      bool ok = true;
      for (int ci = 0; up_chunk(*R, ci, C); ++ci, ++seq) {
        if (C.b != lb || C.k != lk) {
          if (lb >= 0) {  // the previous block is done
            __syncwarp();
            if (lane == 0) mbar_arrive(&tail->blk_empty[(bseq - 1) & 1]);
          }
          lb = C.b, lk = C.k;
          K = dc_u_block(up_band(R->band[C.b]), C.k);
          if (!up_wait(&tail->blk_full[bseq & 1], (bseq >> 1) & 1, tail, P.st)) {
            ok = false;
            break;
          }
          ++bseq;
        }
        if ((int)(seq & 1) != set) continue;  // the other set expands this chunk
        const int s = seq % UP_STAGES;
        if (seq >= UP_STAGES && !up_wait(&tail->empty[s], ((seq / UP_STAGES) - 1) & 1, tail, P.st)) {
          ok = false;
          break;
        }
        const uint8_t* blk = blkring + ((bseq - 1) & 1) * UP_BLK_BYTES;
        up_expand_tile(blk, R->band[C.b], K, C.c0, e, lane, sm + (size_t)s * UP_STAGE_BYTES);
        fence_proxy_async();  // generic-proxy writes -> tensor-core (async proxy) reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&tail->full_a[s]);
      }
      if (!ok) break;
      __syncwarp();
      if (lb >= 0 && lane == 0) mbar_arrive(&tail->blk_empty[(bseq - 1) & 1]);
    }
  } else if (warp == UP_MMA_WARP) {
    // ---------------- MMA issuer
    uint32_t seq = 0, unit = 0;
    while (!up_aborted(tail) && up_next(F, P, tail, it, p, go, R, tok0, ntok)) {
      const int N = (ntok + 15) & ~15;
      const uint32_t idesc = umma_idesc_f16(128, N);
      const int b = unit & 1;
      if (unit >= 2 && !up_wait(&tail->acc_empty[b], ((unit >> 1) - 1) & 1, tail, P.st)) break;
      tc_fence_after();
      const uint32_t dt = tbase + (uint32_t)(b * 256);
      UpChunk C;
      bool ok = true;
      for (int ci = 0; up_chunk(*R, ci, C); ++ci, ++seq) {
        const int s = seq % UP_STAGES;
        const uint32_t ph = (seq / UP_STAGES) & 1;
        if (!up_wait(&tail->full_b[s], ph, tail, P.st) || !up_wait(&tail->full_a[s], ph, tail, P.st)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sm + (size_t)s * UP_STAGE_BYTES);
          const uint64_t ad = umma_desc_sw128(a0), bd = umma_desc_sw128(a0 + UP_A_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t o = (uint64_t)(2 * kk);  // 32 bytes further inside the swizzle atom
            umma_f16(dt, ad + o, bd + o, idesc, (ci > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(smem_u32(&tail->empty[s]));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) umma_commit(smem_u32(&tail->acc_full[b]));
      __syncwarp();
      ++unit;
    }
  } else {
    // ---------------- epilogue warps 10-13 (TMEM lane quarter warp % 4); exits agreed by a vote
    const int q4 = warp & 3, row = 32 * q4 + lane;
    uint32_t unit = 0;
    while (up_next(F, P, tail, it, p, go, R, tok0, ntok)) {
      const int b = unit & 1;
      const bool okw = up_wait(&tail->acc_full[b], (unit >> 1) & 1, tail, P.st);
      if (!bar_and(1, 128, okw)) break;
      tc_fence_after();
      const uint32_t ta = tbase + ((uint32_t)(32 * q4) << 16) + (uint32_t)(b * 256);
      float* yd = P.yd + ((int64_t)p * T + tok0) * F.ws.max_d_in + 128 * go + row;
      const int* xe = P.xe + F.lin[p].input * T + tok0;  // e = 22 - E per token
      for (int cb = 0; cb < ntok; cb += 16) {
        uint32_t r[16];
        tmem_ld16(ta + cb, r);
        // lane l < 16 holds 2^E of token cb + l
        const float pe = (lane < 16 && cb + lane < ntok) ? ldexpf(1.f, 22 - xe[cb + lane]) : 0.f;
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const float sc = __shfl_sync(FULLMASK, pe, jj);
          if (cb + jj < ntok) yd[(int64_t)(cb + jj) * F.ws.max_d_in] = __uint_as_float(r[jj]) * sc;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->acc_empty[b]);
      ++unit;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == UP_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// k_vpre: t = S * (V_hat^T x) for segments of at least DC_PF_MIN tokens, on tcgen05.
// Unit = (linear p, long segment, V group of the tenant: up to 8 tiles of 16 ranks of one band);
// the segment's tokens in tiles of up to 256 (the MMA N).  K = d_in in chunks of 64 columns.
// Both operands are fp16: V_hat as the fp16 rounding of (c - z) * scale, and the token's x scaled
// by 2^(14 - E) (2^E > max |x|), written by the prep kernel and exact for bf16 inputs.
//   warp 0      TMA: per chunk the activation tile (256 tenant-sorted tokens x 64); per 512-column
//               block the group's V block (codes + meta of its tiles) into a two-slot ring
//   warps 1-8   expansion: (c - z) * scale of the chunk's 128 ranks x 64 columns as fp16
//   warp 9      TMEM owner and MMA issuer: D[rank][token] += V_hat x (M 128, K 16)
//   warps 10-13 epilogue: the fp16 t plane, S * D * 2^-14 = t / 2^E, read by k_upre
// Units are claimed dynamically in their order, linears of the largest d_in first (a global
// counter, posted to every warp through a shared-memory ring); every wait is bounded.
// ---------------------------------------------------------------------------------------------
#define VP_THREADS 448
#define VP_A_BYTES 16384  // 128 ranks x 64 fp16
#define VP_B_BYTES 32768  // 256 tokens x 64 fp16
#define VP_STAGE_BYTES (VP_A_BYTES + VP_B_BYTES)
#define VP_STAGES 3
#define VP_BLK_BYTES 18432  // largest V group block (2-bit: 8 tiles x 2304 bytes)
#define VP_MAX_PJ 512
#define VP_UQ 4                                // slots of the unit ring
#define VP_COUNTER_SLOT 6                      // status word: next unit to claim (zeroed per call)
#define VP_TAKERS (VP_THREADS / 32 - 1)        // warps that read the unit ring

struct VpTail {
  uint64_t full_b[VP_STAGES], full_a[VP_STAGES], empty[VP_STAGES];
  uint64_t blk_full[2], blk_empty[2];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t uq_full[VP_UQ], uq_empty[VP_UQ];
  int uq[VP_UQ];  // units claimed by the producer, in order
  uint32_t tmem_base;
  int abort;
  int nlong, npj, box;
  int lseg[UP_MAX_LONG];
  int pref[VP_MAX_PJ + 1];  // units (V groups) before each (linear slot, long segment) pair
};

static_assert(1024 + VP_STAGES * VP_STAGE_BYTES + 2 * VP_BLK_BYTES + sizeof(VpTail) <= 232448,
              "k_vpre shared memory exceeds the 227 KB a block may use");

// Codes of lane `ln` of half h of one (tile, block) region A, group grp: c[s][hh] holds the codes of
// columns 32 t + 8 s + 4 hh + b (byte b), t = ln % 4.  The same extraction as the decode V kernel.
__device__ __forceinline__ void vp_lane_codes(const uint8_t* A, int bits, int rows, int ngrp, int h, int ln, int grp,
                                              uint32_t (&c)[4][2]) {
  const int nh = h == 0 ? min(rows, 8) : rows - 8;
#pragma unroll
  for (int s = 0; s < 4; ++s) c[s][0] = c[s][1] = 0u;
  if ((ln >> 2) >= nh) return;
  const uint8_t* hb = A + dc_v_half_off(bits, rows, ngrp, h);
  const int p0 = dc_v_plane0_bytes(bits, ngrp);
  if (bits == 2 && ngrp == 4) {
    const uint4 w0 = *reinterpret_cast<const uint4*>(hb + dc_v_mask_off(4 * nh, ln, 0));
    const uint4 w1 = *reinterpret_cast<const uint4*>(hb + dc_v_mask_off(4 * nh, ln, 1));
    const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) c[s][hh] = (w[2 * s + hh] >> (2 * grp)) & 0x03030303u;
  } else if (bits == 8) {
    const uint4 q0 = *reinterpret_cast<const uint4*>(hb + ln * p0 + 32 * grp);
    const uint4 q1 = *reinterpret_cast<const uint4*>(hb + ln * p0 + 32 * grp + 16);
    const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) c[s][hh] = w[2 * s + hh];
  } else {
    const uint2 w2 = *reinterpret_cast<const uint2*>(hb + ln * p0 + 8 * grp);
    uint32_t w1 = 0;
    if (bits == 3) w1 = *reinterpret_cast<const uint32_t*>(hb + 4 * nh * p0 + ln * (4 * ngrp) + 4 * grp);
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r = reg_shift2((s >> 1) ? w2.y : w2.x, 2 * (s & 1) + hh);
        if (bits == 3) r |= v_reg_hi3(w1, s, hh);
        c[s][hh] = r;
      }
  }
}

__device__ __forceinline__ bool vp_aborted(VpTail* tail) { return *reinterpret_cast<volatile int*>(&tail->abort) != 0; }
__device__ __forceinline__ bool vp_wait(uint64_t* bar, uint32_t parity, VpTail* tail, int* st) {
  if (vp_aborted(tail)) return false;
  if (mbar_wait(bar, parity)) return true;
  tail->abort = 1;
  set_status(st, DC_ERR_CUDA);
  return false;
}

// Units are claimed dynamically, largest first (linears by d_in, longest first): the producer warp
// takes the next unit index from a global counter and posts it in a ring; the other warps take
// the same sequence from the ring.  A failed wait returns an index past the last unit.
__device__ __forceinline__ int vp_claim(VpTail* tail, const WsPtr& P, uint32_t& k) {
  const int slot = k % VP_UQ;
  if (k >= VP_UQ && !vp_wait(&tail->uq_empty[slot], ((k / VP_UQ) - 1) & 1, tail, P.st)) return 1 << 30;
  int u = 0;
  if ((threadIdx.x & 31) == 0) {
    u = atomicAdd(P.st + VP_COUNTER_SLOT, 1);
    tail->uq[slot] = u;
    mbar_arrive(&tail->uq_full[slot]);
  }
  ++k;
  return __shfl_sync(FULLMASK, u, 0);
}
__device__ __forceinline__ int vp_take(VpTail* tail, const WsPtr& P, uint32_t& k) {
  const int slot = k % VP_UQ;
  if (!vp_wait(&tail->uq_full[slot], (k / VP_UQ) & 1, tail, P.st)) return 1 << 30;
  const int u = *reinterpret_cast<volatile int*>(&tail->uq[slot]);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&tail->uq_empty[slot]);
  ++k;
  return u;
}

// A V group: band b, group index inside the band, its tiles and first rank.
struct VpGroup {
  int b, grp, t0, ntiles, rows_left, r0;  // first tile, tiles, ranks from the first tile on, first rank
};

struct VpUnit {  // compact: kept in registers by every role
  int p, j;            // linear, long segment index
  int64_t base, s_off; // blob address, offset of S
  DcBand B;            // the group's band
  int nkb, tail_groups, bandcol, st, len;
  VpGroup G;
};

// Unit u of this batch -> its linear, segment and V group (false past the last unit).
__device__ __forceinline__ bool vp_unit(const DcFwd& F, const WsPtr& P, const VpTail* tail, int u, VpUnit& U) {
  if (u >= tail->pref[tail->npj]) return false;
  int pj = 0;
  while (tail->pref[pj + 1] <= u) ++pj;
  const int slot = pj / tail->nlong;
  U.j = pj % tail->nlong;
  U.p = F.order[slot];
  const DcURec& R = P.urecs[(int64_t)U.p * F.ws.T + tail->lseg[U.j]];
  U.st = R.st;
  U.len = R.len;
  const dc_delta_handle* h = F.lin[U.p].tenants + R.tenant;
  const DcLayout L = dc_layout(h->desc);
  U.base = (int64_t)h->dev_base;
  U.s_off = L.s_off;
  U.nkb = L.nkb;
  U.tail_groups = L.tail_groups;
  int gi = u - tail->pref[pj];
  U.bandcol = 0;
  for (int b = 0; b < L.n_bands; ++b) {
    const DcBand& B = L.band[b];
    const int ng = (B.v_tiles + B.v_group - 1) / B.v_group;
    if (gi < ng) {
      U.B = B;
      U.G.b = b;
      U.G.grp = gi;
      U.G.t0 = gi * B.v_group;
      U.G.ntiles = dc_v_group_ntiles(B, gi);
      U.G.rows_left = B.rank - 16 * U.G.t0;
      U.G.r0 = B.r0 + 16 * U.G.t0;
      return true;
    }
    gi -= ng;
    U.bandcol += (B.rank + 63) & ~63;
  }
  return false;
}

__global__ void __launch_bounds__(VP_THREADS, 1) k_vpre(const __grid_constant__ DcFwd F, uint8_t* ws) {
  extern __shared__ __align__(1024) uint8_t vp_raw[];
  uint8_t* sm = vp_raw + ((1024 - (smem_u32(vp_raw) & 1023)) & 1023);
  uint8_t* blkring = sm + VP_STAGES * VP_STAGE_BYTES;
  VpTail* tail = reinterpret_cast<VpTail*>(blkring + 2 * VP_BLK_BYTES);
  WsPtr P = ws_ptr(F.ws, ws);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = F.ws.T;
  if (threadIdx.x == 0) {
    for (int s = 0; s < VP_STAGES; ++s) {
      mbar_init(&tail->full_b[s], 1);
      mbar_init(&tail->full_a[s], 8);
      mbar_init(&tail->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tail->blk_full[b], 1);
      mbar_init(&tail->blk_empty[b], 8);
      mbar_init(&tail->acc_full[b], 1);
      mbar_init(&tail->acc_empty[b], 4);
    }
    for (int q = 0; q < VP_UQ; ++q) {
      mbar_init(&tail->uq_full[q], 1);
      mbar_init(&tail->uq_empty[q], VP_TAKERS);
    }
    tail->abort = 0;
    const int nseg = P.st[DC_WS_NSEG];
    int n = 0;
    for (int sg = 0; sg < nseg && n < UP_MAX_LONG; ++sg)
      if (P.segs[3 * sg] >= 0 && P.segs[3 * sg + 2] >= DC_PF_MIN) tail->lseg[n++] = sg;
    tail->nlong = n;
    tail->npj = min(VP_MAX_PJ, F.n_lin * n);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {  // V groups per (linear slot, long segment): the unit prefix table
    for (int pj = lane; pj < tail->npj; pj += 32) {
      const int p = F.order[pj / tail->nlong];
      const DcURec& R = P.urecs[(int64_t)p * T + tail->lseg[pj % tail->nlong]];
      int cnt = 0;
      if (R.valid) {
        const DcLayout L = dc_layout(F.lin[p].tenants[R.tenant].desc);
        for (int b = 0; b < L.n_bands; ++b) cnt += (L.band[b].v_tiles + L.band[b].v_group - 1) / L.band[b].v_group;
      }
      tail->pref[pj + 1] = cnt;
    }
    __syncwarp();
    if (lane == 0) {
      tail->pref[0] = 0;
      for (int pj = 0; pj < tail->npj; ++pj) tail->pref[pj + 1] += tail->pref[pj];
    }
  } else if (warp == 9) {
    tmem_alloc(smem_u32(&tail->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tail->tmem_base;
  const int box = F.pf_box;
  VpUnit U;
  if (warp == 0) {
    // ---------------- TMA producer
    uint32_t seq = 0, bseq = 0, kq = 0;
    for (int u = vp_claim(tail, P, kq); !vp_aborted(tail) && vp_unit(F, P, tail, u, U); u = vp_claim(tail, P, kq)) {
      const DcBand& B = U.B;
      const int m = F.lin[U.p].input;
      for (int tok0 = U.st; tok0 < U.st + U.len && !vp_aborted(tail); tok0 += 256) {
        for (int kb = 0; kb < U.nkb; ++kb) {
          const int ngrp = kb == U.nkb - 1 ? U.tail_groups : 4;
          const int bs = bseq & 1;
          if (bseq >= 2 && !vp_wait(&tail->blk_empty[bs], ((bseq >> 1) - 1) & 1, tail, P.st)) break;
          const int bytes = (int)dc_v_group_block_bytes(B, U.G.grp, ngrp);
          if (lane == 0) {
            const uint8_t* src = reinterpret_cast<const uint8_t*>(U.base) + B.v_off +
                                 (int64_t)U.G.grp * B.v_group * B.v_tile_bytes +
                                 (int64_t)kb * dc_v_group_block_bytes(B, U.G.grp, 4);
            mbar_arrive_expect_tx(&tail->blk_full[bs], (uint32_t)bytes);
            bulk_g2s(blkring + bs * VP_BLK_BYTES, src, (uint32_t)bytes, &tail->blk_full[bs]);
          }
          __syncwarp();
          ++bseq;
          for (int ch = 0; ch < 2 * ngrp; ++ch, ++seq) {
            const int s = seq % VP_STAGES;
            if (seq >= VP_STAGES && !vp_wait(&tail->empty[s], ((seq / VP_STAGES) - 1) & 1, tail, P.st)) break;
            if (lane == 0) {
              uint8_t* st = sm + (size_t)s * VP_STAGE_BYTES + VP_A_BYTES;
              mbar_arrive_expect_tx(&tail->full_b[s], (uint32_t)(box * 128));
              tma_load_2d(st, &F.xpf[m], 512 * kb + 64 * ch, tok0, &tail->full_b[s]);
            }
            __syncwarp();
          }
        }
      }
    }
  } else if (warp <= 8) {
    // ---------------- expansion warps: thread e -> rank row e % 128, column half e / 128 of a chunk
    const int e = threadIdx.x - 32;
    const int row = e & 127, part = e >> 7;
    const int tile = row >> 4, h = (row >> 3) & 1, g = row & 7;
    uint32_t seq = 0, bseq = 0, kq = 0;
    for (int u = vp_take(tail, P, kq); !vp_aborted(tail) && vp_unit(F, P, tail, u, U); u = vp_take(tail, P, kq)) {
      const DcBand& B = U.B;
      const int rows_t = tile < U.G.ntiles ? min(16, U.G.rows_left - 16 * tile) : 0;
      bool ok = true;
      for (int tok0 = U.st; ok && tok0 < U.st + U.len; tok0 += 256) {
        for (int kb = 0; ok && kb < U.nkb; ++kb) {
          const int ngrp = kb == U.nkb - 1 ? U.tail_groups : 4;
          const int bs = bseq & 1;
          if (!vp_wait(&tail->blk_full[bs], (bseq >> 1) & 1, tail, P.st)) {
            ok = false;
            break;
          }
          ++bseq;
          const uint8_t* A = blkring + bs * VP_BLK_BYTES + tile * dc_v_block_bytes(B.bits, 16, ngrp);
          for (int ch = 0; ch < 2 * ngrp; ++ch, ++seq) {
            const int s = seq % VP_STAGES;
            if (seq >= VP_STAGES && !vp_wait(&tail->empty[s], ((seq / VP_STAGES) - 1) & 1, tail, P.st)) {
              ok = false;
              break;
            }
            const int grp = ch >> 1, hc = ch & 1;
            uint32_t c[4][2];
            __half2 mz = __float2half2_rn(0.f);  // (scale, zero) of this row's group; zero: no row
            if (rows_t > 0) {
              vp_lane_codes(A, B.bits, rows_t, ngrp, h, 4 * g + 2 * hc + part, grp, c);
              if (8 * h + g < rows_t)
                mz = *reinterpret_cast<const __half2*>(A + dc_v_block_code_bytes(B.bits, rows_t, ngrp) +
                                                       4 * (grp * 16 + g * 2 + h));
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k) c[k][0] = c[k][1] = 0u;
            }
            __half2 s2[4], zb2[4];
            pf_meta_bcast(mz, s2[0], zb2[0]);
#pragma unroll
            for (int k = 1; k < 4; ++k) s2[k] = s2[0], zb2[k] = zb2[0];
            uint8_t* at = sm + (size_t)s * VP_STAGE_BYTES;
#pragma unroll
            for (int sidx = 0; sidx < 4; ++sidx) sw128_store(at, row, 4 * part + sidx, pf_deq16(c[sidx][0], c[sidx][1], s2, zb2));
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tail->full_a[s]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&tail->blk_empty[bs]);
        }
      }
      if (!ok) break;
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer
    uint32_t seq = 0, unit = 0, kq = 0;
    for (int u = vp_take(tail, P, kq); !vp_aborted(tail) && vp_unit(F, P, tail, u, U); u = vp_take(tail, P, kq)) {
      bool ok = true;
      for (int tok0 = U.st; ok && tok0 < U.st + U.len; tok0 += 256, ++unit) {
        const int ntok = min(256, U.st + U.len - tok0);
        const uint32_t idesc = umma_idesc_f16(128, (ntok + 15) & ~15);
        const int b = unit & 1;
        if (unit >= 2 && !vp_wait(&tail->acc_empty[b], ((unit >> 1) - 1) & 1, tail, P.st)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dt = tbase + (uint32_t)(b * 256);
        int ci = 0;
        for (int kb = 0; ok && kb < U.nkb; ++kb) {
          const int ngrp = kb == U.nkb - 1 ? U.tail_groups : 4;
          for (int ch = 0; ch < 2 * ngrp; ++ch, ++seq, ++ci) {
            const int s = seq % VP_STAGES;
            const uint32_t ph = (seq / VP_STAGES) & 1;
            if (!vp_wait(&tail->full_b[s], ph, tail, P.st) || !vp_wait(&tail->full_a[s], ph, tail, P.st)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (lane == 0) {
              const uint32_t a0 = smem_u32(sm + (size_t)s * VP_STAGE_BYTES);
              const uint64_t ad = umma_desc_sw128(a0), bx = umma_desc_sw128(a0 + VP_A_BYTES);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t o = (uint64_t)(2 * kk);
                umma_f16(dt, ad + o, bx + o, idesc, (ci > 0 || kk > 0) ? 1u : 0u);
              }
              umma_commit(smem_u32(&tail->empty[s]));
            }
            __syncwarp();
          }
        }
        if (!ok) break;
        if (lane == 0) umma_commit(smem_u32(&tail->acc_full[b]));
        __syncwarp();
      }
      if (!ok) break;
    }
  } else {
    // ---------------- epilogue warps 10-13 (TMEM lane quarter warp % 4); exits agreed by a vote
    const int q4 = warp & 3, row = 32 * q4 + lane;
    uint32_t unit = 0, kq = 0;
    bool go_on = true;
    for (int u = vp_take(tail, P, kq); go_on && vp_unit(F, P, tail, u, U); u = vp_take(tail, P, kq)) {
      const DcBand& B = U.B;
      const int nvalid = min(16 * U.G.ntiles, U.G.rows_left);
      const int rank = U.G.r0 + row;
      // S * 2^-14: D carries x * 2^(14 - E), so S * D * 2^-14 = t / 2^E (scaling by 2^-14 is exact)
      const float Sv = row < nvalid ? reinterpret_cast<const float*>(U.base + U.s_off)[rank] * 0x1p-14f : 0.f;
      const int col = U.bandcol + (rank - B.r0);
      const bool padrow = row >= nvalid && rank - B.r0 >= B.rank && rank - B.r0 < ((B.rank + 63) & ~63);
      for (int tok0 = U.st; tok0 < U.st + U.len; tok0 += 256, ++unit) {
        const int ntok = min(256, U.st + U.len - tok0);
        const int b = unit & 1;
        const bool okw = vp_wait(&tail->acc_full[b], (unit >> 1) & 1, tail, P.st);
        if (!bar_and(1, 128, okw)) {
          go_on = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tbase + ((uint32_t)(32 * q4) << 16) + (uint32_t)(b * 256);
        const int64_t trow0 = (int64_t)U.p * T + tok0;
        for (int cb = 0; cb < ntok; cb += 16) {
          uint32_t r[16];
          tmem_ld16(ta + cb, r);
          tmem_ld_wait();
          if (row < nvalid) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              if (cb + jj < ntok) P.t16[(trow0 + cb + jj) * F.ws.tcols + col] = __float2half_rn(Sv * __uint_as_float(r[jj]));
          } else if (padrow) {  // zero the band's padding columns of the t plane (read by k_upre)
            for (int jj = 0; jj < 16; ++jj)
              if (cb + jj < ntok) P.t16[(trow0 + cb + jj) * F.ws.tcols + col] = __float2half_rn(0.f);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tail->acc_empty[b]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// Debug unpacker: the integer codes back out of the packed layout with the extraction helpers
// the serving kernels use.  One thread per (V: tile, block, half, lane) or (U: o-tile16, lane).
// ---------------------------------------------------------------------------------------------
__global__ void k_unpack_v(const uint8_t* blob, DcLayout L, int bi, uint8_t* out) {
  const DcBand& B = L.band[bi];
  const int64_t n = (int64_t)B.v_tiles * L.nkb * 2 * 32;
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= n) return;
  const int lane = (int)(id & 31), h = (int)((id >> 5) & 1);
  const int kb = (int)((id >> 6) % L.nkb), tile = (int)((id >> 6) / L.nkb);
  const int g = lane >> 2, t = lane & 3;
  const int rows = min(16, B.rank - 16 * tile);
  const int nh = h == 0 ? min(rows, 8) : max(0, rows - 8);
  if (g >= nh) return;
  const int ngrp = (kb == L.nkb - 1) ? L.tail_groups : 4;
  const uint8_t* blk = blob + B.v_off + dc_v_group_block_off(B, L, tile / B.v_group, kb) +
                       (int64_t)(tile % B.v_group) * dc_v_block_bytes(B.bits, 16, ngrp) + dc_v_half_off(B.bits, rows, ngrp, h);
  const int p0 = dc_v_plane0_bytes(B.bits, ngrp);
  const int rank = B.r0 + 16 * tile + 8 * h + g;
  for (int grp = 0; grp < ngrp; ++grp)
    for (int s = 0; s < 4; ++s)
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r;
        if (B.bits == 2 && ngrp == 4) {
          const uint4 q = ldg128(blk + dc_v_mask_off(4 * nh, lane, s >> 1));
          r = v_reg_mask2(wsel(q, 2 * (s & 1) + hh), grp) >> (2 * grp);
        } else if (B.bits == 8) {
          r = ldg32(blk + lane * p0 + 32 * grp + 4 * (2 * s + hh));
        } else {
          const uint2 w2 = ldg64(blk + lane * p0 + 8 * grp);
          r = reg_shift2((s >> 1) ? w2.y : w2.x, 2 * (s & 1) + hh);
          if (B.bits == 3) r |= v_reg_hi3(ldg32(blk + (int64_t)4 * nh * p0 + lane * (4 * ngrp) + 4 * grp), s, hh);
        }
        for (int b = 0; b < 4; ++b)
          out[(int64_t)rank * L.d_in + 512 * kb + 128 * grp + 32 * t + 8 * s + 4 * hh + b] = (uint8_t)(r >> (8 * b));
      }
}

__global__ void k_unpack_u(const uint8_t* blob, DcLayout L, int bi, uint8_t* out) {
  const DcBand& B = L.band[bi];
  const int64_t id = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= (int64_t)B.rank * L.d_out) return;
  const int i = (int)(id / L.d_out), o = (int)(id % L.d_out);  // rank inside the band, output row
  const uint8_t* band = blob + L.u_off + (int64_t)(o >> 7) * L.u_unit + B.u_boff;
  uint32_t code;
  if (B.bits == 8) {
    const int k = i / 64;
    const DcUBlk K = dc_u_block(B, k);
    code = band[(int64_t)k * B.u_full + (o & 127) * K.nr + (i - K.rr0)];
  } else {
    const int Q = B.u_quads;
    const bool in_quad = i < 128 * Q;
    const int k = B.bits == 3 ? i / 256 : (in_quad && (i / 128) / 2 < Q / 2 ? (i / 128) / 2 : B.u_nblk - 1);
    const DcUBlk K = dc_u_block(B, k);
    const int r16 = o & 15, g = r16 & 7, jrow = r16 >> 3;
    const uint8_t* tile = band + (int64_t)k * B.u_full + ((o & 127) >> 4) * K.tile_bytes;
    if (in_quad) {
      const int q = i / 128, pp = (i % 128) / 32, w32 = i % 32;
      const int t = w32 / 8, jhi = (w32 % 8) / 4, b = w32 % 4;
      const int j = jrow + 2 * jhi, ln = 4 * g + t;
      const uint32_t w = ldg32(tile + 512 * (q - K.q0) + 16 * ln + 4 * j);
      code = (w >> (8 * b + 2 * pp)) & 3u;
    } else {
      const int sidx = (i - 128 * Q) / 32, w32 = (i - 128 * Q) % 32;
      const uint8_t* sb = tile + 512 * K.nq;
      for (int s2 = K.s0; s2 < sidx; ++s2)
        sb += dc_u_step_bytes(B.bits, dc_u_step_lanes(s2 == B.u_steps - 1 ? B.u_last : 32));
      const int valid = sidx == B.u_steps - 1 ? B.u_last : 32;
      const int nl = dc_u_step_lanes(valid), ntv = nl / 8;
      const int t = w32 / 8, jhi = (w32 % 8) / 4, b = w32 % 4;
      const int j = jrow + 2 * jhi, idx = g * ntv + t;
      code = (ldg32(sb + 4 * idx) >> (8 * b + 2 * j)) & 3u;
      if (B.bits == 3) code |= ((ldg16(sb + dc_align((int64_t)nl * 4, 16) + 2 * idx) >> (4 * j + b)) & 1u) << 2;
    }
  }
  out[(int64_t)(B.r0 + i) * L.d_out + o] = (uint8_t)code;
}

// ---------------------------------------------------------------------------------------------
// Device quantiser (same rule as the host one, fp64 arithmetic) and packer.
// One warp per (vector, group of 128): V rows first, then U columns.
// ---------------------------------------------------------------------------------------------
__global__ void k_quant_plain(DcLayout L, const float* __restrict__ U, const float* __restrict__ Vt, uint8_t* cu,
                              uint8_t* cv, uint16_t* szu, uint16_t* szv, int* status) {
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t nv = (int64_t)L.r * L.groups_in, nu = (int64_t)L.r * L.groups_out;
  if (wid >= nv + nu) return;
  const bool isv = wid < nv;
  const int64_t k = isv ? wid : wid - nv;
  const int G = isv ? L.groups_in : L.groups_out;
  const int rank = (int)(k / G), gi = (int)(k % G);
  const int d = isv ? L.d_in : L.d_out;
  const float* src = (isv ? Vt : U) + (int64_t)rank * d + gi * 128 + 4 * lane;
  int bits = 2;
  for (int b = 0; b < L.n_bands; ++b)
    if (rank >= L.band[b].r0 && rank < L.band[b].r0 + L.band[b].rank) bits = L.band[b].bits;
  const float4 q = *reinterpret_cast<const float4*>(src);
  const double v[4] = {q.x, q.y, q.z, q.w};
  double lo = 0.0, hi = 0.0;
  bool finite = true;
  for (int i = 0; i < 4; ++i) {
    finite = finite && isfinite(v[i]);
    lo = fmin(lo, v[i]);
    hi = fmax(hi, v[i]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(FULLMASK, lo, o));
    hi = fmax(hi, __shfl_xor_sync(FULLMASK, hi, o));
  }
  finite = __all_sync(FULLMASK, finite);
  const double qmax = (double)((1 << bits) - 1);
  const __half sh = __double2half((hi - lo) / qmax);
  double sc = (double)__half2float(sh);
  unsigned short shb = __half_as_ushort(sh);
  bool ok = finite && isfinite(sc);
  if (ok && sc == 0.0) {
    sc = 1.0;
    shb = 0x3C00;
  }
  double z = ok ? rint(-lo / sc) : 0.0;
  z = fmin(fmax(z, 0.0), qmax);
  uint32_t packed = 0;
  for (int i = 0; i < 4; ++i) {
    double c = ok ? rint(v[i] / sc) + z : 0.0;
    c = fmin(fmax(c, 0.0), qmax);
    packed |= (uint32_t)c << (8 * i);
  }
  uint8_t* dst = (isv ? cv : cu) + (int64_t)rank * d + gi * 128 + 4 * lane;
  *reinterpret_cast<uint32_t*>(dst) = packed;
  if (lane == 0) {
    uint16_t* sz = (isv ? szv : szu) + ((int64_t)rank * G + gi) * 2;
    sz[0] = ok ? shb : (unsigned short)0;
    sz[1] = __half_as_ushort(__double2half(z));
    if (!ok) atomicCAS(status, 0, DC_ERR_INVALID_ARG);
  }
}

__global__ void k_pack_words(DcLayout L, DcPlain Pl, uint32_t* dst) {
  const int64_t nw = L.bytes / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nw; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = dc_pack_word(L, i * 4, Pl);
}

// Largest U scale over the 2/3-bit bands and every output group -> the blob's bound word.
__global__ void k_umax(DcLayout L, const uint16_t* __restrict__ szu, float* dst) {
  __shared__ float red[32];
  float m = 0.f;
  for (int b = 0; b < L.n_bands; ++b) {
    const DcBand& B = L.band[b];
    if (B.bits == 8) continue;
    const int64_t a = (int64_t)B.r0 * L.groups_out, e = (int64_t)(B.r0 + B.rank) * L.groups_out;
    for (int64_t i = a + threadIdx.x; i < e; i += blockDim.x)
      m = fmaxf(m, fabsf(__half2float(__ushort_as_half(szu[2 * i]))));
  }
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULLMASK, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
    *dst = m;
  }
}

// ---------------------------------------------------------------------------------------------
// Host entry points
// ---------------------------------------------------------------------------------------------
static inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// ---- per-kernel timing hook (dc_profile_begin / dc_profile_end)
struct ProfState {
  cudaEvent_t* ev = nullptr;
  int32_t* kind = nullptr;
  int32_t cap = 0, n = 0;
};
static thread_local ProfState g_prof;

static void prof_before(cudaStream_t s, int kind) {
  if (!g_prof.ev || g_prof.n >= g_prof.cap) return;
  cudaEventRecord(g_prof.ev[2 * g_prof.n], s);
  g_prof.kind[g_prof.n] = kind;
}
static void prof_after(cudaStream_t s) {
  if (!g_prof.ev || g_prof.n >= g_prof.cap) return;
  cudaEventRecord(g_prof.ev[2 * g_prof.n + 1], s);
  g_prof.n++;
}

extern "C" dc_status dc_profile_begin(int32_t capacity) {
  DC_NVTX("dc_profile_begin");
  dc_clear_error();
  if (g_prof.ev) return dc_fail(DC_ERR_INVALID_ARG, "profiling already active");
  if (capacity <= 0) return dc_fail(DC_ERR_INVALID_ARG, "capacity must be positive");
  g_prof.ev = new cudaEvent_t[2 * (size_t)capacity];
  g_prof.kind = new int32_t[capacity];
  g_prof.cap = capacity;
  g_prof.n = 0;
  for (int i = 0; i < 2 * capacity; ++i) {
    dc_status st = dc_cuda_check(cudaEventCreate(&g_prof.ev[i]), "event create");
    if (st) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(g_prof.ev[j]);
      delete[] g_prof.ev;
      delete[] g_prof.kind;
      g_prof = ProfState();
      return st;
    }
  }
  return DC_OK;
}

extern "C" int32_t dc_profile_end(float* ms_out, int32_t* kind_out, int32_t capacity) {
  DC_NVTX("dc_profile_end");
  dc_clear_error();
  if (!g_prof.ev) return -1;
  int32_t n = g_prof.n;
  int32_t rc = n;
  for (int i = 0; i < n; ++i) {
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess) {
      rc = -1;
      break;
    }
    float ms = 0.f;
    cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]);
    if (i < capacity) {
      if (ms_out) ms_out[i] = ms;
      if (kind_out) kind_out[i] = g_prof.kind[i];
    }
  }
  for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
  delete[] g_prof.ev;
  delete[] g_prof.kind;
  g_prof = ProfState();
  return rc;
}

// E4M3 rows: one block per row, 256 threads; the rounding is k_prep's (IEEE quotient, one conversion).
__global__ void __launch_bounds__(256) k_quant_fp8_rows(const void* __restrict__ W, int bf16, int cols,
                                                        uint8_t* __restrict__ codes, float* __restrict__ scales) {
  const int64_t r = blockIdx.x;
  const int tid = threadIdx.x;
  auto load2 = [&](int k, float& a, float& b) {
    if (bf16) {
      const uint32_t q = *reinterpret_cast<const uint32_t*>((const __nv_bfloat16*)W + r * cols + k);
      a = __uint_as_float(q << 16), b = __uint_as_float(q & 0xffff0000u);
    } else {
      const float2 q = *reinterpret_cast<const float2*>((const float*)W + r * cols + k);
      a = q.x, b = q.y;
    }
  };
  float mx = 0.f;
  int bad = 0;
  for (int k = 2 * tid; k < cols; k += 512) {
    float a, b;
    load2(k, a, b);
    mx = fmaxf(mx, fmaxf(fabsf(a), fabsf(b)));
    bad |= (a - a != 0.f) | (b - b != 0.f);  // an infinity or a NaN
  }
  __shared__ float red[8];
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(FULLMASK, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  bad = __syncthreads_or(bad);
  mx = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) mx = fmaxf(mx, red[w]);
  float s = __fdiv_rn(mx, 448.f);
  if (s == 0.f) s = 1.f;
  if (bad) s = __int_as_float(0x7fc00000);
  for (int k = 2 * tid; k < cols; k += 512) {
    float a, b;
    load2(k, a, b);
    *reinterpret_cast<uint16_t*>(codes + r * cols + k) = (uint16_t)e4m3x2(__fdiv_rn(a, s), __fdiv_rn(b, s));
  }
  if (tid == 0) scales[r] = s;
}

extern "C" dc_status dc_quantize_fp8_rows_device(const void* W, int32_t dtype, int32_t rows, int32_t cols,
                                                 uint8_t* codes, float* scales, void* stream) {
  DC_NVTX("dc_quantize_fp8_rows_device");
  dc_clear_error();
  if (rows < 0 || cols < 0) return dc_fail(DC_ERR_INVALID_ARG, "negative size");
  if (cols % 16) return dc_fail(DC_ERR_SHAPE, "cols %d must be a multiple of 16", cols);
  if (dtype != DC_DTYPE_F32 && dtype != DC_DTYPE_BF16) return dc_fail(DC_ERR_INVALID_ARG, "dtype");
  if (rows == 0) return DC_OK;
  if (!W || !codes || !scales) return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(W) || !aligned16(codes) || !aligned16(scales)) return dc_fail(DC_ERR_ALIGN, "pointers must be 16-byte aligned");
  k_quant_fp8_rows<<<rows, 256, 0, (cudaStream_t)stream>>>(W, dtype == DC_DTYPE_BF16, cols, codes, scales);
  return dc_cuda_check(cudaGetLastError(), "fp8 quantise kernel");
}

extern "C" size_t dc_quantize_scratch_size(const dc_factor_desc* desc) {
  DC_NVTX("dc_quantize_scratch_size");
  DcLayout L;
  if (dc_check_desc(desc, &L) != DC_OK) return 0;
  return (size_t)(256 + dc_align((int64_t)L.r * L.d_out, 256) + dc_align((int64_t)L.r * L.d_in, 256) +
                  dc_align((int64_t)L.r * L.groups_out * 4, 256) + dc_align((int64_t)L.r * L.groups_in * 4, 256));
}

extern "C" dc_status dc_quantize_pack_device(const dc_factor_desc* desc, const float* U_dev, const float* Vt_dev,
                                             const float* S_dev, void* dev_dst, size_t dev_bytes, void* scratch,
                                             size_t scratch_bytes, void* stream, dc_delta_handle* out) {
  DC_NVTX("dc_quantize_pack_device");
  dc_clear_error();
  DcLayout L;
  dc_status st = dc_check_desc(desc, &L);
  if (st) return st;
  if (!dev_dst || !out || !scratch) return dc_fail(DC_ERR_INVALID_ARG, "null destination, scratch or handle");
  if (L.r > 0 && (!U_dev || !Vt_dev || !S_dev)) return dc_fail(DC_ERR_INVALID_ARG, "null factor pointer");
  if (((uintptr_t)dev_dst) % 256 || ((uintptr_t)scratch) % 256) return dc_fail(DC_ERR_ALIGN, "dst/scratch must be 256-byte aligned");
  if (!aligned16(U_dev) || !aligned16(Vt_dev)) return dc_fail(DC_ERR_ALIGN, "factors must be 16-byte aligned");
  if (dev_bytes < (size_t)L.bytes) return dc_fail(DC_ERR_WORKSPACE, "destination too small");
  if (scratch_bytes < dc_quantize_scratch_size(desc)) return dc_fail(DC_ERR_WORKSPACE, "scratch too small");
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* sc = (uint8_t*)scratch;
  int* status = (int*)sc;
  uint8_t* cu = sc + 256;
  uint8_t* cv = cu + dc_align((int64_t)L.r * L.d_out, 256);
  uint16_t* szu = (uint16_t*)(cv + dc_align((int64_t)L.r * L.d_in, 256));
  uint16_t* szv = (uint16_t*)((uint8_t*)szu + dc_align((int64_t)L.r * L.groups_out * 4, 256));
  if (L.r > 0) {
    const int64_t warps = (int64_t)L.r * (L.groups_in + L.groups_out);
    const int64_t blocks = (warps * 32 + 255) / 256;
    k_quant_plain<<<(unsigned)blocks, 256, 0, s>>>(L, U_dev, Vt_dev, cu, cv, szu, szv, status);
    st = dc_cuda_check(cudaGetLastError(), "quantise kernel");
    if (st) return st;
  }
  DcPlain Pl{cu, cv, szu, szv, S_dev, 0.f};  // the bound word is written by k_umax
  const int64_t nw = L.bytes / 4;
  const unsigned blocks = (unsigned)std::min<int64_t>((nw + 255) / 256, 148 * 64);
  k_pack_words<<<blocks, 256, 0, s>>>(L, Pl, (uint32_t*)dev_dst);
  st = dc_cuda_check(cudaGetLastError(), "pack kernel");
  if (st) return st;
  k_umax<<<1, 256, 0, s>>>(L, szu, (float*)((uint8_t*)dev_dst + L.umax_off));
  st = dc_cuda_check(cudaGetLastError(), "scale bound kernel");
  if (st) return st;
  dc_fill_handle(desc, L, dev_dst, out);
  return DC_OK;
}

// Per-device launch state (SM count, dynamic shared-memory limits set per kernel): these belong to
// each device's context, so they are keyed by the current device under one mutex.
static DcDevState g_devstate;

static int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) d = 0;
  return d;
}

static int device_sm_count(int dev) {
  return g_devstate.sm_count(dev, [](int d) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) return 0;
    return n;
  });
}

// Allow kernel `fn` (id `kid`) `need` bytes of dynamic shared memory on device `dev`.
static dc_status allow_smem(int dev, int kid, const void* fn, size_t need) {
  const int e = g_devstate.ensure_smem(dev, kid, need, [&](size_t n) {
    return (int)cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)n);
  });
  if (e == -1) return dc_fail(DC_ERR_UNSUPPORTED, "device index %d is beyond this build's table", dev);
  return e ? dc_cuda_check((cudaError_t)e, "shared-memory attribute") : DC_OK;
}

extern "C" dc_status dc_build_segments(const int32_t* tenant_ids_dev, int32_t T, int32_t n_tenants, void* ws,
                                       size_t ws_bytes, void* stream) {
  DC_NVTX("dc_build_segments");
  dc_clear_error();
  if (T < 0 || n_tenants < 0) return dc_fail(DC_ERR_INVALID_ARG, "negative T or tenant count");
  if (n_tenants > DC_MAX_TENANTS) return dc_fail(DC_ERR_UNSUPPORTED, "at most %d tenants per call", DC_MAX_TENANTS);
  if (!ws || (T > 0 && !tenant_ids_dev)) return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(ws)) return dc_fail(DC_ERR_ALIGN, "workspace must be 16-byte aligned");
  const DcWs W = dc_ws_layout(T, 0, 0, 1, 0);
  if (ws_bytes < (size_t)W.total) return dc_fail(DC_ERR_WORKSPACE, "workspace too small for routing");
  const size_t smem = (size_t)2 * (n_tenants + 1) * 4;
  if (smem > 48 * 1024) {
    const dc_status st = allow_smem(current_device(), DC_K_SEGMENTS, (const void*)k_segments, smem);
    if (st) return st;
  }
  k_segments<<<1, 256, smem, (cudaStream_t)stream>>>(tenant_ids_dev, T, n_tenants, (uint8_t*)ws, W);
  return dc_cuda_check(cudaGetLastError(), "routing kernel");
}

extern "C" dc_status dc_read_segments(const void* ws, int32_t T, int32_t* perm_dev, int32_t* inv_perm_dev,
                                      int32_t* segments_dev, int32_t* n_segments_dev, void* stream) {
  DC_NVTX("dc_read_segments");
  dc_clear_error();
  if (!ws || T < 0) return dc_fail(DC_ERR_INVALID_ARG, "bad arguments");
  if (!aligned16(ws) || !aligned16(perm_dev) || !aligned16(inv_perm_dev) || !aligned16(segments_dev) ||
      !aligned16(n_segments_dev))
    return dc_fail(DC_ERR_ALIGN, "device pointers must be 16-byte aligned");
  const DcWs W = dc_ws_layout(T, 0, 0, 1, 0);
  cudaStream_t s = (cudaStream_t)stream;
  const uint8_t* b = (const uint8_t*)ws;
  dc_status st = DC_OK;
  if (T > 0 && perm_dev) st = dc_cuda_check(cudaMemcpyAsync(perm_dev, b + W.perm, (size_t)T * 4, cudaMemcpyDeviceToDevice, s), "copy");
  if (!st && T > 0 && inv_perm_dev)
    st = dc_cuda_check(cudaMemcpyAsync(inv_perm_dev, b + W.inv, (size_t)T * 4, cudaMemcpyDeviceToDevice, s), "copy");
  if (!st && T > 0 && segments_dev)
    st = dc_cuda_check(cudaMemcpyAsync(segments_dev, b + W.segs, (size_t)T * 12, cudaMemcpyDeviceToDevice, s), "copy");
  if (!st && n_segments_dev)
    st = dc_cuda_check(cudaMemcpyAsync(n_segments_dev, b + W.status + 4 * DC_WS_NSEG, 4, cudaMemcpyDeviceToDevice, s), "copy");
  return st;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda dependency).
// The driver entry point is process-wide; the first call looks it up (thread-safe static init).
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return nullptr;
  }();
  return fn;
}

// 2-D tensor map of 16-bit elements (bf16 unless `dtype` says fp16): `rows` x `cols` (row pitch
// `pitch` elements), box 64 columns x box_rows rows, 128-byte swizzle.
// 2-D map of a row-major matrix (`pitch` elements between rows) whose box is one 128-byte row
// segment (64 16-bit or 128 8-bit elements) by `box_rows` rows, 128-byte swizzle.
static dc_status encode_map16(CUtensorMap* map, const void* base, int64_t cols, int64_t rows, int64_t pitch,
                                 int box_rows, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  auto enc = tensor_map_encoder();
  if (!enc) return dc_fail(DC_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int esz = dtype == CU_TENSOR_MAP_DATA_TYPE_UINT8 ? 1 : 2;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)pitch * esz};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return dc_fail(DC_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DC_OK;
}

// Shared driver of the single-linear and the 7-linear calls.
static dc_status run_forward(const dc_linear* lins, int n_lin, const void* const* xs, const int* dxs, void* const* ys,
                             const int32_t* ids, int32_t T, int32_t dtype_in, int32_t dtype_out, int32_t flags,
                             void* ws, size_t ws_bytes, void* stream) {
  if (T < 0) return dc_fail(DC_ERR_INVALID_ARG, "negative T");
  if (T == 0) return DC_OK;
  if (!ws || !ids) return dc_fail(DC_ERR_INVALID_ARG, "null workspace or tenant ids");
  if (!aligned16(ws)) return dc_fail(DC_ERR_ALIGN, "workspace must be 16-byte aligned");
  if (dtype_in != DC_DTYPE_F32 && dtype_in != DC_DTYPE_BF16) return dc_fail(DC_ERR_INVALID_ARG, "dtype_in");
  if (dtype_out != DC_DTYPE_F32 && dtype_out != DC_DTYPE_BF16) return dc_fail(DC_ERR_INVALID_ARG, "dtype_out");
  if (!(flags & (DC_BASE | DC_DELTA))) return dc_fail(DC_ERR_INVALID_ARG, "flags select neither base nor delta");
  DcFwd F;
  std::memset(&F, 0, sizeof(F));
  F.n_lin = n_lin;
  F.T = T;
  F.dtype_in = dtype_in;
  F.dtype_out = dtype_out;
  F.flags = flags;
  int max_rank = 0, max_d_in = 0, max_ten = 0;
  const int n_in = n_lin == 7 ? 3 : 1;
  for (int m = 0; m < n_in; ++m) {
    F.x[m] = xs[m];
    F.dx[m] = dxs[m];
    if (!xs[m]) return dc_fail(DC_ERR_INVALID_ARG, "null input %d", m);
    if (!aligned16(xs[m])) return dc_fail(DC_ERR_ALIGN, "input %d not 16-byte aligned", m);
    max_d_in = std::max(max_d_in, dxs[m]);
  }
  for (int p = 0; p < n_lin; ++p) {
    const dc_linear& l = lins[p];
    if (!l.W_base && (flags & DC_BASE)) return dc_fail(DC_ERR_INVALID_ARG, "linear %d: null W_base", p);
    if (!ys[p]) return dc_fail(DC_ERR_INVALID_ARG, "linear %d: null output", p);
    if (!aligned16(l.W_base) || !aligned16(ys[p])) return dc_fail(DC_ERR_ALIGN, "linear %d: pointer not 16-byte aligned", p);
    if (l.d_out <= 0 || l.d_in <= 0 || l.d_out % 128 || l.d_in % 128)
      return dc_fail(DC_ERR_SHAPE, "linear %d: d_out=%d d_in=%d must be multiples of 128", p, l.d_out, l.d_in);
    const int m = n_lin == 7 ? (p == 3 ? 1 : (p == 6 ? 2 : 0)) : 0;
    if (l.d_in != dxs[m]) return dc_fail(DC_ERR_SHAPE, "linear %d: d_in %d does not match its input (%d)", p, l.d_in, dxs[m]);
    if (l.w_dtype != DC_DTYPE_BF16 && l.w_dtype != DC_DTYPE_F32 && l.w_dtype != DC_DTYPE_FP8)
      return dc_fail(DC_ERR_INVALID_ARG, "linear %d: w_dtype", p);
    if ((flags & DC_BASE) && (l.w_dtype == DC_DTYPE_FP8) != (lins[0].w_dtype == DC_DTYPE_FP8))
      return dc_fail(DC_ERR_UNSUPPORTED, "linear %d: an fp8 backbone needs every linear of the call in fp8", p);
    if (l.w_dtype == DC_DTYPE_BF16 && dtype_in != DC_DTYPE_BF16 && (flags & DC_BASE))
      return dc_fail(DC_ERR_UNSUPPORTED, "linear %d: bf16 weights need bf16 activations", p);
    if (l.n_tenants < 0 || l.n_tenants > DC_MAX_TENANTS) return dc_fail(DC_ERR_INVALID_ARG, "linear %d: tenant count", p);
    if ((flags & DC_DELTA) && l.n_tenants > 0 && !l.tenants_dev) return dc_fail(DC_ERR_INVALID_ARG, "linear %d: null tenant table", p);
    if (l.max_rank < 0 || l.max_rank > std::min(l.d_out, l.d_in)) return dc_fail(DC_ERR_SHAPE, "linear %d: max_rank", p);
    max_rank = std::max(max_rank, l.max_rank);
    max_ten = std::max(max_ten, l.n_tenants);
    max_d_in = std::max(max_d_in, l.d_out);  // the workspace's per-token rows also hold outputs
    F.lin[p].W = l.W_base;
    F.lin[p].tenants = l.tenants_dev;
    F.lin[p].y = ys[p];
    F.lin[p].d_out = l.d_out;
    F.lin[p].d_in = l.d_in;
    F.lin[p].n_tenants = l.n_tenants;
    F.lin[p].w_dtype = l.w_dtype;
    F.lin[p].input = m;
  }
  F.ws = dc_ws_layout(T, max_rank, max_d_in, n_lin, max_ten);
  if (ws_bytes < (size_t)F.ws.total)
    return dc_fail(DC_ERR_WORKSPACE, "workspace holds %zu bytes, need %lld", ws_bytes, (long long)F.ws.total);
  // bf16 backbones with bf16 activations, and fp8 backbones (activations quantised per token by
  // k_prep), run on the tcgen05 tensor cores
  F.fp8 = (flags & DC_BASE) && lins[0].w_dtype == DC_DTYPE_FP8;
  bool use_tc = (flags & DC_BASE) && dtype_in == DC_DTYPE_BF16;
  for (int p = 0; p < n_lin; ++p) use_tc = use_tc && lins[p].w_dtype == DC_DTYPE_BF16;
  use_tc = use_tc || F.fp8;
  if (F.fp8) {
    for (int p = 0; p < n_lin; ++p) {
      dc_status st0 = encode_map16(&F.wmap[p], lins[p].W_base, lins[p].d_in, lins[p].d_out, lins[p].d_in, 128,
                                   CU_TENSOR_MAP_DATA_TYPE_UINT8);
      if (st0) return st0;
    }
    for (int m = 0; m < n_in; ++m) {
      const uint8_t* xb = (const uint8_t*)ws + F.ws.x8 + (int64_t)m * T * F.ws.max_d_in;
      dc_status st0 = encode_map16(&F.xmap[m], xb, dxs[m], T, F.ws.max_d_in, F.ws.bt_nb, CU_TENSOR_MAP_DATA_TYPE_UINT8);
      if (st0) return st0;
    }
  } else if (flags & DC_BASE) {
    for (int p = 0; p < n_lin; ++p)
      if (lins[p].w_dtype == DC_DTYPE_BF16) {
        dc_status st0 = encode_map16(&F.wmap[p], lins[p].W_base, lins[p].d_in, lins[p].d_out, lins[p].d_in, 128);
        if (st0) return st0;
      }
    if (dtype_in == DC_DTYPE_BF16)
      for (int m = 0; m < n_in; ++m) {
        const uint8_t* xb = (const uint8_t*)ws + F.ws.xsort + (int64_t)m * T * F.ws.max_d_in * 2;
        dc_status st0 = encode_map16(&F.xmap[m], xb, dxs[m], T, F.ws.max_d_in, use_tc ? F.ws.bt_nb : std::min(64, T));
        if (st0) return st0;
      }
  }
  // U-kernel and backbone order: largest output tiles first (d_in decides the bytes per tile)
  bt_plan_order(F);
  // long segments take the tensor-core delta path when the batch is large enough
  F.pf = (flags & DC_DELTA) && !(flags & DC_DECODE_ONLY) && T >= 2 * DC_PF_MIN;
  if (F.pf) {
    if (dtype_in != DC_DTYPE_BF16) return dc_fail(DC_ERR_UNSUPPORTED, "the prefill path needs bf16 activations");
    dc_status st0 = encode_map16(&F.tmap, (const uint8_t*)ws + F.ws.t16, F.ws.tcols, (int64_t)n_lin * T,
                                    F.ws.tcols, 256, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (st0) return st0;
    F.pf_box = std::min(256, T);
    for (int m = 0; m < n_in; ++m) {
      const uint8_t* xb = (const uint8_t*)ws + F.ws.xs16 + (int64_t)m * T * F.ws.max_d_in * 2;
      st0 = encode_map16(&F.xpf[m], xb, dxs[m], T, F.ws.max_d_in, F.pf_box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
      if (st0) return st0;
    }
  }
  cudaStream_t s = (cudaStream_t)stream;
  const int dev = current_device();
  dc_status st;
  if (!(flags & DC_REUSE_ROUTING)) {
    if (max_ten > DC_MAX_TENANTS) return dc_fail(DC_ERR_UNSUPPORTED, "too many tenants");
    const size_t smem = (size_t)2 * (max_ten + 1) * 4;
    if (smem > 48 * 1024) {
      st = allow_smem(dev, DC_K_SEGMENTS, (const void*)k_segments, smem);
      if (st) return st;
    }
    prof_before(s, 0);
    k_segments<<<1, 256, smem, s>>>(ids, T, max_ten, (uint8_t*)ws, F.ws);
    prof_after(s);
    st = dc_cuda_check(cudaGetLastError(), "routing kernel");
    if (st) return st;
  }
  prof_before(s, 1);
  // work counters (item count, work cursors) and per-token delta flags start from zero on every call
  static_assert(VP_COUNTER_SLOT < UP_COUNTER_SLOT && UP_COUNTER_SLOT < DC_WS_SLOTS, "status words");
  st = dc_cuda_check(cudaMemsetAsync((uint8_t*)ws + F.ws.status + 4 * DC_WS_VCOUNTER, 0, 4 * (UP_COUNTER_SLOT - DC_WS_VCOUNTER + 1), s),
                     "counter reset");
  if (st) return st;
  // the delta flags are written for every token by k_prep's record blocks (every token is in a
  // segment); its limb blocks zero the output bounds and the backbone unit counters
  const int nb_items = (T + 255) / 256;
  k_prep<<<dim3(T + nb_items, std::max(n_in, n_lin)), 256, 0, s>>>(F, (uint8_t*)ws);
  prof_after(s);
  st = dc_cuda_check(cudaGetLastError(), "prep kernel");
  if (st) return st;
  const int n_sm = device_sm_count(dev);
  if (flags & DC_DELTA) {
    const size_t vsmem = (size_t)V_STAGES * V_STAGE_BYTES + sizeof(VSmemTail);
    st = allow_smem(dev, DC_K_VSTAGE, (const void*)k_vstage, vsmem);
    if (st) return st;
    prof_before(s, 2);
    k_vstage<<<V_CTAS_PER_SM * n_sm, V_THREADS, vsmem, s>>>(F, (uint8_t*)ws);
    prof_after(s);
    st = dc_cuda_check(cudaGetLastError(), "rank-reduction kernel");
    if (st) return st;
    if (F.pf) {
      const size_t qsmem = 1024 + (size_t)VP_STAGES * VP_STAGE_BYTES + 2 * VP_BLK_BYTES + sizeof(VpTail);
      st = allow_smem(dev, DC_K_VPRE, (const void*)k_vpre, qsmem);
      if (st) return st;
      prof_before(s, 2);
      k_vpre<<<n_sm, VP_THREADS, qsmem, s>>>(F, (uint8_t*)ws);
      prof_after(s);
      st = dc_cuda_check(cudaGetLastError(), "prefill rank-reduction kernel");
      if (st) return st;
    }
  }
  if (flags & DC_DELTA) {
    const size_t usmem = (size_t)U_STAGES * U_STAGE_BYTES + 2 * U_GSTAGE * U_LBUF + sizeof(USmemTail);
    if (usmem > 227 * 1024)
      return dc_fail(DC_ERR_UNSUPPORTED, "max_rank %d needs %zu bytes of shared memory", max_rank, usmem);
    st = allow_smem(dev, DC_K_UDELTA, (const void*)k_udelta, usmem);
    if (st) return st;
    prof_before(s, 3);
    k_udelta<<<U_CTAS_PER_SM * n_sm, U_THREADS, usmem, s>>>(F, (uint8_t*)ws);
    prof_after(s);
    st = dc_cuda_check(cudaGetLastError(), "delta output kernel");
    if (st) return st;
    if (F.pf) {
      const size_t psmem = 1024 + (size_t)UP_STAGES * UP_STAGE_BYTES + 2 * UP_BLK_BYTES + sizeof(UpTail);
      st = allow_smem(dev, DC_K_UPRE, (const void*)k_upre, psmem);
      if (st) return st;
      prof_before(s, 3);
      k_upre<<<n_sm, UP_THREADS, psmem, s>>>(F, (uint8_t*)ws);
      prof_after(s);
      st = dc_cuda_check(cudaGetLastError(), "prefill delta output kernel");
      if (st) return st;
    }
  }
  if (use_tc) {
    bt_plan(F, T, F.ws.bt_nb, std::min(n_sm, DC_BT_MAX_CTAS));
    const int stage_bytes = BT_A_BYTES + F.ws.bt_nb * 128;
    F.bt_ns = std::min(BT_MAX_STAGES, (int)((200 * 1024) / stage_bytes));
    const size_t tsmem = 1024 + (size_t)F.bt_ns * stage_bytes + sizeof(BtTail);
    st = allow_smem(dev, DC_K_BASE_TC, (const void*)k_base_tc, tsmem);
    if (st) return st;
    prof_before(s, 4);  // the unit counters were zeroed with the call's other per-call state
    k_base_tc<<<F.bt_grid, BT_THREADS, tsmem, s>>>(F, (uint8_t*)ws);
    prof_after(s);
    return dc_cuda_check(cudaGetLastError(), "tensor-core output kernel");
  }
  const size_t bsmem = 1024 + (size_t)B_STAGES * B_STAGE_BYTES + sizeof(BSmemTail);
  st = allow_smem(dev, DC_K_BASE, (const void*)k_base, bsmem);
  if (st) return st;
  const int n_units = F.tile_prefix[n_lin] * ((T + DC_TOK_BLOCK - 1) / DC_TOK_BLOCK);
  prof_before(s, 4);
  k_base<<<std::min(n_sm, n_units), KB_THREADS, bsmem, s>>>(F, (uint8_t*)ws);
  prof_after(s);
  return dc_cuda_check(cudaGetLastError(), "output kernel");
}

extern "C" dc_status dc_delta_linear_segmented(const dc_linear* lin, const void* x, void* y, const int32_t* tenant_ids_dev,
                                               int32_t T, int32_t dtype_in, int32_t dtype_out, int32_t flags, void* ws,
                                               size_t ws_bytes, void* stream) {
  DC_NVTX("dc_delta_linear_segmented");
  dc_clear_error();
  if (!lin) return dc_fail(DC_ERR_INVALID_ARG, "null linear");
  const void* xs[1] = {x};
  const int dx[1] = {lin->d_in};
  void* ys[1] = {y};
  return run_forward(lin, 1, xs, dx, ys, tenant_ids_dev, T, dtype_in, dtype_out, flags, ws, ws_bytes, stream);
}

extern "C" dc_status dc_layer_forward(const dc_linear lin[7], const void* x_h, const void* x_o, const void* x_f,
                                      void* const y[7], const int32_t* tenant_ids_dev, int32_t T, int32_t dtype_in,
                                      int32_t dtype_out, int32_t flags, void* ws, size_t ws_bytes, void* stream) {
  DC_NVTX("dc_layer_forward");
  dc_clear_error();
  if (!lin || !y) return dc_fail(DC_ERR_INVALID_ARG, "null linear array or outputs");
  const void* xs[3] = {x_h, x_o, x_f};
  const int dx[3] = {lin[0].d_in, lin[3].d_in, lin[6].d_in};
  return run_forward(lin, 7, xs, dx, y, tenant_ids_dev, T, dtype_in, dtype_out, flags, ws, ws_bytes, stream);
}

extern "C" dc_status dc_unpack_codes_debug(const dc_delta_handle* h, int32_t which, uint8_t* out_dev, void* stream) {
  DC_NVTX("dc_unpack_codes_debug");
  dc_clear_error();
  if (!h || !out_dev || h->dev_base == 0) return dc_fail(DC_ERR_INVALID_ARG, "bad handle or output");
  if (!aligned16(out_dev) || (h->dev_base & 255) != 0) return dc_fail(DC_ERR_ALIGN, "output or blob misaligned");
  DcLayout L;
  dc_status st = dc_check_desc(&h->desc, &L);
  if (st) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const uint8_t* blob = (const uint8_t*)(uintptr_t)h->dev_base;
  for (int b = 0; b < L.n_bands; ++b) {
    const DcBand& B = L.band[b];
    if (which == 1) {
      const int64_t n = (int64_t)B.v_tiles * L.nkb * 64;
      k_unpack_v<<<(unsigned)((n + 127) / 128), 128, 0, s>>>(blob, L, b, out_dev);
    } else if (which == 0) {
      const int64_t n = (int64_t)L.d_out * B.rank;
      k_unpack_u<<<(unsigned)((n + 127) / 128), 128, 0, s>>>(blob, L, b, out_dev);
    } else {
      return dc_fail(DC_ERR_INVALID_ARG, "which must be 0 (U) or 1 (V)");
    }
    st = dc_cuda_check(cudaGetLastError(), "unpack kernel");
    if (st) return st;
  }
  return DC_OK;
}

extern "C" dc_status dc_read_device_status(void* ws, void* stream, int32_t* host_status) {
  DC_NVTX("dc_read_device_status");
  dc_clear_error();
  if (!ws || !host_status) return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(ws)) return dc_fail(DC_ERR_ALIGN, "workspace must be 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  int32_t v = 0;
  dc_status st = dc_cuda_check(cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, s), "status read");
  if (st) return st;
  st = dc_cuda_check(cudaStreamSynchronize(s), "status sync");
  if (st) return st;
  *host_status = v;
  return dc_cuda_check(cudaMemsetAsync(ws, 0, 4, s), "status clear");
}

// ---------------------------------------------------------------------------------------------
// Allocation-free serving of one linear from a workspace compiled into the library.  For callers
// that cannot allocate per call (no caching allocator, or a device memory plan fixed at start-up):
// the workspace is a static device array, and its device address is looked up once per device.
// ---------------------------------------------------------------------------------------------
static __device__ __align__(256) uint8_t dc_static_ws[DC_STATIC_WORKSPACE_BYTES];

namespace {
std::mutex g_static_mu;
void* g_static_ptr[DC_MAX_DEVICES];  // device address of dc_static_ws per device, once looked up
}  // namespace

extern "C" dc_status dc_delta_linear_segmented_static(const dc_linear* lin, const void* x, void* y,
                                                      const int32_t* tenant_ids_dev, int32_t T, int32_t dtype_in,
                                                      int32_t dtype_out, int32_t flags, void* stream,
                                                      int32_t* host_status) {
  DC_NVTX("dc_delta_linear_segmented_static");
  dc_clear_error();
  if (!lin) return dc_fail(DC_ERR_INVALID_ARG, "null linear");
  if (flags & DC_REUSE_ROUTING)
    return dc_fail(DC_ERR_INVALID_ARG, "the static workspace rebuilds the routing on every call (no DC_REUSE_ROUTING)");
  if (T < 0) return dc_fail(DC_ERR_INVALID_ARG, "negative T");
  if (!aligned16(x) || !aligned16(y) || !aligned16(lin->W_base))
    return dc_fail(DC_ERR_ALIGN, "device pointers must be 16-byte aligned");
  if (T == 0) {  // nothing launched: report a clean status
    if (host_status) *host_status = 0;
    return DC_OK;
  }
  const size_t need =
      dc_workspace_size(T, lin->max_rank, std::max(lin->d_in, lin->d_out), 1, lin->n_tenants);
  if (need == 0) return dc_fail(DC_ERR_INVALID_ARG, "invalid sizes in the linear");
  if (need > DC_STATIC_WORKSPACE_BYTES)
    return dc_fail(DC_ERR_WORKSPACE,
                   "this request needs %zu bytes of workspace; the static workspace holds %zu "
                   "(use dc_delta_linear_segmented with a caller workspace)",
                   need, (size_t)DC_STATIC_WORKSPACE_BYTES);
  int dev = 0;
  dc_status st = dc_cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (st) return st;
  if (dev < 0 || dev >= DC_MAX_DEVICES) return dc_fail(DC_ERR_UNSUPPORTED, "device index %d", dev);
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
      void* p = nullptr;
      st = dc_cuda_check(cudaGetSymbolAddress(&p, dc_static_ws), "cudaGetSymbolAddress(static workspace)");
      if (st) return st;
      g_static_ptr[dev] = p;
    }
    ws = g_static_ptr[dev];
  }
  st = dc_delta_linear_segmented(lin, x, y, tenant_ids_dev, T, dtype_in, dtype_out, flags, ws,
                                 DC_STATIC_WORKSPACE_BYTES, stream);
  if (st || !host_status) return st;
  return dc_read_device_status(ws, stream, host_status);
}
