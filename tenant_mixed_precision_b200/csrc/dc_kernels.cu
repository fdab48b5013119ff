// Serving kernels for multi-tenant mixed-precision deltas on B200 (sm_100a).
//
// Per batch (one call of dc_delta_linear_segmented / dc_layer_forward):
//   k_segments  token routing: stable counting sort of tenant ids into segments.
//   k_prep      per sorted token: the activation as a 24-bit fixed-point integer split into three
//               signed 8-bit limbs (so u8 x s8 tensor-core MMAs reproduce x exactly to 2^-22 of
//               the token's largest entry), limb sums per group of 128, and (one extra block)
//               the per-(linear, tenant) layouts plus the V work list.
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
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "dc.h"
#include "dc_internal.h"
#include "dc_layout.h"
#include "dc_pack.h"

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
  W.layouts = take((int64_t)n_lin * max_tenants * sizeof(DcLayout));
  W.xl = take((int64_t)W.n_in * 3 * T * W.max_d_in);
  W.xs = take((int64_t)W.n_in * T * (W.max_d_in / 128) * 16);
  W.xe = take((int64_t)W.n_in * T * 4);
  W.tws = take((int64_t)n_lin * T * W.r_stride * 4);
  W.total = off;
  return W;
}

extern "C" size_t dc_workspace_size(int32_t T, int32_t max_rank, int32_t max_d_in, int32_t n_linears,
                                    int32_t max_tenants) {
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
  DcLinDev lin[7];
  const void* x[3];
  int32_t dx[3];
  int32_t n_lin, T, dtype_in, dtype_out, flags, bsm_max;
  int32_t order[7];        // launch order of the linears in the U kernel (largest first)
  int32_t tile_prefix[8];  // cumulative 128-row output tiles in that order
  DcWs ws;
};

struct WsPtr {
  int* st;
  int* perm;
  int* inv;
  int* segs;
  DcVItem* items;
  DcLayout* layouts;
  int8_t* xl;
  int* xs;
  int* xe;
  float* tws;
};
__device__ __forceinline__ WsPtr ws_ptr(const DcWs& W, uint8_t* ws) {
  WsPtr p;
  p.st = (int*)(ws + W.status);
  p.perm = (int*)(ws + W.perm);
  p.inv = (int*)(ws + W.inv);
  p.segs = (int*)(ws + W.segs);
  p.items = (DcVItem*)(ws + W.items);
  p.layouts = (DcLayout*)(ws + W.layouts);
  p.xl = (int8_t*)(ws + W.xl);
  p.xs = (int*)(ws + W.xs);
  p.xe = (int*)(ws + W.xe);
  p.tws = (float*)(ws + W.tws);
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
// k_prep: activation limbs, limb sums, exponents; the last block builds layouts and V items.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ int sext8(int v) { return (int)(int8_t)(v & 0xff); }

__device__ void build_layouts_and_items(const DcFwd& F, const WsPtr& P) {
  const DcWs& W = F.ws;
  const int tid = threadIdx.x;
  for (int idx = tid; idx < F.n_lin * W.max_tenants; idx += blockDim.x) {
    const int p = idx / W.max_tenants, tau = idx % W.max_tenants;
    DcLayout L;
    L.valid = 0;
    if (tau < F.lin[p].n_tenants) {
      const dc_delta_handle* h = F.lin[p].tenants + tau;
      if (h->dev_base != 0) {
        L = dc_layout(h->desc);
        if (L.valid && (L.d_out != F.lin[p].d_out || L.d_in != F.lin[p].d_in || L.r > W.r_stride ||
                        L.bsm_total > F.bsm_max)) {
          L.valid = 0;
          set_status(P.st, DC_ERR_SHAPE);
        }
        if (!L.valid) set_status(P.st, DC_ERR_SHAPE);
        L.dev_base = (int64_t)h->dev_base;
      }
    }
    P.layouts[idx] = L;
  }
  __syncthreads();
  __shared__ int n_items;
  if (tid == 0) n_items = 0;
  __syncthreads();
  const int nseg = P.st[DC_WS_NSEG];
  if (F.flags & DC_DELTA) {
    // projections in decreasing d_in so that long items are handed out first
    int ord[7];
    for (int i = 0; i < F.n_lin; ++i) ord[i] = i;
    for (int i = 0; i < F.n_lin; ++i)
      for (int j = i + 1; j < F.n_lin; ++j)
        if (F.lin[ord[j]].d_in > F.lin[ord[i]].d_in) {
          const int tmp = ord[i];
          ord[i] = ord[j];
          ord[j] = tmp;
        }
    for (int oi = 0; oi < F.n_lin; ++oi) {
      const int p = ord[oi];
      for (int s = tid; s < nseg; s += blockDim.x) {
        const int tau = P.segs[3 * s], len = P.segs[3 * s + 2];
        if (tau >= F.lin[p].n_tenants || tau >= W.max_tenants) continue;
        const DcLayout& L = P.layouts[p * W.max_tenants + tau];
        if (!L.valid) continue;
        const int passes = (len + DC_V_TOKS - 1) / DC_V_TOKS;
        int per_pass = 0;
        for (int b = 0; b < L.n_bands; ++b) per_pass += (L.band[b].v_tiles + DC_V_NT - 1) / DC_V_NT;
        const int count = passes * per_pass;
        const int base = atomicAdd(&n_items, count);
        if (base + count > W.max_items) {
          set_status(P.st, DC_ERR_WORKSPACE);
          continue;
        }
        int k = base;
        for (int ps = 0; ps < passes; ++ps)
          for (int b = 0; b < L.n_bands; ++b)
            for (int t0 = 0; t0 < L.band[b].v_tiles; t0 += DC_V_NT) {
              DcVItem it;
              it.p = (int16_t)p;
              it.band = (int16_t)b;
              it.seg = s;
              it.tile0 = t0;
              it.ntiles = (int16_t)min(DC_V_NT, L.band[b].v_tiles - t0);
              it.pass = (int16_t)ps;
              P.items[k++] = it;
            }
      }
      __syncthreads();
    }
  }
  __syncthreads();
  if (tid == 0) {
    P.st[DC_WS_NITEMS] = min(n_items, W.max_items);
    P.st[DC_WS_VCOUNTER] = 0;
  }
}

__global__ void __launch_bounds__(256) k_prep(const __grid_constant__ DcFwd F, uint8_t* ws) {
  const DcWs& W = F.ws;
  WsPtr P = ws_ptr(W, ws);
  if (blockIdx.x == (unsigned)W.T) {
    if (blockIdx.y == 0) build_layouts_and_items(F, P);
    return;
  }
  if (!(F.flags & DC_DELTA)) return;
  const int j = blockIdx.x, m = blockIdx.y;
  const int d = F.dx[m];
  const int T = W.T, maxd = W.max_d_in, G = maxd / 128;
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
  for (int k = tid * 4; k < d; k += 1024) {
    float v[4];
    load4(k, v);
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
    int8_t* base = P.xl + ((int64_t)(m * 3) * T + j) * maxd + k;
    *reinterpret_cast<uint32_t*>(base) = w0;
    *reinterpret_cast<uint32_t*>(base + (int64_t)T * maxd) = w1;
    *reinterpret_cast<uint32_t*>(base + (int64_t)2 * T * maxd) = w2;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      s0 += __shfl_xor_sync(FULLMASK, s0, o);
      s1 += __shfl_xor_sync(FULLMASK, s1, o);
      s2 += __shfl_xor_sync(FULLMASK, s2, o);
    }
    if (lane == 0) {
      int* xs = P.xs + ((int64_t)(m * T + j) * G + k / 128) * 4;
      xs[0] = s0, xs[1] = s1, xs[2] = s2, xs[3] = 0;
    }
  }
  if (tid == 0) P.xe[m * T + j] = e;
}

// ---------------------------------------------------------------------------------------------
// k_vstage: t = S * (V_hat^T x) for every (linear, segment, token pass, band, 2 tiles)
// ---------------------------------------------------------------------------------------------
struct VCtx {
  const uint8_t* blob;
  const DcLayout* L;
  int band;
  int tile0, ntiles;
  int tok0, ntok;  // sorted token positions of this pass
  int m, p;
};

// Epilogue of one group for one tile: acc += (s/w) * (C - w z XS) for the valid pairs.
__device__ __forceinline__ void v_group_epilogue(float (&acc)[2][4], const int (&C)[2][4], uint2 meta, float w,
                                                 const int (&xs)[2][2], int npair) {
  const __half2 m0 = *reinterpret_cast<const __half2*>(&meta.x);  // (scale, zero) of row g
  const __half2 m1 = *reinterpret_cast<const __half2*>(&meta.y);  // row g+8
  const float inv = 1.f / w;
  const float sA = __low2float(m0) * inv, zA = __high2float(m0) * w;
  const float sB = __low2float(m1) * inv, zB = __high2float(m1) * w;
#pragma unroll
  for (int pr = 0; pr < 2; ++pr) {
    if (pr < npair) {
      acc[pr][0] += sA * fmaf(-zA, (float)xs[pr][0], (float)C[pr][0]);
      acc[pr][1] += sA * fmaf(-zA, (float)xs[pr][1], (float)C[pr][1]);
      acc[pr][2] += sB * fmaf(-zB, (float)xs[pr][0], (float)C[pr][2]);
      acc[pr][3] += sB * fmaf(-zB, (float)xs[pr][1], (float)C[pr][3]);
    }
  }
}

template <int BITS>
__device__ void v_item(const DcFwd& F, const WsPtr& P, const VCtx& c, int lane) {
  const DcLayout& L = *c.L;
  const DcBand& B = L.band[c.band];
  const int g = lane >> 2, t = lane & 3;
  const int T = F.ws.T, maxd = F.ws.max_d_in, G = maxd / 128;
  const int npair = (c.ntok + 1) >> 1;
  // B operand: lane g < 6 supplies limb g>>1 of token (g&1) of each pair
  const int limb = g >> 1;
  const int8_t* xsrc[2];
  bool xval[2];
#pragma unroll
  for (int pr = 0; pr < 2; ++pr) {
    const int tk = 2 * pr + (g & 1);
    xval[pr] = (g < 6) && (tk < c.ntok);
    xsrc[pr] = P.xl + ((int64_t)(c.m * 3 + (g < 6 ? limb : 0)) * T + c.tok0 + (xval[pr] ? tk : 0)) * maxd + 32 * t;
  }
  const int* xsp[2][2];
  bool xsv[2][2];
#pragma unroll
  for (int pr = 0; pr < 2; ++pr)
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int tk = 2 * pr + q;
      xsv[pr][q] = (t < 3) && (tk < c.ntok);
      xsp[pr][q] = P.xs + ((int64_t)(c.m * T + c.tok0 + (xsv[pr][q] ? tk : 0)) * G) * 4 + (t < 3 ? t : 0);
    }
  float acc[DC_V_NT][2][4];
#pragma unroll
  for (int a = 0; a < DC_V_NT; ++a)
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[a][b][q] = 0.f;
  int rows[DC_V_NT], nh[DC_V_NT][2];
  const uint8_t* tb[DC_V_NT];
#pragma unroll
  for (int ti = 0; ti < DC_V_NT; ++ti) {
    const int tile = c.tile0 + ti;
    rows[ti] = ti < c.ntiles ? min(16, B.rank - 16 * tile) : 0;
    nh[ti][0] = min(rows[ti], 8);
    nh[ti][1] = max(0, rows[ti] - 8);
    tb[ti] = c.blob + B.v_off + (int64_t)tile * B.v_tile_bytes;
  }
  const uint8_t* vmeta = c.blob + B.v_meta_off;
  for (int kb = 0; kb < L.nkb; ++kb) {
    const int ngrp = (kb == L.nkb - 1) ? L.tail_groups : 4;
    const bool mask_layout = (BITS == 2) && (ngrp == 4);
    uint4 wm[DC_V_NT][2][2];  // 2-bit mask layout: 8 words per lane-row for the block
    if (mask_layout) {
#pragma unroll
      for (int ti = 0; ti < DC_V_NT; ++ti)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (g < nh[ti][h]) {
            const uint8_t* pp = tb[ti] + (int64_t)kb * dc_v_block_bytes(2, rows[ti], 4) +
                                dc_v_half_off(2, rows[ti], 4, h) + lane * 32;
            wm[ti][h][0] = ldg128(pp);
            wm[ti][h][1] = ldg128(pp + 16);
          } else {
            wm[ti][h][0] = make_uint4(0, 0, 0, 0);
            wm[ti][h][1] = make_uint4(0, 0, 0, 0);
          }
        }
    }
    for (int grp = 0; grp < ngrp; ++grp) {
      const int gi = 4 * kb + grp;
      uint32_t bw[2][8];
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        if (xval[pr]) {
          const uint4 q0 = ldg128(xsrc[pr] + gi * 128), q1 = ldg128(xsrc[pr] + gi * 128 + 16);
          bw[pr][0] = q0.x, bw[pr][1] = q0.y, bw[pr][2] = q0.z, bw[pr][3] = q0.w;
          bw[pr][4] = q1.x, bw[pr][5] = q1.y, bw[pr][6] = q1.z, bw[pr][7] = q1.w;
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) bw[pr][q] = 0u;
        }
      }
      int xs[2][2];
#pragma unroll
      for (int pr = 0; pr < 2; ++pr)
#pragma unroll
        for (int q = 0; q < 2; ++q) xs[pr][q] = xsv[pr][q] ? xsp[pr][q][gi * 4] : 0;
#pragma unroll
      for (int ti = 0; ti < DC_V_NT; ++ti) {
        if (ti >= c.ntiles) continue;
        const uint2 meta = ldg64(vmeta + (((int64_t)(c.tile0 + ti) * L.groups_in + gi) * 8 + g) * 8);
        // the lane-row words for this group (shift layouts and 8-bit load per group)
        uint32_t a[4][4];  // [step][reg]
        if (mask_layout) {
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            a[s][0] = v_reg_mask2(wsel(wm[ti][0][s >> 1], 2 * (s & 1)), grp);
            a[s][1] = v_reg_mask2(wsel(wm[ti][1][s >> 1], 2 * (s & 1)), grp);
            a[s][2] = v_reg_mask2(wsel(wm[ti][0][s >> 1], 2 * (s & 1) + 1), grp);
            a[s][3] = v_reg_mask2(wsel(wm[ti][1][s >> 1], 2 * (s & 1) + 1), grp);
          }
        } else {
          const uint8_t* blk = tb[ti] + (int64_t)kb * dc_v_block_bytes(BITS, rows[ti], 4);
          const int p0 = dc_v_plane0_bytes(BITS, ngrp);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const bool ok = g < nh[ti][h];
            const uint8_t* hb = blk + dc_v_half_off(BITS, rows[ti], ngrp, h);
            if (BITS == 8) {
              uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0;
              if (ok) {
                q0 = ldg128(hb + lane * p0 + 32 * grp);
                q1 = ldg128(hb + lane * p0 + 32 * grp + 16);
              }
#pragma unroll
              for (int s = 0; s < 4; ++s) {
                const uint4& q = (s < 2) ? q0 : q1;
                a[s][h] = wsel(q, 2 * (s & 1));
                a[s][h + 2] = wsel(q, 2 * (s & 1) + 1);
              }
            } else {
              uint2 w2 = make_uint2(0, 0);
              uint32_t w1 = 0;
              if (ok) {
                w2 = ldg64(hb + lane * p0 + 8 * grp);
                if (BITS == 3) w1 = ldg32(hb + (int64_t)4 * nh[ti][h] * p0 + lane * (4 * ngrp) + 4 * grp);
              }
#pragma unroll
              for (int s = 0; s < 4; ++s)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                  const uint32_t w = (s >> 1) ? w2.y : w2.x;
                  uint32_t r = reg_shift2(w, 2 * (s & 1) + hh);
                  if (BITS == 3) r |= v_reg_hi3(w1, s, hh);
                  a[s][h + 2 * hh] = r;
                }
            }
          }
        }
        int C[2][4];
#pragma unroll
        for (int pr = 0; pr < 2; ++pr)
#pragma unroll
          for (int q = 0; q < 4; ++q) C[pr][q] = 0;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          mma_u8s8(C[0], a[s][0], a[s][1], a[s][2], a[s][3], bw[0][2 * s], bw[0][2 * s + 1]);
          if (npair > 1) mma_u8s8(C[1], a[s][0], a[s][1], a[s][2], a[s][3], bw[1][2 * s], bw[1][2 * s + 1]);
        }
        const float w = mask_layout ? (float)(1 << (2 * grp)) : 1.f;
        v_group_epilogue(acc[ti], C, meta, w, xs, npair);
      }
    }
  }
  // combine the three limbs (lane t holds limb t), scale by 2^-e and S, store t
  const float lw = (float)(1 << (8 * min(t, 2)));
  const float* S = reinterpret_cast<const float*>(c.blob);
#pragma unroll
  for (int ti = 0; ti < DC_V_NT; ++ti)
#pragma unroll
    for (int pr = 0; pr < 2; ++pr)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v = t < 3 ? acc[ti][pr][q] * lw : 0.f;
        v += __shfl_xor_sync(FULLMASK, v, 1);
        v += __shfl_xor_sync(FULLMASK, v, 2);
        const int row = g + 8 * (q >> 1);
        const int tk = 2 * pr + (q & 1);
        const int rowb = 16 * (c.tile0 + ti) + row;
        if (t == 0 && ti < c.ntiles && row < rows[ti] && tk < c.ntok) {
          const int rank = B.r0 + rowb;
          const int tok = c.tok0 + tk;
          const int e = P.xe[c.m * T + tok];
          P.tws[((int64_t)c.p * T + tok) * F.ws.r_stride + rank] = ldexpf(v, -e) * S[rank];
        }
      }
}

__global__ void __launch_bounds__(256) k_vstage(const __grid_constant__ DcFwd F, uint8_t* ws) {
  WsPtr P = ws_ptr(F.ws, ws);
  const int lane = threadIdx.x & 31;
  const int nitems = P.st[DC_WS_NITEMS];
  for (;;) {
    int it = 0;
    if (lane == 0) it = atomicAdd(P.st + DC_WS_VCOUNTER, 1);
    it = __shfl_sync(FULLMASK, it, 0);
    if (it >= nitems) break;
    const DcVItem I = P.items[it];
    const int tau = P.segs[3 * I.seg], st = P.segs[3 * I.seg + 1], len = P.segs[3 * I.seg + 2];
    const DcLayout* L = P.layouts + I.p * F.ws.max_tenants + tau;
    VCtx c;
    c.blob = reinterpret_cast<const uint8_t*>(L->dev_base);
    c.L = L;
    c.band = I.band;
    c.tile0 = I.tile0;
    c.ntiles = I.ntiles;
    c.tok0 = st + DC_V_TOKS * I.pass;
    c.ntok = min(DC_V_TOKS, len - DC_V_TOKS * I.pass);
    c.m = F.lin[I.p].input;
    c.p = I.p;
    const int bits = L->band[I.band].bits;
    if (bits == 2)
      v_item<2>(F, P, c, lane);
    else if (bits == 3)
      v_item<3>(F, P, c, lane);
    else
      v_item<8>(F, P, c, lane);
  }
}

// ---------------------------------------------------------------------------------------------
// k_ustage: y = W_base x + sum over segments of U_hat (scale * t), one CTA per (linear, 128-row
// output tile, 64-token block); warp w owns rows 16w..16w+15 of the tile.
// ---------------------------------------------------------------------------------------------
#define U_KC 128
#define U_XROW (U_KC + 8)  // padded bf16 row of the staged activations

struct USmem {
  int exps[DC_V_TOKS];
  int zc[2][3][2];
  float red[8][DC_V_TOKS];
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ void u_base_bf16(const DcFwd& F, const DcLinDev& lin, const int* perm, int ot, int tb, int Tb,
                            __nv_bfloat16* xst, float (&acc)[8][4]) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 2, t = lane & 3;
  const int d_in = lin.d_in;
  const __nv_bfloat16* X = (const __nv_bfloat16*)F.x[lin.input];
  const __nv_bfloat16* Wm = (const __nv_bfloat16*)lin.W;
  const int row = ot * 128 + 16 * w + g;
  const __nv_bfloat16* wr0 = Wm + (int64_t)row * d_in + 8 * t;
  const __nv_bfloat16* wr1 = wr0 + (int64_t)8 * d_in;
  const int nkc = d_in / U_KC;
  const int ntv = (Tb + 7) >> 3;
  auto stage = [&](int kc, int buf) {
    __nv_bfloat16* dst = xst + buf * 64 * U_XROW;
    for (int idx = tid; idx < 64 * (U_KC / 8); idx += blockDim.x) {
      const int tok = idx / (U_KC / 8), cc = idx % (U_KC / 8);
      if (tok < Tb) cp_async16(dst + tok * U_XROW + 8 * cc, X + (int64_t)perm[tb + tok] * d_in + kc * U_KC + 8 * cc);
    }
    cp_async_commit();
  };
  stage(0, 0);
  for (int kc = 0; kc < nkc; ++kc) {
    uint4 wa[4], wb[4];
#pragma unroll
    for (int k32 = 0; k32 < 4; ++k32) {
      wa[k32] = ldg128(wr0 + kc * U_KC + 32 * k32);
      wb[k32] = ldg128(wr1 + kc * U_KC + 32 * k32);
    }
    if (kc + 1 < nkc) {
      stage(kc + 1, (kc + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16* xb = xst + (kc & 1) * 64 * U_XROW;
    // Each 128-column chunk is summed in a fresh MMA chain and added to the running sum with an
    // IEEE fp32 add, so the tensor core's internal accumulation rounding spans 8 steps, not d_in/16.
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      if (nt < ntv) {
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k32 = 0; k32 < 4; ++k32) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xb + (8 * nt + g) * U_XROW + 32 * k32 + 8 * t);
          mma_bf16(part, wa[k32].x, wb[k32].x, wa[k32].y, wb[k32].y, xv.x, xv.y);
          mma_bf16(part, wa[k32].z, wb[k32].z, wa[k32].w, wb[k32].w, xv.z, xv.w);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[nt][q] += part[q];
      }
    }
    __syncthreads();
  }
}

// fp32 backbone (small fp32 layers): plain FFMA in the same fragment layout.
__device__ void u_base_f32(const DcFwd& F, const DcLinDev& lin, const int* perm, int ot, int tb, int Tb,
                           float (&acc)[8][4]) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
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
      acc[nt][q] = s0;
      acc[nt][2 + q] = s1;
    }
  }
}

__global__ void __launch_bounds__(256, 2) k_ustage(const __grid_constant__ DcFwd F, uint8_t* ws) {
  extern __shared__ __align__(16) uint8_t usm[];
  WsPtr P = ws_ptr(F.ws, ws);
  int slot = 0;
  while (slot + 1 < F.n_lin && (int)blockIdx.x >= F.tile_prefix[slot + 1]) ++slot;
  const int p = F.order[slot];
  const int ot = blockIdx.x - F.tile_prefix[slot];
  const DcLinDev& lin = F.lin[p];
  const int T = F.ws.T;
  const int tb = blockIdx.y * DC_TOK_BLOCK;
  const int Tb = min(DC_TOK_BLOCK, T - tb);
  if (Tb <= 0) return;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 2, t = lane & 3;
  // shared memory: [x staging 2 x 64 x U_XROW bf16 | B staging 2 x 8 x bsm_max | yd 8x16x64 f32 | USmem]
  __nv_bfloat16* xst = reinterpret_cast<__nv_bfloat16*>(usm);
  uint8_t* bsm = usm + 2 * 64 * U_XROW * 2;
  float* yd = reinterpret_cast<float*>(bsm + 16 * F.bsm_max);
  USmem* us = reinterpret_cast<USmem*>(yd + 8 * 16 * DC_TOK_BLOCK);
  float* ydw = yd + w * 16 * DC_TOK_BLOCK;

  float acc[8][4];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[a][q] = 0.f;
  for (int i = tid; i < 8 * 16 * DC_TOK_BLOCK; i += blockDim.x) yd[i] = 0.f;
  if (F.flags & DC_BASE) {
    if (lin.w_dtype == DC_DTYPE_BF16)
      u_base_bf16(F, lin, P.perm, ot, tb, Tb, xst, acc);
    else
      u_base_f32(F, lin, P.perm, ot, tb, Tb, acc);
  }
  __syncthreads();

  if (F.flags & DC_DELTA) {
    const int nseg = P.st[DC_WS_NSEG];
    const int go = ot;  // 128-row output group = quantisation group of the U columns
    const int orow = ot * 128 + 16 * w;  // first row of this warp
    for (int s = 0; s < nseg; ++s) {
      const int tau = P.segs[3 * s], st = P.segs[3 * s + 1], len = P.segs[3 * s + 2];
      const int s0 = max(st, tb), s1 = min(st + len, tb + Tb);
      if (s0 >= s1 || tau >= lin.n_tenants || tau >= F.ws.max_tenants) continue;
      const DcLayout& L = P.layouts[p * F.ws.max_tenants + tau];
      if (!L.valid) continue;
      const uint8_t* blob = reinterpret_cast<const uint8_t*>(L.dev_base);
      const uint8_t* umeta = blob + L.u_meta_off + (int64_t)go * L.r * 4;
      for (int pt0 = s0; pt0 < s1; pt0 += DC_V_TOKS) {
        const int ntok = min(DC_V_TOKS, s1 - pt0);
        const int npair = (ntok + 1) >> 1;
        const float* tw = P.tws + ((int64_t)p * T + pt0) * F.ws.r_stride;
        // ---- B = scale * t: per-token exponent from the largest |B| (MMA bands only)
        float mx[DC_V_TOKS] = {0.f, 0.f, 0.f, 0.f};
        for (int b = 0; b < L.n_bands; ++b) {
          const DcBand& Bd = L.band[b];
          if (Bd.bits == 8) continue;
          for (int i = tid; i < Bd.rank; i += blockDim.x) {
            const int r = Bd.r0 + i;
            const float sc = __low2float(*reinterpret_cast<const __half2*>(umeta + 4 * r));
#pragma unroll
            for (int q = 0; q < DC_V_TOKS; ++q)
              if (q < ntok) mx[q] = fmaxf(mx[q], fabsf(sc * tw[(int64_t)q * F.ws.r_stride + r]));
          }
        }
#pragma unroll
        for (int q = 0; q < DC_V_TOKS; ++q) {
#pragma unroll
          for (int o = 16; o; o >>= 1) mx[q] = fmaxf(mx[q], __shfl_xor_sync(FULLMASK, mx[q], o));
          if (lane == 0) us->red[w][q] = mx[q];
        }
        for (int i = tid; i < 16 * F.bsm_max / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(bsm)[i] = 0u;
        if (tid < 12) (&us->zc[0][0][0])[tid] = 0;
        __syncthreads();
        if (tid < DC_V_TOKS) {
          float m = 0.f;
          for (int ww = 0; ww < 8; ++ww) m = fmaxf(m, us->red[ww][tid]);
          int e = 0;
          if (m > 0.f) {
            int E;
            frexpf(m, &E);
            e = 22 - E;
          }
          us->exps[tid] = e;
        }
        __syncthreads();
        // ---- limbs of B into the staging buffer; zero-point correction sums
        int zc[2][3][2];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int b = 0; b < 3; ++b) zc[a][b][0] = zc[a][b][1] = 0;
        for (int b = 0; b < L.n_bands; ++b) {
          const DcBand& Bd = L.band[b];
          if (Bd.bits == 8) continue;
          for (int i = tid; i < Bd.rank; i += blockDim.x) {
            const int r = Bd.r0 + i;
            const __half2 mz = *reinterpret_cast<const __half2*>(umeta + 4 * r);
            const float sc = __low2float(mz);
            const int z = (int)__high2float(mz);
#pragma unroll
            for (int q = 0; q < DC_V_TOKS; ++q) {
              if (q >= ntok) continue;
              const int bi = __float2int_rn(ldexpf(sc * tw[(int64_t)q * F.ws.r_stride + r], us->exps[q]));
              const int l0 = sext8(bi);
              const int x1 = (bi - l0) >> 8;
              const int l1 = sext8(x1);
              const int l2 = (x1 - l1) >> 8;
              const int pr = q >> 1, tk = q & 1;
              uint8_t* col = bsm + (int64_t)(pr * 8) * F.bsm_max + Bd.bsm_off + i;
              col[(0 * 2 + tk) * F.bsm_max] = (uint8_t)(l0 & 0xff);
              col[(1 * 2 + tk) * F.bsm_max] = (uint8_t)(l1 & 0xff);
              col[(2 * 2 + tk) * F.bsm_max] = (uint8_t)(l2 & 0xff);
              zc[pr][0][tk] += z * l0;
              zc[pr][1][tk] += z * l1;
              zc[pr][2][tk] += z * l2;
            }
          }
        }
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int b = 0; b < 3; ++b)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              int v = zc[a][b][k];
#pragma unroll
              for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(FULLMASK, v, o);
              if (lane == 0 && v != 0) atomicAdd(&us->zc[a][b][k], v);
            }
        __syncthreads();
        // ---- MMA over the rank steps of every 2/3-bit band
        int C[2][4][4];  // [pair][position][reg]
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int q = 0; q < 4; ++q) C[a][b][q] = 0;
        for (int b = 0; b < L.n_bands; ++b) {
          const DcBand& Bd = L.band[b];
          if (Bd.bits == 8) continue;
          const uint8_t* ub = blob + Bd.u_off + (int64_t)(ot * 8 + w) * Bd.u_otile_bytes;
          const uint8_t* bcol0 = bsm + (int64_t)g * F.bsm_max + Bd.bsm_off + 8 * t;
          const uint8_t* bcol1 = bcol0 + (int64_t)8 * F.bsm_max;
          for (int q = 0; q < Bd.u_quads; ++q) {
            const uint4 wq = ldg128(ub + 512 * q + 16 * lane);
#pragma unroll
            for (int ps = 0; ps < 4; ++ps) {
              const int step = 4 * q + ps;
              const uint2 b0 = *reinterpret_cast<const uint2*>(bcol0 + 32 * step);
              const uint32_t a0 = u_reg_mask2(wq.x, ps), a1 = u_reg_mask2(wq.y, ps);
              const uint32_t a2 = u_reg_mask2(wq.z, ps), a3 = u_reg_mask2(wq.w, ps);
              mma_u8s8(C[0][ps], a0, a1, a2, a3, b0.x, b0.y);
              if (npair > 1) {
                const uint2 b1 = *reinterpret_cast<const uint2*>(bcol1 + 32 * step);
                mma_u8s8(C[1][ps], a0, a1, a2, a3, b1.x, b1.y);
              }
            }
          }
          const uint8_t* sb = ub + (int64_t)512 * Bd.u_quads;
          for (int sidx = 0; sidx < Bd.u_steps; ++sidx) {
            const int valid = (sidx == Bd.u_steps - 1) ? Bd.u_last : 32;
            const int nl = dc_u_step_lanes(valid);
            const int ntv = nl / 8;
            uint32_t wv = 0, hv = 0;
            if (t < ntv) {
              wv = ldg32(sb + 4 * (g * ntv + t));
              if (Bd.bits == 3) hv = ldg16(sb + dc_align((int64_t)nl * 4, 16) + 2 * (g * ntv + t));
            }
            uint32_t a[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              a[j] = reg_shift2(wv, j);
              if (Bd.bits == 3) a[j] |= u_reg_hi3(hv, j);
            }
            const int step = 4 * Bd.u_quads + sidx;
            const uint2 b0 = *reinterpret_cast<const uint2*>(bcol0 + 32 * step);
            mma_u8s8(C[0][0], a[0], a[1], a[2], a[3], b0.x, b0.y);
            if (npair > 1) {
              const uint2 b1 = *reinterpret_cast<const uint2*>(bcol1 + 32 * step);
              mma_u8s8(C[1][0], a[0], a[1], a[2], a[3], b1.x, b1.y);
            }
            sb += dc_u_step_bytes(Bd.bits, nl);
          }
        }
        // ---- combine positions and limbs; lane t holds limb t of columns (tok 0, tok 1) of a pair
        const float lw = (float)(1 << (8 * min(t, 2)));
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
          if (pr >= npair) continue;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int tk = q & 1;
            int cl = C[pr][0][q] + (C[pr][1][q] >> 2) + (C[pr][2][q] >> 4) + (C[pr][3][q] >> 6);
            float v = 0.f;
            if (t < 3) v = (float)(cl - us->zc[pr][t][tk]) * lw;
            v += __shfl_xor_sync(FULLMASK, v, 1);
            v += __shfl_xor_sync(FULLMASK, v, 2);
            const int qq = 2 * pr + tk;
            if (t == 0 && qq < ntok) {
              const int row = g + 8 * (q >> 1);
              ydw[row * DC_TOK_BLOCK + (pt0 - tb) + qq] += ldexpf(v, -us->exps[qq]);
            }
          }
        }
        __syncwarp();
        // ---- 8-bit bands: scalar path, lane -> (row = lane & 15, token parity = lane >> 4)
        for (int b = 0; b < L.n_bands; ++b) {
          const DcBand& Bd = L.band[b];
          if (Bd.bits != 8) continue;
          const int row = lane & 15;
          const uint8_t* ur = blob + Bd.u_off + (int64_t)(orow + row) * Bd.rank;
          for (int q = lane >> 4; q < ntok; q += 2) {
            float sum = 0.f;
            for (int i = 0; i < Bd.rank; ++i) {
              const int r = Bd.r0 + i;
              const __half2 mz = *reinterpret_cast<const __half2*>(umeta + 4 * r);
              const float code = (float)ur[i];
              sum = fmaf((code - __high2float(mz)) * __low2float(mz), tw[(int64_t)q * F.ws.r_stride + r], sum);
            }
            ydw[row * DC_TOK_BLOCK + (pt0 - tb) + q] += sum;
          }
        }
        __syncthreads();
      }
    }
  }
  __syncwarp();
  // ---- output in the tokens' original order
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int tok = 8 * nt + 2 * t + (q & 1);
      const int row = g + 8 * (q >> 1);
      if (tok < Tb) {
        const float v = acc[nt][q] + ydw[row * DC_TOK_BLOCK + tok];
        const int dst = P.perm[tb + tok];
        const int64_t o = (int64_t)dst * lin.d_out + ot * 128 + 16 * w + row;
        if (F.dtype_out == DC_DTYPE_F32)
          reinterpret_cast<float*>(lin.y)[o] = v;
        else
          reinterpret_cast<__nv_bfloat16*>(lin.y)[o] = __float2bfloat16_rn(v);
      }
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
  const uint8_t* blk = blob + B.v_off + (int64_t)tile * B.v_tile_bytes + (int64_t)kb * dc_v_block_bytes(B.bits, rows, 4) +
                       dc_v_half_off(B.bits, rows, ngrp, h);
  const int p0 = dc_v_plane0_bytes(B.bits, ngrp);
  const int rank = B.r0 + 16 * tile + 8 * h + g;
  for (int grp = 0; grp < ngrp; ++grp)
    for (int s = 0; s < 4; ++s)
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r;
        if (B.bits == 2 && ngrp == 4) {
          const uint4 q = ldg128(blk + lane * 32 + 16 * (s >> 1));
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
  if (B.bits == 8) {
    if (id >= (int64_t)L.d_out * B.rank) return;
    const int o = (int)(id / B.rank), i = (int)(id % B.rank);
    out[(int64_t)(B.r0 + i) * L.d_out + o] = blob[B.u_off + id];
    return;
  }
  if (id >= (int64_t)(L.d_out / 16) * 32) return;
  const int lane = (int)(id & 31), ot = (int)(id >> 5);
  const int g = lane >> 2, t = lane & 3;
  const uint8_t* ub = blob + B.u_off + (int64_t)ot * B.u_otile_bytes;
  auto put = [&](uint32_t reg, int j, int rank_base) {
    for (int b = 0; b < 4; ++b) {
      const int rank = rank_base + 8 * t + 4 * (j >> 1) + b;
      if (rank < B.rank) out[(int64_t)(B.r0 + rank) * L.d_out + 16 * ot + g + 8 * (j & 1)] = (uint8_t)(reg >> (8 * b));
    }
  };
  for (int q = 0; q < B.u_quads; ++q) {
    const uint4 wq = ldg128(ub + 512 * q + 16 * lane);
    for (int ps = 0; ps < 4; ++ps)
      for (int j = 0; j < 4; ++j) put(u_reg_mask2(wsel(wq, j), ps) >> (2 * ps), j, 128 * q + 32 * ps);
  }
  const uint8_t* sb = ub + (int64_t)512 * B.u_quads;
  for (int s = 0; s < B.u_steps; ++s) {
    const int valid = (s == B.u_steps - 1) ? B.u_last : 32;
    const int nl = dc_u_step_lanes(valid), ntv = nl / 8;
    if (t < ntv) {
      const uint32_t wv = ldg32(sb + 4 * (g * ntv + t));
      const uint32_t hv = B.bits == 3 ? ldg16(sb + dc_align((int64_t)nl * 4, 16) + 2 * (g * ntv + t)) : 0u;
      for (int j = 0; j < 4; ++j) {
        uint32_t r = reg_shift2(wv, j);
        if (B.bits == 3) r |= u_reg_hi3(hv, j);
        put(r, j, 128 * B.u_quads + 32 * s);
      }
    }
    sb += dc_u_step_bytes(B.bits, nl);
  }
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

extern "C" size_t dc_quantize_scratch_size(const dc_factor_desc* desc) {
  DcLayout L;
  if (dc_check_desc(desc, &L) != DC_OK) return 0;
  return (size_t)(256 + dc_align((int64_t)L.r * L.d_out, 256) + dc_align((int64_t)L.r * L.d_in, 256) +
                  dc_align((int64_t)L.r * L.groups_out * 4, 256) + dc_align((int64_t)L.r * L.groups_in * 4, 256));
}

extern "C" dc_status dc_quantize_pack_device(const dc_factor_desc* desc, const float* U_dev, const float* Vt_dev,
                                             const float* S_dev, void* dev_dst, size_t dev_bytes, void* scratch,
                                             size_t scratch_bytes, void* stream, dc_delta_handle* out) {
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
  DcPlain Pl{cu, cv, szu, szv, S_dev};
  const int64_t nw = L.bytes / 4;
  const unsigned blocks = (unsigned)std::min<int64_t>((nw + 255) / 256, 148 * 64);
  k_pack_words<<<blocks, 256, 0, s>>>(L, Pl, (uint32_t*)dev_dst);
  st = dc_cuda_check(cudaGetLastError(), "pack kernel");
  if (st) return st;
  dc_fill_handle(desc, L, dev_dst, out);
  return DC_OK;
}

extern "C" dc_status dc_build_segments(const int32_t* tenant_ids_dev, int32_t T, int32_t n_tenants, void* ws,
                                       size_t ws_bytes, void* stream) {
  dc_clear_error();
  if (T < 0 || n_tenants < 0) return dc_fail(DC_ERR_INVALID_ARG, "negative T or tenant count");
  if (n_tenants > DC_MAX_TENANTS) return dc_fail(DC_ERR_UNSUPPORTED, "at most %d tenants per call", DC_MAX_TENANTS);
  if (!ws || (T > 0 && !tenant_ids_dev)) return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(ws)) return dc_fail(DC_ERR_ALIGN, "workspace must be 16-byte aligned");
  const DcWs W = dc_ws_layout(T, 0, 0, 1, 0);
  if (ws_bytes < (size_t)W.total) return dc_fail(DC_ERR_WORKSPACE, "workspace too small for routing");
  const size_t smem = (size_t)2 * (n_tenants + 1) * 4;
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(k_segments, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  k_segments<<<1, 256, smem, (cudaStream_t)stream>>>(tenant_ids_dev, T, n_tenants, (uint8_t*)ws, W);
  return dc_cuda_check(cudaGetLastError(), "routing kernel");
}

extern "C" dc_status dc_read_segments(const void* ws, int32_t T, int32_t* perm_dev, int32_t* inv_perm_dev,
                                      int32_t* segments_dev, int32_t* n_segments_dev, void* stream) {
  dc_clear_error();
  if (!ws || T < 0) return dc_fail(DC_ERR_INVALID_ARG, "bad arguments");
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
  int max_rank = 0, max_d_in = 0, max_ten = 0, bsm_max = 32;
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
    if (l.w_dtype != DC_DTYPE_BF16 && l.w_dtype != DC_DTYPE_F32) return dc_fail(DC_ERR_INVALID_ARG, "linear %d: w_dtype", p);
    if (l.w_dtype == DC_DTYPE_BF16 && dtype_in != DC_DTYPE_BF16 && (flags & DC_BASE))
      return dc_fail(DC_ERR_UNSUPPORTED, "linear %d: bf16 weights need bf16 activations", p);
    if (l.n_tenants < 0 || l.n_tenants > DC_MAX_TENANTS) return dc_fail(DC_ERR_INVALID_ARG, "linear %d: tenant count", p);
    if ((flags & DC_DELTA) && l.n_tenants > 0 && !l.tenants_dev) return dc_fail(DC_ERR_INVALID_ARG, "linear %d: null tenant table", p);
    if (l.max_rank < 0 || l.max_rank > std::min(l.d_out, l.d_in)) return dc_fail(DC_ERR_SHAPE, "linear %d: max_rank", p);
    max_rank = std::max(max_rank, l.max_rank);
    max_ten = std::max(max_ten, l.n_tenants);
    bsm_max = std::max(bsm_max, (int)dc_align(l.max_rank, 32) + 32 * DC_MAX_BANDS);
    F.lin[p].W = l.W_base;
    F.lin[p].tenants = l.tenants_dev;
    F.lin[p].y = ys[p];
    F.lin[p].d_out = l.d_out;
    F.lin[p].d_in = l.d_in;
    F.lin[p].n_tenants = l.n_tenants;
    F.lin[p].w_dtype = l.w_dtype;
    F.lin[p].input = m;
  }
  F.bsm_max = bsm_max;
  F.ws = dc_ws_layout(T, max_rank, max_d_in, n_lin, max_ten);
  if (ws_bytes < (size_t)F.ws.total)
    return dc_fail(DC_ERR_WORKSPACE, "workspace holds %zu bytes, need %lld", ws_bytes, (long long)F.ws.total);
  // U-kernel order: largest output tiles first (d_in decides the bytes per tile)
  int ord[7];
  for (int p = 0; p < n_lin; ++p) ord[p] = p;
  std::stable_sort(ord, ord + n_lin, [&](int a, int b) { return lins[a].d_in > lins[b].d_in; });
  F.tile_prefix[0] = 0;
  for (int i = 0; i < n_lin; ++i) {
    F.order[i] = ord[i];
    F.tile_prefix[i + 1] = F.tile_prefix[i] + lins[ord[i]].d_out / 128;
  }
  cudaStream_t s = (cudaStream_t)stream;
  dc_status st;
  if (!(flags & DC_REUSE_ROUTING)) {
    if (max_ten > DC_MAX_TENANTS) return dc_fail(DC_ERR_UNSUPPORTED, "too many tenants");
    const size_t smem = (size_t)2 * (max_ten + 1) * 4;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k_segments, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    prof_before(s, 0);
    k_segments<<<1, 256, smem, s>>>(ids, T, max_ten, (uint8_t*)ws, F.ws);
    prof_after(s);
    st = dc_cuda_check(cudaGetLastError(), "routing kernel");
    if (st) return st;
  }
  prof_before(s, 1);
  k_prep<<<dim3(T + 1, n_in), 256, 0, s>>>(F, (uint8_t*)ws);
  prof_after(s);
  st = dc_cuda_check(cudaGetLastError(), "prep kernel");
  if (st) return st;
  if (flags & DC_DELTA) {
    static int n_sm = 0;
    if (!n_sm) {
      int dev = 0;
      cudaGetDevice(&dev);
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
      if (n_sm <= 0) n_sm = 148;
    }
    prof_before(s, 2);
    k_vstage<<<n_sm * 4, 256, 0, s>>>(F, (uint8_t*)ws);
    prof_after(s);
    st = dc_cuda_check(cudaGetLastError(), "rank-reduction kernel");
    if (st) return st;
  }
  const size_t usmem = (size_t)2 * 64 * U_XROW * 2 + (size_t)16 * bsm_max + (size_t)8 * 16 * DC_TOK_BLOCK * 4 + sizeof(USmem);
  static size_t usmem_set = 0;
  if (usmem > usmem_set) {
    st = dc_cuda_check(cudaFuncSetAttribute(k_ustage, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)usmem), "smem attr");
    if (st) return st;
    usmem_set = usmem;
  }
  const dim3 ugrid(F.tile_prefix[n_lin], (T + DC_TOK_BLOCK - 1) / DC_TOK_BLOCK);
  prof_before(s, 3);
  k_ustage<<<ugrid, 256, usmem, s>>>(F, (uint8_t*)ws);
  prof_after(s);
  return dc_cuda_check(cudaGetLastError(), "output kernel");
}

extern "C" dc_status dc_delta_linear_segmented(const dc_linear* lin, const void* x, void* y, const int32_t* tenant_ids_dev,
                                               int32_t T, int32_t dtype_in, int32_t dtype_out, int32_t flags, void* ws,
                                               size_t ws_bytes, void* stream) {
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
  dc_clear_error();
  if (!lin || !y) return dc_fail(DC_ERR_INVALID_ARG, "null linear array or outputs");
  const void* xs[3] = {x_h, x_o, x_f};
  const int dx[3] = {lin[0].d_in, lin[3].d_in, lin[6].d_in};
  return run_forward(lin, 7, xs, dx, y, tenant_ids_dev, T, dtype_in, dtype_out, flags, ws, ws_bytes, stream);
}

extern "C" dc_status dc_unpack_codes_debug(const dc_delta_handle* h, int32_t which, uint8_t* out_dev, void* stream) {
  dc_clear_error();
  if (!h || !out_dev || h->dev_base == 0) return dc_fail(DC_ERR_INVALID_ARG, "bad handle or output");
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
      const int64_t n = B.bits == 8 ? (int64_t)L.d_out * B.rank : (int64_t)(L.d_out / 16) * 32;
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
  dc_clear_error();
  if (!ws || !host_status) return dc_fail(DC_ERR_INVALID_ARG, "null pointer");
  cudaStream_t s = (cudaStream_t)stream;
  int32_t v = 0;
  dc_status st = dc_cuda_check(cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, s), "status read");
  if (st) return st;
  st = dc_cuda_check(cudaStreamSynchronize(s), "status sync");
  if (st) return st;
  *host_status = v;
  return dc_cuda_check(cudaMemsetAsync(ws, 0, 4, s), "status clear");
}
