// Packing of plain codes into the serving layout (dc_layout.h), one 32-bit word at a time.
//
// The same word function serves the host packer (a loop over every word of the blob) and the
// device packer (one thread per word), so both produce identical bytes.
#pragma once
#include "dc_layout.h"

// Plain (unpacked) quantisation result of one tenant's linear.
struct DcPlain {
  const uint8_t* cu;    // [r][d_out]  codes of u_i (row i)
  const uint8_t* cv;    // [r][d_in]   codes of v_i
  const uint16_t* szu;  // [r][d_out/128][2] fp16 (scale, zero)
  const uint16_t* szv;  // [r][d_in/128][2]
  const float* S;       // [r]
  float umax;           // largest U scale over the 2/3-bit bands and every output group
};


DC_HD int64_t dc_v_band_bytes(const DcLayout& L, const DcBand& B) {
  int32_t last_rows = B.rank - 16 * (B.v_tiles - 1);
  return B.v_tile_bytes * (B.v_tiles - 1) + dc_v_block_bytes(B.bits, last_rows, L.groups_in);
}

DC_HD uint32_t dc_cv(const DcLayout& L, const DcPlain& P, int32_t rank, int32_t k) {
  return P.cv[(int64_t)rank * L.d_in + k];
}
DC_HD uint32_t dc_cu(const DcLayout& L, const DcPlain& P, int32_t rank, int32_t o) {
  return P.cu[(int64_t)rank * L.d_out + o];
}

// Word at byte offset `off` (a multiple of 4) inside the V codes of band B.
DC_HD uint32_t dc_pack_v_word(const DcLayout& L, const DcBand& B, int64_t off, const DcPlain& P) {
  const int32_t bits = B.bits;
  const int64_t gbytes = (int64_t)B.v_group * B.v_tile_bytes;  // a full group
  const int32_t ngroups = (B.v_tiles + B.v_group - 1) / B.v_group;
  int32_t grp = (int32_t)(off / gbytes);
  if (grp > ngroups - 1) grp = ngroups - 1;
  const int64_t in_g = off - (int64_t)grp * gbytes;
  const int64_t f4 = dc_v_group_block_bytes(B, grp, 4);
  int32_t kb = (int32_t)(in_g / f4);
  if (kb > L.nkb - 1) kb = L.nkb - 1;
  const int64_t in_kb = in_g - (int64_t)kb * f4;
  const int32_t ngrp = (kb == L.nkb - 1) ? L.tail_groups : 4;
  const int64_t tb16 = dc_v_block_bytes(bits, 16, ngrp);
  int32_t ti = (int32_t)(in_kb / tb16);
  const int32_t nt = dc_v_group_ntiles(B, grp);
  if (ti > nt - 1) ti = nt - 1;
  const int64_t in_blk = in_kb - (int64_t)ti * tb16;
  const int32_t j = grp * B.v_group + ti;
  const int32_t rows = dc_v_tile_rows(B, j);
  const int64_t cb = dc_v_block_code_bytes(bits, rows, ngrp);
  if (in_blk >= cb) {  // inline meta: entry (group, g, half)
    const int64_t e = (in_blk - cb) / 4;
    const int32_t h = (int32_t)(e & 1), g = (int32_t)((e >> 1) & 7), cg = (int32_t)(e >> 4);
    const int32_t row = 16 * j + 8 * h + g;
    if (row >= B.rank || cg >= ngrp) return 0u;
    const uint16_t* sz = P.szv + ((int64_t)(B.r0 + row) * L.groups_in + 4 * kb + cg) * 2;
    return (uint32_t)sz[0] | ((uint32_t)sz[1] << 16);
  }
  const int64_t h1 = dc_v_half_off(bits, rows, ngrp, 1);
  const int32_t h = (rows > 8 && in_blk >= h1) ? 1 : 0;
  const int64_t in_half = in_blk - (h ? h1 : 0);
  const int32_t nh = h == 0 ? (rows < 8 ? rows : 8) : rows - 8;
  const int32_t nl = 4 * nh;
  const int32_t p0 = dc_v_plane0_bytes(bits, ngrp);
  int32_t plane, lane, wi;
  if (bits == 2 && ngrp == 4) {  // mask layout: words 0-3 of every lane, then words 4-7
    plane = 0;
    const int32_t hi = (int32_t)(in_half / (16 * nl));
    const int32_t within = (int32_t)(in_half % (16 * nl));
    lane = within / 16;
    wi = 4 * hi + (within % 16) / 4;
  } else if (in_half < (int64_t)nl * p0) {
    plane = 0;
    lane = (int32_t)(in_half / p0);
    wi = (int32_t)((in_half % p0) / 4);
  } else {
    plane = 1;
    const int64_t x = in_half - (int64_t)nl * p0;
    const int32_t p1 = 4 * ngrp;
    lane = (int32_t)(x / p1);
    wi = (int32_t)((x % p1) / 4);
  }
  if (lane >= nl) return 0u;
  const int32_t g = lane >> 2, t = lane & 3;
  const int32_t rank = B.r0 + 16 * j + 8 * h + g;
  const int32_t kbase = 512 * kb;
  uint32_t w = 0;
  if (bits == 8) {
    const int32_t grp = wi >> 3, ww = wi & 7, s = ww >> 1, hh = ww & 1;
    for (int b = 0; b < 4; ++b)
      w |= dc_cv(L, P, rank, kbase + 128 * grp + 32 * t + 8 * s + 4 * hh + b) << (8 * b);
  } else if (bits == 2 && ngrp == 4) {  // mask layout
    const int32_t s = wi >> 1, hh = wi & 1;
    for (int p = 0; p < 4; ++p)
      for (int b = 0; b < 4; ++b)
        w |= (dc_cv(L, P, rank, kbase + 128 * p + 32 * t + 8 * s + 4 * hh + b) & 3u) << (8 * b + 2 * p);
  } else if (plane == 0) {  // shift layout, 2 words per group
    const int32_t grp = wi >> 1, hs = wi & 1;
    for (int s2 = 0; s2 < 2; ++s2)
      for (int hh = 0; hh < 2; ++hh)
        for (int b = 0; b < 4; ++b) {
          const int32_t s = 2 * hs + s2, q = 2 * s2 + hh;
          w |= (dc_cv(L, P, rank, kbase + 128 * grp + 32 * t + 8 * s + 4 * hh + b) & 3u) << (8 * b + 2 * q);
        }
  } else {  // 3-bit high plane, one word per group
    const int32_t grp = wi;
    for (int s = 0; s < 4; ++s)
      for (int hh = 0; hh < 2; ++hh)
        for (int b = 0; b < 4; ++b)
          w |= ((dc_cv(L, P, rank, kbase + 128 * grp + 32 * t + 8 * s + 4 * hh + b) >> 2) & 1u)
               << (8 * b + 2 * s + hh);
  }
  return w;
}

// Word at byte offset `off` inside band B's part of the 128-row group `go`'s run.
DC_HD uint32_t dc_pack_u_word(const DcLayout& L, const DcBand& B, int32_t go, int64_t off, const DcPlain& P) {
  int32_t k = (int32_t)(off / B.u_full);
  if (k > B.u_nblk - 1) k = B.u_nblk - 1;
  const DcUBlk K = dc_u_block(B, k);
  const int64_t lo = off - (int64_t)k * B.u_full;
  if (lo >= K.code_bytes) {  // meta of the block's ranks
    const int32_t i = (int32_t)((lo - K.code_bytes) / 4);
    if (i >= K.nr) return 0u;
    const uint16_t* sz = P.szu + ((int64_t)(B.r0 + K.rr0 + i) * L.groups_out + go) * 2;
    return (uint32_t)sz[0] | ((uint32_t)sz[1] << 16);
  }
  uint32_t w = 0;
  if (B.bits == 8) {  // row-major 128 x nr
    for (int b = 0; b < 4; ++b) {
      const int64_t idx = lo + b;
      const int64_t o = idx / K.nr;
      const int32_t i = (int32_t)(idx % K.nr);
      if (o < 128) w |= dc_cu(L, P, B.r0 + K.rr0 + i, (int32_t)(128 * go + o)) << (8 * b);
    }
    return w;
  }
  const int32_t ot = (int32_t)(lo / K.tile_bytes);  // 16-row tile inside the group
  int64_t x = lo - (int64_t)ot * K.tile_bytes;
  const int32_t o0 = 128 * go + 16 * ot;
  if (x < (int64_t)512 * K.nq) {  // mask layout quads
    const int32_t q = K.q0 + (int32_t)(x / 512);
    const int32_t y = (int32_t)(x % 512);
    const int32_t lane = y / 16, j = (y % 16) / 4;
    const int32_t g = lane >> 2, t = lane & 3;
    const int32_t o = o0 + g + 8 * (j & 1);
    for (int p = 0; p < 4; ++p)
      for (int b = 0; b < 4; ++b) {
        const int32_t rank = 128 * q + 32 * p + 8 * t + 4 * (j >> 1) + b;
        if (rank < B.rank) w |= (dc_cu(L, P, B.r0 + rank, o) & 3u) << (8 * b + 2 * p);
      }
    return w;
  }
  x -= (int64_t)512 * K.nq;
  for (int s = K.s0; s < K.s0 + K.ns; ++s) {
    const int32_t valid = (s == B.u_steps - 1) ? B.u_last : 32;
    const int32_t nl = dc_u_step_lanes(valid);
    const int32_t ntv = nl / 8;
    const int64_t sb = dc_u_step_bytes(B.bits, nl);
    if (x >= sb) {
      x -= sb;
      continue;
    }
    const int32_t rank_base = 128 * B.u_quads + 32 * s;
    const int64_t r2 = dc_align((int64_t)nl * 4, 16);
    if (x < r2) {
      const int32_t idx = (int32_t)(x / 4);
      if (idx >= nl) return 0u;
      const int32_t g = idx / ntv, t = idx % ntv;
      for (int jj = 0; jj < 4; ++jj)
        for (int b = 0; b < 4; ++b) {
          const int32_t rank = rank_base + 8 * t + 4 * (jj >> 1) + b;
          if (rank < B.rank) w |= (dc_cu(L, P, B.r0 + rank, o0 + g + 8 * (jj & 1)) & 3u) << (8 * b + 2 * jj);
        }
      return w;
    }
    const int64_t y = x - r2;  // 3-bit high plane: 2 bytes per lane
    for (int half = 0; half < 2; ++half) {
      const int32_t idx = (int32_t)(y / 2) + half;
      if (idx >= nl) continue;
      const int32_t g = idx / ntv, t = idx % ntv;
      uint32_t hb = 0;
      for (int jj = 0; jj < 4; ++jj)
        for (int b = 0; b < 4; ++b) {
          const int32_t rank = rank_base + 8 * t + 4 * (jj >> 1) + b;
          if (rank < B.rank) hb |= ((dc_cu(L, P, B.r0 + rank, o0 + g + 8 * (jj & 1)) >> 2) & 1u) << (4 * jj + b);
        }
      w |= hb << (16 * half);
    }
    return w;
  }
  return 0u;
}

DC_HD uint32_t dc_f32_bits(float f) {
  uint32_t u;
#if defined(__CUDA_ARCH__)
  u = __float_as_uint(f);
#else
  __builtin_memcpy(&u, &f, 4);
#endif
  return u;
}

// Word at byte offset `off` of the whole blob.
DC_HD uint32_t dc_pack_word(const DcLayout& L, int64_t off, const DcPlain& P) {
  if (off < (int64_t)L.r * 4) return dc_f32_bits(P.S[off / 4]);
  if (off == L.umax_off) return dc_f32_bits(P.umax);
  for (int i = 0; i < L.n_bands; ++i) {
    const DcBand& B = L.band[i];
    if (off >= B.v_off && off < B.v_off + dc_v_band_bytes(L, B)) return dc_pack_v_word(L, B, off - B.v_off, P);
  }
  if (off >= L.u_off && off < L.u_off + L.u_unit * L.groups_out) {
    const int64_t rel = off - L.u_off;
    const int32_t go = (int32_t)(rel / L.u_unit);
    const int64_t in = rel - (int64_t)go * L.u_unit;
    for (int i = 0; i < L.n_bands; ++i) {
      const DcBand& B = L.band[i];
      if (in >= B.u_boff && in < B.u_boff + B.u_bytes) return dc_pack_u_word(L, B, go, in - B.u_boff, P);
    }
  }
  return 0u;
}
