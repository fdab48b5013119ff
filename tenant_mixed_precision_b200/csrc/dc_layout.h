// Packed serving layout of one tenant's delta (host packer and device kernels share it).
//
// A tenant's delta for one linear is Delta_hat = U_hat diag(S) V_hat^T with ranks split into
// bands of equal bit width in descending singular-value order (the 8/3/2/0-bit groups of
// "Delta-CoMe: Training-Free Delta-Compression with Mixed-Precision for Large Language Models",
// section "Approach").  Each kept vector is quantised in groups of 128 with an fp16 scale and
// zero per group.  The blob is laid out for the two serving kernels, which stream it through
// shared memory with 1-D bulk copies (every region below starts on 16 bytes and is a multiple of
// 16 bytes long):
//
//   [S fp32 r] [V codes + V meta, band by band] [U runs: one per 128-row output group]
//
// V side (rank reduction t = S * (V_hat^T x)): the kernel's MMA tile is 16 ranks x 32 columns of
// d_in (mma.m16n8k32, u8 codes).  Ranks of a band are cut into tiles of 16 (the last may be
// partial); rows of a tile are in two halves (rows 0-7, rows 8-15); d_in is cut into blocks of
// 4 groups (512 columns, the last block may hold fewer groups).  Within a block a lane
// (g = lane/4, t = lane%4) of a half owns row g of the half, and within each group the 32
// columns 32t .. 32t+31; the column of MMA step s (0..3), k-half hh (0/1) and byte b is
// 32t + 8s + 4hh + b (the B operand uses the same permutation, so activations stay in natural
// order).  A (tile, block) region is [half 0 planes][half 1 planes][meta of the block's groups].
// Tiles are gathered in groups of 8 (2-bit), 5 (3-bit) or 2 (8-bit) tiles -- one serving work
// item -- stored block-major: [group][block][tile][(tile, block) region], so that one block of
// every tile of a group is one contiguous run of bytes.
// Storage per (tile, block, half): one array per bit plane, lanes in order, only the lanes of
// valid rows (4 per row) present:
//   2-bit, full block : 8 words per lane; word 2s+hh, bits [8b+2p, 8b+2p+2) hold the code of
//                       group p (p = 0..3) -- a register is extracted with one AND and carries
//                       the weight 4^p, removed in the fp32 epilogue ("mask" layout); words 0-3
//                       of every lane come first, then words 4-7 of every lane (dc_v_mask_off);
//   2-bit, tail block : 2 words per group; word s/2, bits [8b+2q, 8b+2q+2), q = 2(s%2)+hh
//                       ("shift" layout);
//   3-bit             : the 2-bit plane in the shift layout plus a 1-bit plane of one word per
//                       group, bit 8b + 2s + hh = bit 2 of the code;
//   8-bit             : 8 words per group, word 2s+hh byte b = the code.
// V meta (inside the block, after the codes): per (group, g, half) the fp16 pair (scale, zero) of
// row g + 8*half: 64 bytes per group, rows past the band padded with zeros.
//
// U side (y += U_hat * B with B = scale * t): the MMA tile is 16 output rows x 32 ranks.  A band
// of 2 or 3 bits is cut into steps of 32 ranks; lane (g, t) owns rows g and g+8 and, within a
// step, ranks 8t .. 8t+7: register j (a0..a3) is row g + 8*(j&1), ranks 8t + 4*(j>>1) + b.
//   2-bit, full quad of 4 steps : 4 words per lane; word j, bits [8b+2p, 8b+2p+2) = step p
//                                 (mask layout, weight 4^p);
//   other steps (2-bit leftovers, every 3-bit step): one word per lane (shift layout: register
//                                 j = bits [8b+2j, 8b+2j+2)); for 3 bits also a 1-bit plane of
//                                 2 bytes per lane, bit 4j+b = bit 2 of the code of register j
//                                 byte b;
//   the last step of a band may be partial: only lanes with 8t < valid ranks are stored
//   (ranks inside a lane padded to 8 with code 0).
// The U side is grouped by 128-row output group (= the quantisation group along d_out): the run
// of group go holds every band's codes and meta for its 128 rows, and is one contiguous run of
// bytes.  Inside the run each band is cut into blocks of at most 8 steps (256 ranks): a 2-bit
// band into blocks of 2 quads plus one tail block (a leftover quad and the shift-layout steps),
// a 3-bit band into blocks of 8 steps, an 8-bit band into blocks of 64 ranks.  A block is
//   [tile 0 codes][tile 1 codes] ... [tile 7 codes][meta: nr fp16 pairs (scale, zero)]
// for 2/3-bit bands (a tile = the 16-row MMA tile: the block's quads, then its shift steps) and
//   [128 rows x nr code bytes, row-major][meta]
// for 8-bit bands (a scalar path).  Every block but a band's last has the band's full-block
// size, so block k of a band starts at k * full_bytes.  One block is one bulk copy.
// After S (fp32, r entries, padded to r4 = r rounded up to 4) the blob holds one fp32: the
// largest U scale over the 2/3-bit bands and every output group (a bound used to pick the
// fixed-point exponent of scale * t without a pass over the data).
#pragma once
#include <stdint.h>

#include "dc.h"

#if defined(__CUDACC__)
#define DC_HD __host__ __device__ __forceinline__
#else
#define DC_HD inline
#endif

struct DcBand {
  int32_t bits;        // 2, 3 or 8
  int32_t rank;        // ranks in the band
  int32_t r0;          // first rank of the band (index into S, t and U meta)
  int32_t v_tiles;     // ceil(rank / 16)
  int32_t v_group;     // tiles per group (8, 5 or 2)
  int32_t u_quads;     // U: full 4-step quads in the mask layout (2-bit only)
  int32_t u_steps;     // U: steps in the shift layout after the quads (incl. a partial last one)
  int32_t u_last;      // U: valid ranks of the last shift-layout step (32 if it is full)
  int32_t u_nblk;      // U: blocks of the band inside one 128-row group's run
  int32_t u_full;      // U: bytes of a full block (every block but the last)
  int64_t v_off;       // V codes of the band
  int64_t v_tile_bytes;// bytes of one full 16-row tile (codes and meta of every block)
  int64_t u_boff;      // offset of the band inside one 128-row group's run
  int64_t u_bytes;     // bytes of the band inside one 128-row group's run
};

struct DcLayout {
  int32_t d_out, d_in, n_bands, r;
  int32_t groups_in;   // d_in / 128
  int32_t groups_out;  // d_out / 128
  int32_t nkb;         // ceil(groups_in / 4) blocks of 512 columns
  int32_t tail_groups; // groups in the last block (1..4)
  int32_t valid;       // 1 if the descriptor is valid
  int32_t r4;          // r rounded up to a multiple of 4
  int64_t s_off, bytes;
  int64_t umax_off;    // fp32 bound on the U scales of the 2/3-bit bands
  int64_t u_off;       // start of the U part (128-row group runs)
  int64_t u_unit;      // bytes of one 128-row group's run
  int64_t dev_base;    // device address of the blob (filled where a layout is bound to a blob)
  DcBand band[DC_MAX_BANDS];
};

// Geometry of block k of a band's U codes inside a 128-row group's run.
struct DcUBlk {
  int32_t nq, q0;      // quads (mask layout) in the block and the band's first one among them
  int32_t ns, s0;      // shift-layout steps in the block and the band's first one among them
  int32_t last;        // valid ranks of the block's final shift step (32 if full or none)
  int32_t nr;          // valid ranks of the block
  int32_t rr0;         // first rank of the block inside the band
  int32_t tile_bytes;  // bytes of one 16-row tile (2/3-bit bands)
  int32_t code_bytes;  // codes of the block (multiple of 16)
  int32_t bytes;       // codes + meta (multiple of 16)
};

DC_HD int64_t dc_align(int64_t x, int64_t a) { return (x + a - 1) / a * a; }
DC_HD int32_t dc_min(int32_t a, int32_t b) { return a < b ? a : b; }

// bytes of one lane's codes for one group of one row (all planes)
DC_HD int32_t dc_v_lane_group_bytes(int32_t bits) { return bits == 2 ? 8 : (bits == 3 ? 12 : 32); }
// bytes of plane 0 (2-bit plane or the 8-bit plane) of one lane for ngrp groups
DC_HD int32_t dc_v_plane0_bytes(int32_t bits, int32_t ngrp) { return (bits == 8 ? 32 : 8) * ngrp; }
// code bytes of one (tile, block): 4 lanes per valid row, all planes
DC_HD int64_t dc_v_block_code_bytes(int32_t bits, int32_t rows, int32_t ngrp) {
  return (int64_t)4 * rows * dc_v_lane_group_bytes(bits) * ngrp;
}
// bytes of one (tile, block): codes, then 64 bytes of meta per group
DC_HD int64_t dc_v_block_bytes(int32_t bits, int32_t rows, int32_t ngrp) {
  return dc_v_block_code_bytes(bits, rows, ngrp) + (int64_t)64 * ngrp;
}
// byte offset of half h inside a (tile, block) region
DC_HD int64_t dc_v_half_off(int32_t bits, int32_t rows, int32_t ngrp, int32_t h) {
  int32_t n0 = rows < 8 ? rows : 8;
  return h == 0 ? 0 : (int64_t)4 * n0 * dc_v_lane_group_bytes(bits) * ngrp;
}
// 2-bit full blocks (mask layout): byte offset, inside a half of nl lanes, of lane `lane`'s words
// 4 hi .. 4 hi + 3 -- the first 16 bytes of every lane, then the second 16 bytes of every lane, so
// that consecutive lanes' 16-byte loads fall on different shared-memory banks.
DC_HD int32_t dc_v_mask_off(int32_t nl, int32_t lane, int32_t hi) { return 16 * nl * hi + 16 * lane; }
// bytes of one U shift-layout step holding nl lanes (both planes, each padded to 16)
DC_HD int64_t dc_u_step_bytes(int32_t bits, int32_t nl) {
  return dc_align((int64_t)nl * 4, 16) + (bits == 3 ? dc_align((int64_t)nl * 2, 16) : 0);
}
DC_HD int32_t dc_u_step_lanes(int32_t valid_ranks) {  // lanes (of 32) stored for a step
  int32_t nt = (valid_ranks + 7) / 8;
  return 8 * nt;
}

DC_HD bool dc_bits_ok(int32_t b) { return b == 0 || b == 2 || b == 3 || b == 8; }

// tiles of 16 ranks per group (= per serving work item) for a bit width
DC_HD int32_t dc_v_group_tiles(int32_t bits) { return bits == 2 ? 8 : (bits == 3 ? 5 : 2); }

// Block k of band B (u_quads/u_steps/u_last must be set).
DC_HD DcUBlk dc_u_block(const DcBand& B, int32_t k) {
  DcUBlk K;
  K.nq = K.q0 = K.ns = K.s0 = 0;
  K.last = 32;
  K.tile_bytes = 0;
  if (B.bits == 8) {
    K.rr0 = 64 * k;
    K.nr = dc_min(64, B.rank - K.rr0);
    K.code_bytes = (int32_t)dc_align((int64_t)128 * K.nr, 16);
    K.bytes = K.code_bytes + (int32_t)dc_align((int64_t)4 * K.nr, 16);
    return K;
  }
  if (B.bits == 2) {
    const int32_t nfull = B.u_quads / 2;
    if (k < nfull) {
      K.nq = 2;
      K.q0 = 2 * k;
    } else {
      K.nq = B.u_quads % 2;
      K.q0 = 2 * nfull;
      K.ns = B.u_steps;
      K.s0 = 0;
    }
    K.rr0 = 256 * k;
  } else {
    K.s0 = 8 * k;
    K.ns = dc_min(8, B.u_steps - K.s0);
    K.rr0 = 256 * k;
  }
  int32_t nr = 128 * K.nq;
  int32_t tb = 512 * K.nq;
  for (int32_t s = K.s0; s < K.s0 + K.ns; ++s) {
    const int32_t valid = (s == B.u_steps - 1) ? B.u_last : 32;
    nr += valid;
    tb += (int32_t)dc_u_step_bytes(B.bits, dc_u_step_lanes(valid));
    if (s == K.s0 + K.ns - 1) K.last = valid;
  }
  K.nr = nr;
  K.tile_bytes = tb;
  K.code_bytes = 8 * tb;
  K.bytes = K.code_bytes + (int32_t)dc_align((int64_t)4 * nr, 16);
  return K;
}

DC_HD int32_t dc_u_nblk(const DcBand& B) {
  if (B.bits == 8) return (B.rank + 63) / 64;
  if (B.bits == 2) return B.u_quads / 2 + ((B.u_quads % 2 + B.u_steps) > 0 ? 1 : 0);
  return (B.u_steps + 7) / 8;
}

// Compute the layout of a descriptor; layout.valid = 0 on an invalid descriptor.
DC_HD DcLayout dc_layout(const dc_factor_desc& d) {
  DcLayout L;
  L.valid = 0;
  L.d_out = d.d_out;
  L.d_in = d.d_in;
  L.n_bands = 0;
  L.r = 0;
  L.bytes = 0;
  L.s_off = 0;
  L.dev_base = 0;
  L.u_off = 0;
  L.u_unit = 0;
  L.umax_off = 0;
  L.r4 = 0;
  L.groups_in = d.d_in / DC_GROUP;
  L.groups_out = d.d_out / DC_GROUP;
  L.nkb = (L.groups_in + 3) / 4;
  L.tail_groups = L.groups_in - 4 * (L.nkb - 1);
  if (d.d_out <= 0 || d.d_in <= 0 || d.d_out % DC_GROUP || d.d_in % DC_GROUP) return L;
  if (d.n_bands < 0 || d.n_bands > DC_MAX_BANDS) return L;
  int32_t r = 0;
  for (int i = 0; i < d.n_bands; ++i) {
    if (!dc_bits_ok(d.bits[i]) || d.rank[i] < 0) return L;
    if (d.bits[i] == 0 || d.rank[i] == 0) continue;
    DcBand& B = L.band[L.n_bands++];
    B.bits = d.bits[i];
    B.rank = d.rank[i];
    B.r0 = r;
    r += d.rank[i];
  }
  int32_t cap = d.d_out < d.d_in ? d.d_out : d.d_in;
  if (r > cap) return L;
  L.r = r;
  L.r4 = (int32_t)dc_align(r, 4);
  L.umax_off = (int64_t)L.r4 * 4;
  int64_t off = dc_align(L.umax_off + 4, 256);  // S, then the U scale bound
  // V codes with inline meta
  for (int i = 0; i < L.n_bands; ++i) {
    DcBand& B = L.band[i];
    B.v_tiles = (B.rank + 15) / 16;
    B.v_group = dc_v_group_tiles(B.bits);
    B.v_off = off;
    B.v_tile_bytes = dc_v_block_bytes(B.bits, 16, L.groups_in);
    int32_t last_rows = B.rank - 16 * (B.v_tiles - 1);
    int64_t sz = B.v_tile_bytes * (B.v_tiles - 1) + dc_v_block_bytes(B.bits, last_rows, L.groups_in);
    off = dc_align(off + sz, 256);
  }
  // U: runs of 128-row groups, band by band, blocks inside a band
  int64_t in_unit = 0;
  for (int i = 0; i < L.n_bands; ++i) {
    DcBand& B = L.band[i];
    if (B.bits == 8) {
      B.u_quads = B.u_steps = 0;
      B.u_last = 32;
    } else {
      B.u_quads = B.bits == 2 ? B.rank / 128 : 0;
      int32_t rest = B.rank - 128 * B.u_quads;
      B.u_steps = (rest + 31) / 32;
      B.u_last = rest - 32 * (B.u_steps - 1);
      if (B.u_steps == 0) B.u_last = 32;
    }
    B.u_nblk = dc_u_nblk(B);
    B.u_full = dc_u_block(B, 0).bytes;
    B.u_boff = in_unit;
    B.u_bytes = (int64_t)(B.u_nblk - 1) * B.u_full + dc_u_block(B, B.u_nblk - 1).bytes;
    in_unit += B.u_bytes;
  }
  L.u_unit = in_unit;
  L.u_off = off;
  off = dc_align(off + L.u_unit * L.groups_out, 256);
  L.bytes = off;
  L.valid = 1;
  return L;
}

// ---- V group geometry (groups of v_group tiles, block-major inside a group)
DC_HD int32_t dc_v_tile_rows(const DcBand& B, int32_t tile) { return dc_min(16, B.rank - 16 * tile); }
DC_HD int32_t dc_v_group_ntiles(const DcBand& B, int32_t grp) { return dc_min(B.v_group, B.v_tiles - grp * B.v_group); }
// bytes of one block (ngrp groups of 128 columns) of every tile of group `grp`
DC_HD int64_t dc_v_group_block_bytes(const DcBand& B, int32_t grp, int32_t ngrp) {
  const int32_t n = dc_v_group_ntiles(B, grp);
  const int32_t last_rows = dc_v_tile_rows(B, grp * B.v_group + n - 1);
  return (int64_t)(n - 1) * dc_v_block_bytes(B.bits, 16, ngrp) + dc_v_block_bytes(B.bits, last_rows, ngrp);
}
// offset (inside the band) of group `grp`'s block `kb`; tile ti of it starts ti * dc_v_block_bytes(bits, 16, ngrp) later
DC_HD int64_t dc_v_group_block_off(const DcBand& B, const DcLayout& L, int32_t grp, int32_t kb) {
  return (int64_t)grp * B.v_group * B.v_tile_bytes + (int64_t)kb * dc_v_group_block_bytes(B, grp, 4);
}
