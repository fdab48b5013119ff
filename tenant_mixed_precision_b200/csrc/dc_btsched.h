// Work schedule of the tensor-core backbone kernel (k_base_tc): which chunks of which units each
// persistent CTA takes, and how a chunk index maps back to its unit.  Host code plans it
// (bt_plan) and the kernel walks it; the same functions compile for both, so the CPU tests drive
// exactly the mapping the kernel uses.
//
// A unit is (linear, 128-row output tile, block of NB tenant-sorted tokens); its K is cut into
// chunks of 128 bytes of a row (64 bf16 or 128 E4M3 columns).
// Stream-K (one token block, or too many blocks for teams): the chunks of all units form one
// sequence (linears largest-K first; inside a linear, groups of G row tiles, then the token block,
// then the tile in the group), split into equal contiguous ranges, CTA c taking range c.
// Teams (several token blocks): a team holds one CTA per token block; the chunks of one token
// block's units (tile-major, k inner) are split into equal ranges, one per team, and CTA
// (team, tb) takes its team's range for token block tb.  A team's CTAs walk the same weight chunks
// in step, so each chunk comes from DRAM once and from L2 for the other token blocks.  Global chunk
// index with teams: tb * ctb + h, h the index inside the token block's sequence.
// A unit whose chunks two or more ranges share is finished by its last contributor from fp32
// partials; its contributors are the CTAs c0, c0 + step, ..., c1 (bt_cta_of of its first and last
// chunk; step 1, or the team size).
//
// FW is the kernel's parameter block (or a test stand-in) with the fields used below.
#pragma once
#include <stdint.h>

#include <algorithm>

#ifdef __CUDACC__
#define DC_HD __host__ __device__ __forceinline__
#else
#define DC_HD inline
#endif

struct BtSeg {
  int u, slot, ot, tb, K;  // unit, linear order slot, tile, token block, chunks of the unit
  int64_t ustart;          // global index of the unit's first chunk
  int k0, k1;              // chunk range of this segment inside the unit
};

DC_HD int64_t bt_share(int64_t total, int parts, int i) { return (int64_t)i * total / parts; }

// [g0, g1): the chunk range of CTA c
template <class FW>
DC_HD void bt_range(const FW& F, int c, int64_t& g0, int64_t& g1) {
  if (F.bt_team) {
    const int nt = F.bt_grid / F.bt_team, tau = c / F.bt_team, tb = c - tau * F.bt_team;
    g0 = (int64_t)tb * F.bt_ctb + bt_share(F.bt_ctb, nt, tau);
    g1 = (int64_t)tb * F.bt_ctb + bt_share(F.bt_ctb, nt, tau + 1);
  } else {
    g0 = bt_share(F.bt_total, F.bt_grid, c);
    g1 = bt_share(F.bt_total, F.bt_grid, c + 1);
  }
}

template <class FW>
DC_HD int64_t bt_g0(const FW& F, int c) {
  int64_t g0, g1;
  bt_range(F, c, g0, g1);
  return g0;
}

// index of the equal share of `total` in `parts` that holds x
DC_HD int bt_part_of(int64_t x, int64_t total, int parts) {
  int i = (int)(x * parts / total);
  while (i + 1 < parts && bt_share(total, parts, i + 1) <= x) ++i;
  while (i > 0 && bt_share(total, parts, i) > x) --i;
  return i;
}

// CTA whose chunk range holds global chunk g
template <class FW>
DC_HD int bt_cta_of(const FW& F, int64_t g) {
  if (F.bt_team) {
    const int nt = F.bt_grid / F.bt_team;
    const int tb = (int)(g / F.bt_ctb);
    return bt_part_of(g - (int64_t)tb * F.bt_ctb, F.bt_ctb, nt) * F.bt_team + tb;
  }
  return bt_part_of(g, F.bt_total, F.bt_grid);
}

// The segment that starts at chunk g of a range ending at g1: its unit and chunk range.
template <class FW>
DC_HD BtSeg bt_seg_at(const FW& F, int64_t g, int64_t g1) {
  BtSeg S;
  if (F.bt_team) {  // h: index inside token block tb's sequence; units tile-major
    const int tb = (int)(g / F.bt_ctb);
    const int64_t h = g - (int64_t)tb * F.bt_ctb;
    int slot = 0;
    while (slot + 1 < F.n_lin && h >= F.bt_chunk_prefix[slot + 1]) ++slot;
    S.slot = slot;
    S.K = F.lin[F.order[slot]].d_in / (F.fp8 ? 128 : 64);
    const int tile = (int)((h - F.bt_chunk_prefix[slot]) / S.K);
    S.u = (F.tile_prefix[slot] + tile) * F.bt_ntb + tb;
    S.ot = tile;
    S.tb = tb;
    S.ustart = (int64_t)tb * F.bt_ctb + F.bt_chunk_prefix[slot] + (int64_t)tile * S.K;
    S.k0 = (int)(g - S.ustart);
    S.k1 = (int)(S.K < g1 - S.ustart ? S.K : g1 - S.ustart);
    return S;
  }
  int slot = 0;
  while (slot + 1 < F.n_lin && g >= F.bt_chunk_prefix[slot + 1]) ++slot;
  S.slot = slot;
  S.K = F.lin[F.order[slot]].d_in / (F.fp8 ? 128 : 64);  // chunks of 128 bytes of a row
  const int64_t local = (g - F.bt_chunk_prefix[slot]) / S.K;
  // unit order inside a linear: groups of G row tiles (about one CTA's share of chunks), then the
  // token block, then the tile inside the group.  The CTAs working on one group for different
  // token blocks start within about one tile of each other and walk the same tiles.
  const int ntiles = F.lin[F.order[slot]].d_out / 128, ntb = F.bt_ntb, G = F.bt_gtiles[slot];
  const int grp = (int)(local / ((int64_t)G * ntb));
  const int gl = G < ntiles - grp * G ? G : ntiles - grp * G;  // tiles of this group (the last may be short)
  const int rem = (int)(local - (int64_t)grp * G * ntb);
  S.u = (int)(F.tile_prefix[slot] * (int64_t)ntb + local);
  S.ot = grp * G + rem % gl;
  S.tb = rem / gl;
  S.ustart = F.bt_chunk_prefix[slot] + local * S.K;
  S.k0 = (int)(g - S.ustart);
  S.k1 = (int)(S.K < g1 - S.ustart ? S.K : g1 - S.ustart);
  return S;
}

// Host: the linears' order (largest d_in first, stable) and the cumulative 128-row tiles in that
// order.  Needs F.n_lin and F.lin[p].d_out, d_in.
template <class FW>
inline void bt_plan_order(FW& F) {
  int ord[8];
  for (int p = 0; p < F.n_lin; ++p) ord[p] = p;
  std::stable_sort(ord, ord + F.n_lin, [&](int a, int b) { return F.lin[a].d_in > F.lin[b].d_in; });
  F.tile_prefix[0] = 0;
  for (int i = 0; i < F.n_lin; ++i) {
    F.order[i] = ord[i];
    F.tile_prefix[i + 1] = F.tile_prefix[i] + F.lin[ord[i]].d_out / 128;
  }
}

// Host: the backbone schedule for T tokens in blocks of nb on at most max_ctas CTAs (after
// bt_plan_order; F.fp8 set).  Fills bt_ntb, bt_team, bt_ctb, bt_chunk_prefix, bt_total, bt_grid,
// bt_gtiles.
template <class FW>
inline void bt_plan(FW& F, int T, int nb, int max_ctas) {
  F.bt_ntb = (T + nb - 1) / nb;
  const int kc = F.fp8 ? 128 : 64;  // elements per 128-byte chunk
  int64_t ctb = 0;                  // chunks of one token block's units
  for (int i = 0; i < F.n_lin; ++i) ctb += (int64_t)(F.lin[F.order[i]].d_out / 128) * (F.lin[F.order[i]].d_in / kc);
  // teams of one CTA per token block when there are several blocks (prefill-sized batches)
  F.bt_team = (F.bt_ntb >= 2 && F.bt_ntb <= max_ctas) ? F.bt_ntb : 0;
  F.bt_ctb = ctb;
  F.bt_chunk_prefix[0] = 0;
  for (int i = 0; i < F.n_lin; ++i) {
    const int p = F.order[i];
    F.bt_chunk_prefix[i + 1] = F.bt_chunk_prefix[i] +
                               (int64_t)(F.lin[p].d_out / 128) * (F.bt_team ? 1 : F.bt_ntb) * (F.lin[p].d_in / kc);
  }
  F.bt_total = ctb * F.bt_ntb;
  if (F.bt_team)
    F.bt_grid = (int)std::min<int64_t>(max_ctas / F.bt_team, ctb) * F.bt_team;
  else
    F.bt_grid = (int)std::min<int64_t>(max_ctas, F.bt_total);
  const int64_t share = (F.bt_total + F.bt_grid - 1) / F.bt_grid;
  for (int i = 0; i < F.n_lin; ++i) {  // stream-K tile groups of about one CTA's share of chunks
    const int p = F.order[i];
    F.bt_gtiles[i] = (int)std::max<int64_t>(1, std::min<int64_t>(F.lin[p].d_out / 128, share / (F.lin[p].d_in / kc)));
  }
}
