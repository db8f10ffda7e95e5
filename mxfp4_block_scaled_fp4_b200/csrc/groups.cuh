// groups.cuh -- the group table of the grouped (mixture-of-experts) GEMMs
// (fp4_gemm_grouped): built per CTA from the device-side group offsets and
// used to map a persistent tile index to (group, rows, N tile).
#pragma once

namespace fp4 {

// A tile of the grouped form: group e, N tile nt; its rows start at a_row0,
// and only rows [a_row_begin, a_row_end) of it belong to group e.  A
// group's first tile starts on the 128-row scale block of the group's first
// row, so that every tile's (and every CTA half's) A scales are one block's
// atoms; its rows before the group's start belong to the previous group and
// are computed but not stored.
struct GTile {
  int e, a_row0, a_row_begin, a_row_end, nt;
};

// Warp 0 builds the table from the E + 1 offsets (clamped to [0, M] and made
// non-decreasing, so that malformed offsets cannot address rows outside A
// and C), 32 groups per step with warp shuffles: gtab[0..E] = the tiles of
// `tile_rows` rows before group e (gtab[E] = all of them; a group's tiles
// cover its rows from the 128-row block of its first row on), gtab[CAP + 1 +
// e] = group e's first row (gtab[CAP + 1 + E] = the end of the last group).
// Every lane of the warp calls it.
template <int CAP>
__device__ __forceinline__ void build_group_table(const int* offsets, int E, int M, int tile_rows,
                                                  int* gtab, int lane) {
  int carry = 0, prev_end = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    // lanes past the last group repeat its end, so that lane 31 carries
    // the true end of the groups into the next step and the table
    const int e0 = min(e, E);
    const int r0 = min(max(offsets[e0], 0), M);
    const int r1 = (e < E) ? min(max(offsets[e + 1], 0), M) : r0;
    // non-decreasing starts: a group starts no earlier than the previous end
    int start = r0;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, start, o);
      if (lane >= o) start = max(start, v);
    }
    start = max(start, prev_end);
    const int end = (e < E) ? max(r1, start) : start;
    const int n = (e < E && end > start) ? (end - (start & ~127) + tile_rows - 1) / tile_rows : 0;
    int incl = n;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    if (e < E) {
      gtab[e] = carry + incl - n;
      gtab[CAP + 1 + e] = start;
    }
    carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    prev_end = __shfl_sync(0xFFFFFFFFu, end, 31);
  }
  if (lane == 0) {
    gtab[E] = carry;
    gtab[CAP + 1 + E] = prev_end;
  }
}

// Tiles of group e occupy [tiles_before[e] * n_tiles, tiles_before[e+1] *
// n_tiles).  Inside a group they run in bands of `band` M tiles, M fastest
// inside a band and the bands one after the other (the plain GEMMs' raster):
// consecutive CTAs share a W tile in L2, and a large group's A rows are
// streamed band by band instead of once per N tile.
template <int CAP>
__device__ __forceinline__ GTile gtile(int t, int E, int n_tiles, int tile_rows, const int* gtab,
                                       int band) {
  const int* before = gtab;
  const int* row0 = gtab + CAP + 1;
  int lo = 0, hi = E;                           // largest e with before[e] * n_tiles <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (before[mid] * n_tiles <= t) lo = mid; else hi = mid;
  }
  GTile g;
  g.e = lo;
  const int mt_e = before[lo + 1] - before[lo];   // >= 1: t lies in a non-empty group
  const int local = t - before[lo] * n_tiles;
  const int per_band = band * n_tiles;
  const int b = local / per_band;
  const int first_m = b * band;
  const int gsize = min(band, mt_e - first_m);
  const int within = local - b * per_band;
  g.nt = within / gsize;
  g.a_row_begin = row0[lo];
  g.a_row0 = (row0[lo] & ~127) + (first_m + within % gsize) * tile_rows;
  g.a_row_end = row0[lo + 1];
  return g;
}

}  // namespace fp4
