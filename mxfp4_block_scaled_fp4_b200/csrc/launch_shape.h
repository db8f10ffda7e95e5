// launch_shape.h -- the launch-shape rules of fp4_gemm (host only): which
// kernel, output-tile width and K split a problem takes.  Free of CUDA types
// so that the rules are checked on the CPU as well (tests/native).
#pragma once
#include <initializer_list>

namespace fp4 {

struct Shape {
  int bn = 256;     // output tile width of the 128-row kernel
  int splits = 1;   // CTAs per tile along K (a thread-block cluster)
};

// The CTA-pair kernel (256 x 256 tiles) for M > 128 when its tiles keep at
// least half of the `sms` SMs busy; otherwise the 128-row kernel.
inline bool takes_pair(int M, int N, int sms) {
  const int pair_ctas = 2 * ((M + 255) / 256) * ((N + 255) / 256);
  return M > 128 && 2 * pair_ctas >= sms;
}

// Tile width and K split for the 128-row kernel on `sms` SMs, from a time
// model fitted to B200 measurements of these kernels (graph-launched, back
// to back): a CTA streams its A and W tiles (128 + BN rows of 144 bytes of
// codes and scales per K step) at about 112 bytes/ns; a split-K cluster
// adds about 1.5 us (two cluster barriers, the exchange's latency) plus the
// (S-1)/S x 128 x BN fp32 partial sums a CTA sends at about 41 bytes/ns
// (the SM-to-SM rate).  Narrow tiles are only taken when all CTAs fit in
// one wave; splits only with BN <= 128 and on at most 85% of the SMs (with
// 256-wide tiles, or clusters on nearly every SM, they measured slower
// than every alternative).  max_clusters(bn, S): clusters of S CTAs of the
// bn-wide kernel the device can hold at once (0 when unknown).
// allow_split = false keeps S = 1 (the epilogue that emits FP4 codes needs
// whole rows of a tile in one CTA).
template <typename MaxClusters>
Shape choose_shape(int m_tiles, int N, int k_steps, int sms, MaxClusters max_clusters,
                   bool allow_split = true) {
  Shape best;
  double best_t = 1e30;
  for (int bn : {256, 128, 64}) {
    const int tiles = m_tiles * ((N + bn - 1) / bn);
    for (int S = 1; S <= 8; ++S) {
      const int k_per = (k_steps + S - 1) / S;
      double t;
      if (S == 1) {
        if (bn != 256 && tiles > sms) continue;
        const int waves = (tiles + sms - 1) / sms;
        t = waves * (128.0 + bn) * k_per * 144.0 / 112.0;
      } else {
        if (!allow_split || bn == 256 || (k_steps + k_per - 1) / k_per != S ||
            tiles * S * 100 > sms * 85)
          continue;
        if (tiles > max_clusters(bn, S)) continue;
        t = (128.0 + bn) * k_per * 144.0 / 112.0 + 1500.0 +
            (S - 1.0) / S * 128.0 * bn * 4.0 / 41.0;
      }
      if (t < best_t) {
        best_t = t;
        best.bn = bn;
        best.splits = S;
      }
    }
  }
  return best;
}

// K slices of the one-kernel decode path (fp4_gemm_fused, small M): at most
// one wave of two CTAs per SM on `sms` SMs and at most 8 (a portable
// cluster).  At M <= 4 with many weight tiles, up to 4 (further splits add
// more cluster-reduction cost than their shorter weight streams save:
// measured on B200, M=1 4096x4096 6.7 us with 8 slices, 5.8 us with 4),
// more only where a slice would exceed max_steps K steps; with few tiles
// (M=1 720x7680: 5.7 us with 8 slices, 7.0 us with 4) or more rows to
// quantize per slice (M=8), up to 8.
inline int decode_splits(int M, int n_tiles, int k_steps, int sms, int max_steps) {
  int cap = 8;
  if (M <= 4 && n_tiles * 4 >= 64) {
    cap = (k_steps + max_steps - 1) / max_steps;   // slices that keep a slice <= max_steps
    if (cap < 4) cap = 4;
  }
  int s = 1;
  for (int t = 2; t <= 8 && t <= cap && t <= k_steps; ++t)
    if (n_tiles * t <= 2 * sms) s = t;
  return s;
}

// K slices of the small-M chain's GEMM (fp4_gemm_fused above the one-kernel
// limit), within one wave of two CTAs per SM and at most 8: up to 4 when 4
// slices still give >= 128 CTAs and the slices' partial sums are large
// (M > 16) or their weight streams long (>= 32 K steps) -- further splits
// then cost more in cluster reduction than they save: measured on B200,
// M=8 4096x14336 18.7 -> 15.4 us, M=32 4096x4096 13.0 -> 11.9 us; else up
// to 8 (M=16 4096x4096 10.0 us with 8 slices, 10.8 with 4; 720x7680 9.3
// vs 11.2 us).
inline int chain_splits(int M, int n_tiles, int k_steps, int sms) {
  const bool few_slices = n_tiles * 4 >= 128 && (M > 16 || k_steps >= 32);
  const int cap = few_slices ? 4 : 8;
  int s = 1;
  for (int t = 2; t <= cap && t <= k_steps; ++t)
    if (n_tiles * t <= 2 * sms) s = t;
  return s;
}

}  // namespace fp4
