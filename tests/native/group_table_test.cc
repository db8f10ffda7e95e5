// The grouped GEMM's group table (csrc/groups.cuh) on the CPU: the header is
// compiled as host code, build_group_table runs on 32 threads that stand in
// for the lanes of warp 0 (each shuffle is a write, a barrier and a read),
// and every tile the table yields is mapped with gtile exactly as the
// kernels map their persistent tile indices.  Checked for well-formed and
// malformed offsets, both tile heights (256 for CTA pairs, 128 for one-CTA
// tiles) and up to the 256-group limit:
//   - the groups are [s_e, end_e) with s_0 = clamp(o_0, 0, M),
//     end_e = max(clamp(o_{e+1}, 0, M), s_e), s_{e+1} = end_e;
//   - every row of every group is stored exactly once per N tile, by a tile
//     of its own group, and no other row is stored;
//   - every tile starts on a 128-row scale block inside [0, M) (its first
//     block of A scale atoms exists), lies in its group's rows and stores at
//     least one row; group and N tile indices are in range;
//   - the tile count stays within the launch's grid bound
//     ceil(M / tile_rows) + 2E tiles per N tile.
// Exit status 0 = all as expected (each mismatch is printed).
#include <algorithm>
#include <barrier>
#include <cstdio>
#include <functional>
#include <random>
#include <thread>
#include <vector>

// host stand-ins for the CUDA qualifiers, integer min/max and the warp
// shuffles that groups.cuh uses
#define __device__
#define __forceinline__ inline
static inline int min(int a, int b) { return a < b ? a : b; }
static inline int max(int a, int b) { return a > b ? a : b; }

namespace warp {
thread_local int lane = 0;
int slot[32];
std::barrier<>* bar = nullptr;
int exchange(int v, int src_lane) {
  slot[lane] = v;
  bar->arrive_and_wait();
  const int r = slot[src_lane];
  bar->arrive_and_wait();
  return r;
}
}  // namespace warp

static inline int __shfl_up_sync(unsigned, int v, int delta) {
  const int src = warp::lane >= delta ? warp::lane - delta : warp::lane;
  return warp::exchange(v, src);
}
static inline int __shfl_sync(unsigned, int v, int src_lane) { return warp::exchange(v, src_lane); }

#include "groups.cuh"

namespace {

constexpr int CAP = 256;
int failures = 0;
int cases = 0;

void fail(const char* what, int M, int E, int tile_rows, int detail) {
  if (failures < 40) std::printf("M=%d E=%d tile_rows=%d: %s (%d)\n", M, E, tile_rows, what, detail);
  ++failures;
}

std::vector<int> build(const std::vector<int>& offsets, int E, int M, int tile_rows) {
  std::vector<int> gtab(2 * CAP + 2, -1);
  std::barrier<> bar(32);
  warp::bar = &bar;
  std::vector<std::thread> lanes;
  for (int l = 0; l < 32; ++l)
    lanes.emplace_back([&, l] {
      warp::lane = l;
      fp4::build_group_table<CAP>(offsets.data(), E, M, tile_rows, gtab.data(), l);
    });
  for (auto& t : lanes) t.join();
  return gtab;
}

void check(const std::vector<int>& offsets, int E, int M, int tile_rows, int band, int n_tiles) {
  ++cases;
  // the groups the clamping rule defines
  std::vector<int> s(E), end(E);
  int prev = std::min(std::max(offsets[0], 0), M);
  for (int e = 0; e < E; ++e) {
    s[e] = prev;
    end[e] = std::max(std::min(std::max(offsets[e + 1], 0), M), s[e]);
    prev = end[e];
  }
  const std::vector<int> gtab = build(offsets, E, M, tile_rows);
  for (int e = 0; e < E; ++e)
    if (gtab[CAP + 1 + e] != s[e]) fail("group start", M, E, tile_rows, e);
  if (gtab[CAP + 1 + E] != (E ? end[E - 1] : 0)) fail("end of the last group", M, E, tile_rows, E);
  const int m_tiles = gtab[E];
  const int bound = (M + tile_rows - 1) / tile_rows + 2 * E;
  if (m_tiles < 0 || m_tiles > bound) fail("tile count above the grid bound", M, E, tile_rows, m_tiles);
  // stores[nt][row]: which group stored the row, how many times
  std::vector<std::vector<int>> count(n_tiles, std::vector<int>(std::max(M, 1), 0));
  std::vector<std::vector<int>> by(n_tiles, std::vector<int>(std::max(M, 1), -1));
  const int blocks = (M + 127) / 128;
  for (int t = 0; t < m_tiles * n_tiles; ++t) {
    const fp4::GTile g = fp4::gtile<CAP>(t, E, n_tiles, tile_rows, gtab.data(), band);
    if (g.e < 0 || g.e >= E) { fail("group index", M, E, tile_rows, g.e); continue; }
    if (g.nt < 0 || g.nt >= n_tiles) { fail("N tile index", M, E, tile_rows, g.nt); continue; }
    if (g.a_row_begin != s[g.e] || g.a_row_end != end[g.e]) fail("tile row range", M, E, tile_rows, t);
    if (g.a_row0 % 128 != 0) fail("tile not on a scale block", M, E, tile_rows, g.a_row0);
    if (g.a_row0 < 0 || g.a_row0 / 128 >= blocks) fail("first scale block outside A", M, E, tile_rows, g.a_row0);
    if (g.a_row0 < (s[g.e] & ~127) || g.a_row0 >= end[g.e])
      fail("tile outside its group", M, E, tile_rows, g.a_row0);
    int stored = 0;
    for (int r = g.a_row0; r < g.a_row0 + tile_rows; ++r) {
      if (r < g.a_row_begin || r >= g.a_row_end) continue;   // the kernels' row mask
      if (r < 0 || r >= M) { fail("stored row outside C", M, E, tile_rows, r); continue; }
      ++stored;
      ++count[g.nt][r];
      if (by[g.nt][r] >= 0 && by[g.nt][r] != g.e) fail("row stored by two groups", M, E, tile_rows, r);
      by[g.nt][r] = g.e;
    }
    if (stored == 0) fail("tile stores no row", M, E, tile_rows, t);
  }
  for (int nt = 0; nt < n_tiles; ++nt) {
    for (int e = 0; e < E; ++e)
      for (int r = s[e]; r < end[e]; ++r)
        if (count[nt][r] != 1 || by[nt][r] != e) {
          fail("group row not stored exactly once by its group", M, E, tile_rows, r);
          break;
        }
    const int first = E ? s[0] : 0, last = E ? end[E - 1] : 0;
    for (int r = 0; r < M; ++r)
      if ((r < first || r >= last) && count[nt][r]) fail("row outside every group stored", M, E, tile_rows, r);
  }
}

// offsets of groups with sizes drawn so that empty, one-row and large
// groups all occur, summing to M
std::vector<int> well_formed(std::mt19937& rng, int E, int M) {
  std::vector<double> w(E);
  std::exponential_distribution<double> ex(1.0);
  std::uniform_int_distribution<int> kind(0, 5);
  for (auto& v : w) {
    const int k = kind(rng);
    v = k == 0 ? 0.0 : k == 1 ? 1e-9 : ex(rng);
  }
  double sum = 0;
  for (double v : w) sum += v;
  std::vector<int> o(E + 1, 0);
  double acc = 0;
  for (int e = 0; e < E; ++e) {
    acc += w[e];
    o[e + 1] = sum > 0 ? static_cast<int>(acc / sum * M) : 0;
  }
  o[E] = M;
  for (int e = 1; e <= E; ++e) o[e] = std::max(o[e], o[e - 1]);
  return o;
}

// offsets no caller should pass: negative, past M, decreasing, a first
// offset above 0 and a last below M
std::vector<int> malformed(std::mt19937& rng, int E, int M) {
  std::uniform_int_distribution<int> any(-300, M + 300);
  std::vector<int> o(E + 1);
  for (auto& v : o) v = any(rng);
  return o;
}

}  // namespace

int main() {
  std::mt19937 rng(12345);
  const int Es[] = {1, 2, 7, 31, 32, 33, 64, 255, 256};
  const int Ms[] = {1, 100, 128, 129, 255, 256, 257, 1000, 4096, 16384};
  for (int pair = 0; pair < 2; ++pair) {
    const int tile_rows = pair ? 256 : 128, band = pair ? 32 : 16;
    for (int E : Es)
      for (int M : Ms)
        for (int n_tiles : {1, 3}) {
          check(well_formed(rng, E, M), E, M, tile_rows, band, n_tiles);
          check(malformed(rng, E, M), E, M, tile_rows, band, n_tiles);
        }
    // one row per group; every group in one scale block; all rows in the
    // last group; all groups empty
    for (int E : {8, 64, 256}) {
      std::vector<int> o(E + 1);
      for (int e = 0; e <= E; ++e) o[e] = e;
      check(o, E, E, tile_rows, band, 2);
      for (int e = 0; e <= E; ++e) o[e] = e * 127 / E;
      check(o, E, 127, tile_rows, band, 2);
      for (int e = 0; e <= E; ++e) o[e] = e == E ? 5000 : 0;
      check(o, E, 5000, tile_rows, band, 1);
      for (int e = 0; e <= E; ++e) o[e] = 0;
      check(o, E, 5000, tile_rows, band, 1);
    }
  }
  std::printf("%d cases, %d failures\n", cases, failures);
  return failures == 0 ? 0 : 1;
}
