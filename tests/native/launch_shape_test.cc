// The launch-shape rules (csrc/launch_shape.h) on the CPU: fp4_gemm's
// choices for the decoder's M=256 shapes and for SM shares (with a device
// that can hold as many clusters as SMs allow), and the K slices of
// fp4_gemm_fused's decode kernel and chain.  Exit status 0 = all as
// expected (each mismatch is printed).
#include <cstdio>

#include "launch_shape.h"

namespace {

int failures = 0;

int clusters_148(int /*bn*/, int size) { return 148 / size; }

void expect(int m_tiles, int N, int k_steps, int sms, int bn, int splits) {
  const fp4::Shape s = fp4::choose_shape(m_tiles, N, k_steps, sms, clusters_148);
  if (s.bn != bn || s.splits != splits) {
    std::printf("m_tiles=%d N=%d k_steps=%d sms=%d: got %dx%d, expected %dx%d\n", m_tiles, N,
                k_steps, sms, s.bn, s.splits, bn, splits);
    ++failures;
  }
}

// the FP4-emitting and macro-block-scaled epilogues take no K split
void expect_nosplit(int m_tiles, int N, int k_steps, int sms, int bn) {
  const fp4::Shape s = fp4::choose_shape(m_tiles, N, k_steps, sms, clusters_148, false);
  if (s.bn != bn || s.splits != 1) {
    std::printf("no split: m_tiles=%d N=%d k_steps=%d sms=%d: got %dx%d, expected %dx1\n",
                m_tiles, N, k_steps, sms, s.bn, s.splits, bn);
    ++failures;
  }
}

void expect_pair(int M, int N, int sms, bool pair) {
  if (fp4::takes_pair(M, N, sms) != pair) {
    std::printf("M=%d N=%d sms=%d: pair %d, expected %d\n", M, N, sms, !pair, pair);
    ++failures;
  }
}

void expect_eq(const char* what, int got, int want) {
  if (got != want) {
    std::printf("%s: got %d, expected %d\n", what, got, want);
    ++failures;
  }
}

}  // namespace

int main() {
  // whole device (148 SMs); K steps of 256
  expect(2, 2880, 12, 148, 64, 1);    // M=256 2880x2880: 90 CTAs, no split
  expect(2, 3840, 12, 148, 64, 1);    // M=256 3840x2880
  expect(2, 720, 30, 148, 64, 5);     // M=256 720x7680: 24 tiles, K over 5-CTA clusters
  expect(2, 2880, 30, 148, 128, 2);   // M=256 2880x7680
  expect(1, 2880, 12, 148, 64, 1);    // M=128 2880x2880
  expect(4, 2880, 12, 148, 128, 1);   // M=512 2880x2880
  expect(1, 720, 30, 148, 64, 8);     // M=8 720x7680
  expect(1, 28672, 32, 148, 256, 1);  // M=128 28672x8192: persistent 256-wide tiles
  // a share of the device (concurrent GEMMs): fewer, wider tiles
  expect(2, 2880, 12, 49, 128, 1);
  expect(2, 3840, 12, 37, 256, 1);
  expect(2, 720, 30, 37, 128, 2);
  // without a K split the few-tile shapes keep their narrowest one-wave tile
  expect_nosplit(2, 720, 30, 148, 64);     // split 5 above
  expect_nosplit(2, 2880, 30, 148, 64);    // split 2 above
  expect_nosplit(1, 720, 30, 148, 64);
  expect_nosplit(2, 2880, 12, 148, 64);    // unchanged (no split above either)
  // the CTA-pair kernel
  expect_pair(8192, 28672, 148, true);
  expect_pair(600, 4104, 148, true);
  expect_pair(256, 2880, 148, false);
  expect_pair(128, 28672, 148, false);   // 128 rows: one CTA per tile
  expect_pair(2048, 4096, 40, true);
  // K slices of the fused small-M path: one-kernel decode (n_tiles = N/128,
  // K steps of 256, slices of at most 8 steps) and the chain's GEMM
  expect_eq("decode M=1 4096x4096", fp4::decode_splits(1, 32, 16, 148, 8), 4);
  expect_eq("decode M=1 2880x2880", fp4::decode_splits(1, 23, 12, 148, 8), 4);
  expect_eq("decode M=1 720x7680", fp4::decode_splits(1, 6, 30, 148, 8), 8);
  expect_eq("decode M=1 4096x14336", fp4::decode_splits(1, 32, 56, 148, 8), 7);
  expect_eq("decode M=1 14336x4096", fp4::decode_splits(1, 112, 16, 148, 8), 2);
  expect_eq("decode M=8 4096x4096", fp4::decode_splits(8, 32, 16, 148, 8), 8);
  expect_eq("decode M=1 2880x2880, 49 SMs", fp4::decode_splits(1, 23, 12, 49, 8), 4);
  expect_eq("decode M=1 2880x2880, 10 SMs", fp4::decode_splits(1, 23, 12, 10, 8), 1);
  expect_eq("chain M=8 4096x14336", fp4::chain_splits(8, 32, 56, 148), 4);
  expect_eq("chain M=16 4096x4096", fp4::chain_splits(16, 32, 16, 148), 8);
  expect_eq("chain M=32 4096x4096", fp4::chain_splits(32, 32, 16, 148), 4);
  expect_eq("chain M=16 2880x2880", fp4::chain_splits(16, 23, 12, 148), 8);
  expect_eq("chain M=16 720x7680", fp4::chain_splits(16, 6, 30, 148), 8);
  expect_eq("chain M=32 14336x4096", fp4::chain_splits(32, 112, 16, 148), 2);
  if (failures == 0) std::printf("launch shapes ok\n");
  return failures == 0 ? 0 : 1;
}
