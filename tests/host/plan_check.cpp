// Host-side check of the fused pass's shared-memory plan (sa_plan.h): for
// every supported (d, padded k) the regions -- Q', the probability tile, the
// X boxes of every stage and the block of ones -- are disjoint 16 KB blocks
// inside the dynamic shared memory, and every MMA2 B operand reads its
// 64-column chunks (X boxes, then the ones) at its descriptor's stride.
#include <cstdio>
#include <map>
#include <string>

#include "sa_plan.h"

using namespace sa;

template <int D, int KM>
static int check() {
  using P = Plan<D, KM>;
  std::map<int, std::string> used;
  auto take = [&](int blk, const std::string& who) {
    if (blk < 0 || blk >= P::kPlanBlocks) {
      std::printf("FAIL D=%d KM=%d: %s block %d outside [0, %d)\n", D, KM, who.c_str(), blk,
                  P::kPlanBlocks);
      return 1;
    }
    if (used.count(blk)) {
      std::printf("FAIL D=%d KM=%d: block %d used by %s and %s\n", D, KM, blk, used[blk].c_str(),
                  who.c_str());
      return 1;
    }
    used[blk] = who;
    return 0;
  };
  int bad = 0;
  const int q_blocks = (KM * D * 2 + kPlanBlock - 1) / kPlanBlock;
  for (int b = 0; b < q_blocks; ++b) bad |= take(b, "Q'");
  for (int c = 0; c < KM / 64; ++c) bad |= take(P::kP0 + c * P::kPStride, "P");
  bad |= take(P::kOnes, "ones");
  for (int s = 0; s < P::S; ++s)
    for (int b = 0; b < D / 64; ++b)
      bad |= take(P::box(s, b), "X" + std::to_string(s) + "." + std::to_string(b));
  // Barrier area (x_full/x_empty per stage; s_full, s_empty, acc_full,
  // drain per group; p_full, p_empty per group and slice; acc_empty,
  // q_full; stage_free per lane quarter; q_empty; the clusters'
  // stats_full per group and tile parity) and the scheduler words (TMEM
  // base, abort, first user, MMA2 count, pad, two range rows: ten 32-bit
  // words) must fit the 512 bytes before the drain staging (128-byte rows).
  const int bar_bytes = (2 * P::S + 4 * 2 + 2 * 8 + 2 + 4 + 1 + 4) * 8 + 10 * 4;
  if (bar_bytes > P::kDrain - P::kBars || P::kDrain % 128 != 0 ||
      P::kDrainRows * 128 > P::kDrainBuf) {
    std::printf("FAIL D=%d KM=%d: barrier area or drain staging\n", D, KM);
    bad = 1;
  }
  if (P::kSmem > kPlanMaxSmem) {
    std::printf("FAIL D=%d KM=%d: %d bytes of shared memory\n", D, KM, P::kSmem);
    bad = 1;
  }
  // MMA2 B operands: part 0 covers boxes [0, 2) (D = 256) or all boxes then
  // the ones; part 1 (D = 256) covers boxes 2, 3 then the ones.
  for (int s = 0; s < P::S; ++s) {
    for (int p = 0; p < P::kParts; ++p) {
      int expect[3], n = 0;
      if (D == 256 && p == 0) {
        expect[n++] = P::box(s, 0);
        expect[n++] = P::box(s, 1);
      } else {
        const int first = D == 256 ? 2 : 0;
        for (int b = first; b < D / 64; ++b) expect[n++] = P::box(s, b);
        expect[n++] = P::kOnes;
      }
      for (int i = 0; i < n; ++i) {
        const int got = P::b_start(s, p) + i * P::b_stride(s, p);
        if (got != expect[i]) {
          std::printf("FAIL D=%d KM=%d stage %d part %d chunk %d: block %d, expected %d\n", D, KM,
                      s, p, i, got, expect[i]);
          bad = 1;
        }
      }
      if (P::b_stride(s, p) * kPlanBlock / 16 >= (1 << 14)) {
        std::printf("FAIL D=%d KM=%d: stride does not fit the descriptor field\n", D, KM);
        bad = 1;
      }
    }
  }
  // TMEM: two S^T buffers and the (D + 16)-column accumulator.
  if (P::kColAcc + D + 16 > 512) {
    std::printf("FAIL D=%d KM=%d: TMEM\n", D, KM);
    bad = 1;
  }
  return bad;
}

int main() {
  int bad = check<64, 64>() | check<64, 128>() | check<128, 64>() | check<128, 128>() |
            check<256, 64>();
  if (!bad) std::printf("OK plans\n");
  return bad;
}
