// Shared-memory and tensor-memory plan of the fused tensor-core pass
// (sa_fused.cu), kept in a header of its own so that a host program can
// check it (tests/host/plan_check.cpp).
#pragma once

#include <stdint.h>

#include "sa_internal.h"

namespace sa {

constexpr int kPlanBlock = 16384;     // shared memory is planned in 16 KB blocks
constexpr int kPlanMaxSmem = 232448;  // 227 KB of dynamic shared memory per block

// Shared-memory plan, in 16 KB blocks (a box is 128 rows x 64 bf16 columns,
// 128-byte swizzled; Q' is KM x D, the probability tile KM x 128).
//   D = 128: 4 stages.  Stage s keeps box 0 at O - 2 L_s and box 1 at
//            O - L_s with L = {1, 3, 4, 5} and the ones at O = 12, so MMA2
//            reads its chunks at stride L_s.  Q' at 0-1, the probability
//            tile at 3 (and 5, stride 2, for 128 prototypes).
//   D = 64:  8 stages at 3..10, ones at 11 (stride 11 - block), Q' at 0,
//            the probability tile at 1 (and 2).
//   D = 256: 2 stages; boxes 0-1 at (3, 4) and (6, 7) read as one N = 128
//            MMA, boxes 2-3 at O - 2 L_s, O - L_s with L = {1, 3} and the
//            ones at O = 11 read as one N = 144 MMA.  Q' at 0-1, the
//            probability tile at 2.
// (tests/host/plan_check.cpp checks that the regions are disjoint and that
// every MMA2 operand's chunks lie at its stride.)
template <int D, int KM>
struct Plan {
  static_assert(D == 64 || D == 128 || D == 256, "width");
  static_assert(KM == 64 || KM == 128, "prototype padding");
  static_assert(D != 256 || KM == 64, "d = 256 supports up to 64 prototypes");
  static constexpr int S = D == 64 ? 8 : (D == 128 ? 4 : 2);
  static constexpr int kOnes = D == 128 ? 12 : 11;
  static constexpr int kP0 = D == 64 ? 1 : (D == 128 ? 3 : 2);
  static constexpr int kPStride = D == 128 ? 2 : 1;  // blocks between the 64-prototype chunks
  static constexpr int kPlanBlocks = D == 128 ? 13 : 12;
  static constexpr int kBars = kPlanBlocks * kPlanBlock;     // barriers and scheduler state after the blocks
  // Staging of the accumulator drain: each softmax lane quarter owns
  // kDrainRows rows x 32 fp32 columns (128-byte rows, the 16-byte unit
  // index XOR-ed with the row mod 8).
  static constexpr int kDrainRows = KM == 128 ? 32 : 16;
  static constexpr int kDrainBuf = 32 * 128;
  static constexpr int kDrain = kBars + 512;
  // Copy of the offsets from the CTA's first user on (kOffCache entries).
  static constexpr int kOffCache = 64;
  static constexpr int kOffs = kDrain + 4 * kDrainBuf;
  static constexpr int kSmem = kOffs + kOffCache * 8;
  static_assert(kSmem <= kPlanMaxSmem, "shared memory budget");
  // Prototype-split clusters (KM = 128 per CTA) reuse the drain staging
  // (their drain stores straight from registers) for the softmax row
  // statistics the other CTAs send: [group][tile parity] regions of 128
  // rows x 8 source CTAs, float.
  static constexpr int kXch = kDrain;
  static_assert(2 * 2 * 8 * 128 * 4 <= 4 * kDrainBuf, "cluster exchange slots");
  // TMEM columns: two S^T buffers (one per softmax group), then the
  // accumulator [X~ | m] with D + 16 columns; the masses are column D.
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColAcc = 2 * KM;
  static_assert(kColAcc + D + 16 <= 512, "TMEM budget");

  __host__ __device__ static constexpr int lstride(int s) {
    return D == 128 ? (s == 0 ? 1 : s + 2) : (s == 0 ? 1 : 3);  // {1,3,4,5} / {1,3}
  }
  // Block of box b of stage s.
  __host__ __device__ static constexpr int box(int s, int b) {
    return D == 64 ? 3 + s
         : D == 128 ? (b == 0 ? kOnes - 2 * lstride(s) : kOnes - lstride(s))
         : (b < 2 ? (s == 0 ? 3 : 6) + b
                  : (b == 2 ? kOnes - 2 * lstride(s) : kOnes - lstride(s)));
  }
  // MMA2 B operand part p (D = 256 has two): first block, chunk stride in
  // blocks, N.
  __host__ __device__ static constexpr int b_start(int s, int p) {
    return D == 256 && p == 0 ? box(s, 0) : box(s, D == 256 ? 2 : 0);
  }
  __host__ __device__ static constexpr int b_stride(int s, int p) {
    return D == 64 ? kOnes - box(s, 0) : (D == 256 && p == 0 ? 1 : lstride(s));
  }
  static constexpr int kParts = D == 256 ? 2 : 1;
  static constexpr int kPartN0 = D == 256 ? 128 : D + 16;  // N of part 0 (part 1: 144)
};

}  // namespace sa
