// Finalize pass: completes the outputs of a call after the partial pass.
//
//  * Split users (a user whose rows cross a CTA boundary of the partial
//    pass): X~ and m are the sums of the user's partial slots, taken in
//    ascending CTA order.  The order is fixed by the row split alone, so the
//    result does not depend on which CTA finished first.  Columns of the
//    sketch are independent (each behaviour's weights depend on that
//    behaviour only, section 2.1 of the SequenceO1 notes), which is what
//    makes a sum of per-range partial sketches exact up to rounding.
//  * Empty users get X~ = 0 and m = 0.
//  * The offsets are validated (offsets[0] == 0, non-decreasing,
//    offsets[B] == N); violations set bits in the workspace header.
//
// Block roles: the grid strides over units of a user: a run of consecutive
// chunks, where a chunk is 1024 entries of the user's k*d sketch (one
// 16-byte piece per thread) and 256 of its k masses, and the runs are long
// enough that the units of the users that can be split fit in about one
// wave.  The user's offsets decide the unit in one round trip: an empty
// user is zero-filled; for the others cta_of_row gives the CTAs that hold
// the first and the last row (pure arithmetic on the two offsets), and if
// they differ the user is split and the unit sums its slots: 2c for each
// later CTA c (the user starts before their ranges), and for the first CTA
// slot 2c if that CTA's range starts at the user's first row, else 2c + 1.
// That last choice has a closed form when the user before is not empty;
// otherwise warp 0 searches the range start while every thread's slot
// loads are in flight.  The validation bits are taken by the first unit of
// each user.
#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {
namespace {

constexpr int kFinThreads = 256;
constexpr int kChunkFloats = 4 * kFinThreads;  // sketch entries per chunk
constexpr int kFinBatch = 8;                   // slots loaded per round trip
constexpr int kFinBlocksPerSm = 2;             // resident blocks per SM (128 registers, no spills)
constexpr int64_t kFinWave = 148 * kFinBlocksPerSm;  // blocks of one wave on a B200

__device__ __forceinline__ float4 add4(float4 s, float4 v) {
  s.x += v.x;
  s.y += v.y;
  s.z += v.z;
  s.w += v.w;
  return s;
}

__global__ void __launch_bounds__(kFinThreads, kFinBlocksPerSm)
    finalize_kernel(const PassArgs a, int64_t G, int chunks, int per_unit) {
  grid_dependency_wait();
  grid_dependency_launch();  // the next call's fused pass may start its local set-up
  const int64_t N = a.total_rows, B = a.batch;
  const int k = a.k;
  const int64_t kd = static_cast<int64_t>(k) * a.d;
  const int groups = (chunks + per_unit - 1) / per_unit;  // units per user
  const int64_t units = B * groups;
  __shared__ long long s_first;  // start of the user's first CTA range
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    // Everything up to the sums is uniform across the block, so every
    // thread takes the same branches and barriers.
    const int64_t b = u / groups;
    const int g = static_cast<int>(u - b * groups);
    const int ch0 = g * per_unit, ch1 = min(ch0 + per_unit, chunks);
    const int64_t lo = a.offsets[b], hi = a.offsets[b + 1];
    const int64_t prev = b > 0 ? a.offsets[b - 1] : -1;
    if (g == 0 && threadIdx.x == 0) {
      uint32_t bits = 0;
      if (b == 0 && lo != 0) bits |= DEVFLAG_OFFSET0_NONZERO;
      if (lo > hi) bits |= DEVFLAG_OFFSETS_DECREASE;
      if (b == B - 1 && hi != N) bits |= DEVFLAG_OFFSET_LAST;
      if (bits != 0) atomicOr(&a.header->flags, bits);
    }
    float* out_x = a.out_x + b * kd;
    float* out_m = a.out_m + b * k;
    if (lo == hi) {
      for (int ch = ch0; ch < ch1; ++ch) {
        const int64_t i = static_cast<int64_t>(ch) * kChunkFloats + 4 * threadIdx.x;
        const int64_t j = static_cast<int64_t>(ch) * kFinThreads + threadIdx.x;
        if (i < kd) *reinterpret_cast<float4*>(out_x + i) = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j < k) out_m[j] = 0.f;
      }
      continue;
    }
    if (lo > hi) continue;  // flagged above
    const int64_t c_lo = cta_of_row(a.offsets, b, B, N, G, lo);
    const int64_t c_hi = cta_of_row(a.offsets, b, B, N, G, hi - 1 < N - 1 ? hi - 1 : N - 1);
    if (c_hi <= c_lo) continue;  // inside one range: the partial pass wrote the outputs

    bool first = false;  // the first CTA's slot is 2 c_lo (else 2 c_lo + 1)
    for (int ch = ch0; ch < ch1; ++ch) {
      const int64_t i = static_cast<int64_t>(ch) * kChunkFloats + 4 * threadIdx.x;  // X~ entry
      const int64_t j = static_cast<int64_t>(ch) * kFinThreads + threadIdx.x;       // mass entry
      const bool has_x = i < kd, has_m = j < k;
      // Both candidates for the first CTA's slot and the first batch of
      // later slots, all in flight at once.  Slots are added in ascending
      // CTA order, the fixed order that makes the result bitwise
      // reproducible.
      const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
      float4 x0 = zero, x1 = zero, xv[kFinBatch];
      float m0 = 0.f, m1 = 0.f, mv[kFinBatch];
      if (has_x) {
        x0 = *reinterpret_cast<const float4*>(a.part_x + (2 * c_lo) * kd + i);
        x1 = *reinterpret_cast<const float4*>(a.part_x + (2 * c_lo + 1) * kd + i);
      }
      if (has_m) {
        m0 = a.part_m[(2 * c_lo) * k + j];
        m1 = a.part_m[(2 * c_lo + 1) * k + j];
      }
#pragma unroll
      for (int t = 0; t < kFinBatch; ++t) {
        const int64_t cc = c_lo + 1 + t;
        xv[t] = zero;  // threads past the sketch's end add zeros (and store nothing)
        mv[t] = 0.f;
        if (cc <= c_hi) {
          if (has_x) xv[t] = *reinterpret_cast<const float4*>(a.part_x + (2 * cc) * kd + i);
          if (has_m) mv[t] = a.part_m[(2 * cc) * k + j];
        }
      }
      if (ch == ch0) {  // once per unit, while the loads above are in flight
        if (prev < lo) {
          // The user before b is not empty (or b = 0): range c_lo starts at
          // lo exactly when its cost target falls in b's start cost or
          // first tile (a target in an earlier user gives a start before
          // that user's end, which is below lo).
          const int64_t tau = c_lo > 0 ? range_target(B, N, c_lo, G) : 0;
          const int64_t cb = lo + kUserStartCost * b;  // cost_before_user(b)
          first = c_lo > 0 ? (tau >= cb && tau < cb + kUserStartCost + kTileRows) : lo == 0;
        } else {
          // Empty users (or bad offsets) just before b: find the range start.
          if (threadIdx.x < 32) {
            int64_t ub;
            const int64_t r = warp_range_begin(a.offsets, B, N, c_lo, G, threadIdx.x, &ub);
            if (threadIdx.x == 0) s_first = r;
          }
          __syncthreads();
          first = lo <= s_first;
          __syncthreads();  // s_first is rewritten by the block's next unit
        }
      }
      float4 sx = first ? x0 : x1;
      float sm = first ? m0 : m1;
#pragma unroll
      for (int t = 0; t < kFinBatch; ++t) {
        if (c_lo + 1 + t <= c_hi) {
          sx = add4(sx, xv[t]);
          sm += mv[t];
        }
      }
      for (int64_t cb = c_lo + 1 + kFinBatch; cb <= c_hi; cb += kFinBatch) {
#pragma unroll
        for (int t = 0; t < kFinBatch; ++t) {
          const int64_t cc = cb + t;
          if (cc <= c_hi) {
            if (has_x) xv[t] = *reinterpret_cast<const float4*>(a.part_x + (2 * cc) * kd + i);
            if (has_m) mv[t] = a.part_m[(2 * cc) * k + j];
          }
        }
#pragma unroll
        for (int t = 0; t < kFinBatch; ++t) {
          if (cb + t <= c_hi) {
            sx = add4(sx, xv[t]);
            sm += mv[t];
          }
        }
      }
      if (has_x) *reinterpret_cast<float4*>(out_x + i) = sx;
      if (has_m) out_m[j] = sm;
    }
  }
}

}  // namespace

cudaError_t launch_finalize(const PassArgs& a, int grid_ctas, cudaStream_t stream) {
  const int64_t kd = static_cast<int64_t>(a.k) * a.d;
  const int chunks = static_cast<int>((kd + kChunkFloats - 1) / kChunkFloats);
  if (a.batch <= 0) return cudaSuccess;
  // Chunks per unit: enough that the units of the users that can be split
  // (at most one per range boundary) fit in about one wave; a unit of a
  // user that is not split ends after its first round trip.
  const int64_t splittable = a.batch < grid_ctas - 1 ? a.batch : grid_ctas - 1;
  const int64_t want = (splittable * chunks + kFinWave - 1) / kFinWave;
  const int per_unit = static_cast<int>(want < chunks ? (want > 0 ? want : 1) : chunks);
  const int64_t units = a.batch * ((chunks + per_unit - 1) / per_unit);
  const int64_t blocks = units < 65535 * 32 ? units : 65535 * 32;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kFinThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, finalize_kernel, a, static_cast<int64_t>(grid_ctas), chunks,
                            per_unit);
}

}  // namespace sa
