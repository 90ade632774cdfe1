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
// Block roles: the first (G-1) * chunks blocks each own one CTA boundary c
// and one chunk of the k*d sketch entries; the boundary owns the reduction
// of the user that crosses it if that user starts inside CTA c-1's range
// (so every split user is reduced exactly once).  The remaining blocks
// stride over users for validation and empty users.
#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {
namespace {

constexpr int kFinThreads = 256;
constexpr int kChunkFloats = 2048;  // sketch entries per reduction block
constexpr int kValidateBlocks = 32;

__global__ void __launch_bounds__(kFinThreads)
    finalize_kernel(const PassArgs a, int64_t G, int chunks, int64_t reduce_blocks) {
  grid_dependency_wait();
  grid_dependency_launch();  // the next call's fused pass may start its local set-up
  const int64_t N = a.total_rows, B = a.batch;
  const int k = a.k, d = a.d;
  const int64_t kd = static_cast<int64_t>(k) * d;

  if (static_cast<int64_t>(blockIdx.x) < reduce_blocks) {
    const int64_t cb = blockIdx.x / chunks + 1;  // boundary between CTAs cb-1 and cb
    const int ch = blockIdx.x % chunks;
    // The two range starts, and the user found for R_cb: if it starts
    // before R_cb, it is the user whose rows contain R_cb.
    __shared__ long long s_rc, s_rp, s_user;
    if (threadIdx.x < 32) {
      int64_t bc, bp;
      const int64_t rc = warp_range_begin(a.offsets, B, N, cb, G, threadIdx.x, &bc);
      const int64_t rp = warp_range_begin(a.offsets, B, N, cb - 1, G, threadIdx.x, &bp);
      if (threadIdx.x == 0) {
        s_rc = rc;
        s_rp = rp;
        s_user = bc;
      }
    }
    __syncthreads();
    const int64_t Rc = s_rc, Rp = s_rp, b = s_user;
    if (b >= B) return;
    const int64_t lo = a.offsets[b], hi = a.offsets[b + 1];
    if (!(lo < Rc && lo >= Rp && hi > Rc)) return;  // not split here, or owned elsewhere
    const int64_t c_hi = cta_of_row(a.offsets, b, B, N, G, hi - 1 < N - 1 ? hi - 1 : N - 1);
    const int64_t c_lo = cb - 1;
    const int64_t slot_lo = 2 * c_lo + (lo <= Rp ? 0 : 1);

    const int64_t e0 = static_cast<int64_t>(ch) * kChunkFloats;
    const int64_t e1 = (e0 + kChunkFloats) < kd ? (e0 + kChunkFloats) : kd;
    float* out = a.out_x + b * kd;
    // The slots are read in batches of independent loads (a user spans
    // about ten CTA ranges; loading them one after another would put their
    // latencies end to end) and added in ascending CTA order, the fixed order
    // that makes the result bitwise reproducible.
    constexpr int kBatch = 8;
    for (int64_t i = e0 + 4 * threadIdx.x; i < e1; i += 4 * kFinThreads) {
      float4 s = *reinterpret_cast<const float4*>(a.part_x + slot_lo * kd + i);
      for (int64_t cc = c_lo + 1; cc <= c_hi; cc += kBatch) {
        float4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          if (cc + u <= c_hi) v[u] = *reinterpret_cast<const float4*>(a.part_x + (2 * (cc + u)) * kd + i);
#pragma unroll
        for (int u = 0; u < kBatch; ++u)
          if (cc + u <= c_hi) { s.x += v[u].x; s.y += v[u].y; s.z += v[u].z; s.w += v[u].w; }
      }
      *reinterpret_cast<float4*>(out + i) = s;
    }
    if (ch == 0) {
      for (int j = threadIdx.x; j < k; j += kFinThreads) {
        float s = a.part_m[slot_lo * k + j];
        for (int64_t cc = c_lo + 1; cc <= c_hi; cc += kBatch) {
          float v[kBatch];
#pragma unroll
          for (int u = 0; u < kBatch; ++u)
            if (cc + u <= c_hi) v[u] = a.part_m[(2 * (cc + u)) * k + j];
#pragma unroll
          for (int u = 0; u < kBatch; ++u)
            if (cc + u <= c_hi) s += v[u];
        }
        a.out_m[b * k + j] = s;
      }
    }
    return;
  }

  // validation and empty users
  const int64_t vb = blockIdx.x - reduce_blocks;
  const int64_t nvb = gridDim.x - reduce_blocks;
  uint32_t bits = 0;
  for (int64_t b = vb; b <= B; b += nvb) {
    const int64_t ob = a.offsets[b];
    if (b == 0 && ob != 0) bits |= DEVFLAG_OFFSET0_NONZERO;
    if (b == B) {
      if (ob != N) bits |= DEVFLAG_OFFSET_LAST;
      continue;
    }
    const int64_t on = a.offsets[b + 1];
    if (ob > on) bits |= DEVFLAG_OFFSETS_DECREASE;
    if (ob == on) {
      float* out = a.out_x + b * kd;
      for (int64_t i = threadIdx.x; i < kd; i += kFinThreads) out[i] = 0.f;
      for (int j = threadIdx.x; j < k; j += kFinThreads) a.out_m[b * k + j] = 0.f;
    }
  }
  if (bits != 0 && threadIdx.x == 0) atomicOr(&a.header->flags, bits);
}

}  // namespace

cudaError_t launch_finalize(const PassArgs& a, int grid_ctas, cudaStream_t stream) {
  const int64_t kd = static_cast<int64_t>(a.k) * a.d;
  const int chunks = static_cast<int>((kd + kChunkFloats - 1) / kChunkFloats);
  const int64_t reduce_blocks = static_cast<int64_t>(grid_ctas - 1) * chunks;
  int64_t vblocks = (a.batch + 1) < kValidateBlocks ? (a.batch + 1) : kValidateBlocks;
  const int64_t total = reduce_blocks + vblocks;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(total));
  cfg.blockDim = dim3(kFinThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, finalize_kernel, a, static_cast<int64_t>(grid_ctas), chunks,
                            reduce_blocks);
}

}  // namespace sa
