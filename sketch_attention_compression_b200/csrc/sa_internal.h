// Internal declarations shared by the kernels and the C-ABI layer.
//
// Work split (all kernels of one call agree on it):
//   The N concatenated history rows are cut into T = ceil(N / 128) row tiles.
//   CTA c of a G-CTA grid (G <= T) owns rows [R_c, R_{c+1}) with
//   R_c = floor(c * T / G) * 128 (clipped to N), so every CTA has at least
//   one tile and the ranges are contiguous.  Inside its range a CTA walks
//   the users in order; user b's part of the range is one "segment".
//   * A user that lies wholly inside one CTA's range is written straight to
//     the outputs by that CTA.
//   * A user that crosses a CTA boundary is "split".  Each CTA writes its
//     share into a partial slot: slot 2c if the user starts at or before
//     R_c (it is the CTA's first user), else slot 2c+1 (it is the CTA's
//     last user).  At most two split users touch a CTA, so 2G slots suffice
//     whatever the batch size.
//   * The finalize kernel sums a split user's slots in ascending CTA order
//     (a fixed order, so results are bitwise reproducible), zero-fills empty
//     users and validates the offsets.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <cuda.h>
#include <cuda_runtime.h>

#define SA_HD __host__ __device__ __forceinline__

namespace sa {

constexpr int kTileRows = 128;

// Workspace: [header 256 B][part_x: 2G * k * d fp32][part_m: 2G * k fp32]
struct WsHeader {
  uint32_t flags;          // offset validation bits (set by the finalize pass)
  uint32_t timeout_flags;  // bounded-wait timeouts (set by the partial pass)
  // Both words are zeroed by CTA 0 of the partial pass at the start of every
  // call; all CTAs of that pass are resident together, so this precedes any
  // timeout report (which takes seconds to arise).
  uint32_t pad[62];
};
constexpr size_t kWsHeaderBytes = 256;

SA_HD int64_t tiles_of(int64_t rows) { return (rows + kTileRows - 1) / kTileRows; }

// First row of CTA c (c in [0, G]); R_G == N.
SA_HD int64_t cta_row_begin(int64_t c, int64_t G, int64_t T, int64_t N) {
  int64_t r = ((c * T) / G) * kTileRows;
  return r < N ? r : N;
}

// The CTA whose range holds row r (0 <= r < N); requires G <= T.
SA_HD int64_t cta_of_row(int64_t r, int64_t G, int64_t T) {
  int64_t u = r / kTileRows;
  return ((u + 1) * G - 1) / T;
}

// Largest b in [0, B) with off[b] <= r (off[0] <= r assumed; with invalid
// offsets the result is still some b in [0, B)).
SA_HD int64_t user_at_or_before(const int64_t* off, int64_t B, int64_t r) {
  int64_t lo = 0, hi = B - 1;
  while (lo < hi) {
    int64_t mid = (lo + hi + 1) >> 1;
    if (off[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Walks the segments of one CTA's row range, in user order.
struct SegmentWalker {
  const int64_t* off;
  int64_t B, R0, R1, b;
  // Optional copy of off[cb0, cb0 + ncache) (the fused pass keeps one in
  // shared memory); other entries are read from `off`.
  const int64_t* cache = nullptr;
  int64_t cb0 = 0, ncache = 0;
  SA_HD int64_t at(int64_t i) const {
    const int64_t ci = i - cb0;
    return (cache != nullptr && ci >= 0 && ci < ncache) ? cache[ci] : off[i];
  }
  SA_HD bool next(int64_t& user, int64_t& s, int64_t& e, int64_t& lo, int64_t& hi) {
    while (b < B) {
      const int64_t l = at(b), h = at(b + 1);
      if (l >= R1) { b = B; return false; }
      const int64_t cur = b++;
      const int64_t ss = l > R0 ? l : R0;
      const int64_t ee = h < R1 ? h : R1;
      if (ss < ee) { user = cur; s = ss; e = ee; lo = l; hi = h; return true; }
    }
    return false;
  }
};

// Walks the tiles of one CTA's row range: each call yields the first row of
// the next 128-row tile (tiles never straddle a segment start).
struct TileCursor {
  SegmentWalker w;
  int64_t r = 0, e = 0;
  bool have = false;
  SA_HD bool next(int64_t& row) {
    if (have && r + kTileRows < e) {
      r += kTileRows;
      row = r;
      return true;
    }
    int64_t user, s, lo, hi;
    have = w.next(user, s, e, lo, hi);
    if (!have) return false;
    r = s;
    row = r;
    return true;
  }
};

// Partial slot of a split user's segment in CTA c, or -1 if the user lies
// wholly inside the CTA's range (then it goes straight to the outputs).
SA_HD int64_t segment_slot(int64_t c, int64_t lo, int64_t hi, int64_t R0, int64_t R1) {
  if (lo >= R0 && hi <= R1) return -1;
  return 2 * c + (lo <= R0 ? 0 : 1);
}

// Arguments common to the partial-pass kernels.
struct PassArgs {
  const int64_t* offsets;
  int64_t batch;
  int64_t total_rows;
  int64_t tiles;     // T
  int k;
  int d;
  float* out_x;      // [B][k][d]
  float* out_m;      // [B][k]
  float* part_x;     // [2G][k][d]
  float* part_m;     // [2G][k]
  WsHeader* header;
};

// ---------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error.

// Q' = (P W_Q) W_K^T * scale * log2(e); writes q_f32 [k][d] and, if q_bf16
// is not null, q_bf16 [k_pad][d] (rows >= k must already be zero).
cudaError_t launch_prepare_query(const void* P, const void* W_Q, const void* W_K, int k,
                                 int d, double scale, bool bf16_inputs, float* q_f32,
                                 uint16_t* q_bf16, cudaStream_t stream);

// Tensor-core pass (bf16 X).  Returns cudaErrorInvalidValue for an
// unsupported (d, k_pad) pair.
cudaError_t launch_fused_bf16(const CUtensorMap& tmap_x, const CUtensorMap& tmap_q,
                              int k_pad, const PassArgs& a, int grid, cudaStream_t stream);
bool fused_bf16_supported(int d, int k_pad);

// Tensor-core pass for d = 256 and 129..256 prototypes: clusters of two CTAs,
// one per prototype half; `ranges` row ranges, 2 * ranges CTAs.  tmap_q_half
// reads 128-row boxes of the padded Q' (256 x 256).
cudaError_t launch_fused_bf16_pair(const CUtensorMap& tmap_x, const CUtensorMap& tmap_q_half,
                                   const PassArgs& a, int ranges, cudaStream_t stream);
// How many two-CTA clusters of that pass fit on the GPU at once (0 on error).
int fused_bf16_pair_max_clusters();

// fp32 CUDA-core pass.
cudaError_t launch_simt_fp32(const float* q_f32, const float* X, const PassArgs& a, int grid,
                             cudaStream_t stream);

// Fixed-order reduction of split users, zero-fill of empty users, offset
// validation.  Launched with programmatic stream serialization.
cudaError_t launch_finalize(const PassArgs& a, int grid_ctas, cudaStream_t stream);

}  // namespace sa
