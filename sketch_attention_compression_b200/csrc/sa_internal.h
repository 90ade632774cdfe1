// Internal declarations shared by the kernels and the C-ABI layer.
//
// Work split (all kernels of one call agree on it):
//   Splitting the N concatenated history rows over the G CTAs of a pass
//   charges each row 1 and each user start kUserStartCost rows: a user that
//   ends inside a CTA's range costs that range the drain of its sketch and
//   a part-filled last tile.  CTA c owns rows [R_c, R_{c+1}), where R_c is
//   the row at which the cost reaches c/G of the total C = N +
//   kUserStartCost * B, moved back to the user's first row or to a whole
//   number of 128-row tiles into the user, so every user's tiles are
//   aligned to its own first row.  Inside its range a CTA walks the users
//   in order; user b's part of the range is one "segment".
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

#include "sa.h"

#define SA_HD __host__ __device__ __forceinline__

struct sa_action_s;

namespace sa {

constexpr int kTileRows = 128;

// Workspace: [header 256 B][part_x: 2G * k * d fp32][part_m: 2G * k fp32]
struct WsHeader {
  uint32_t flags;          // offset validation bits (set by the finalize pass)
  uint32_t timeout_flags;  // bounded-wait timeouts (set by the partial pass)
  // Both words are zeroed by block 0 of the partial pass as its first global
  // write of every call.  Another CTA of that pass reports a timeout only
  // after one of its bounded waits has run out (seconds), and the finalize
  // pass sets the offset bits after the partial pass has completed, so the
  // clearing precedes every report of the call.  On misaligned shared memory
  // every CTA stops at once and block 0 alone writes both words.
  uint32_t pad[62];
};
constexpr size_t kWsHeaderBytes = 256;

SA_HD int64_t tiles_of(int64_t rows) { return (rows + kTileRows - 1) / kTileRows; }

// Cost, in rows, charged to each user start by the work split.
constexpr int64_t kUserStartCost = 640;

// Cost of everything before user b's first row.
SA_HD int64_t cost_before_user(const int64_t* off, int64_t b) { return off[b] + kUserStartCost * b; }

// Cost position at which CTA range c starts (0 < c < G).
SA_HD int64_t range_target(int64_t B, int64_t N, int64_t c, int64_t G) {
  return (c * (N + kUserStartCost * B)) / G;
}

// First row of CTA range c, given user b with cost_before_user(b) <= tau <
// cost_before_user(b + 1) for tau = range_target(c): the user's first row,
// or a whole number of tiles into it.  Clipped to [0, N] and to the user's
// rows (which only matters for invalid offsets).
SA_HD int64_t range_row(const int64_t* off, int64_t b, int64_t N, int64_t tau) {
  const int64_t into = tau - cost_before_user(off, b) - kUserStartCost;
  int64_t r = off[b] + (into > 0 ? (into / kTileRows) * kTileRows : 0);
  if (r > off[b + 1]) r = off[b + 1];
  if (r > N) r = N;
  return r < 0 ? 0 : r;
}

// First row of CTA range c (c in [0, G]; R_0 = 0, R_G = N).  *user, if
// given, receives the user found for it (range_row's b).  Serial binary
// search; the fused pass uses a warp-wide search with the same result.
SA_HD int64_t range_begin(const int64_t* off, int64_t B, int64_t N, int64_t c, int64_t G,
                          int64_t* user = nullptr) {
  if (c <= 0 || B <= 0 || c >= G) {
    if (user) *user = c <= 0 || B <= 0 ? 0 : B;
    return c <= 0 ? 0 : N;
  }
  const int64_t tau = range_target(B, N, c, G);
  int64_t lo = 0, hi = B - 1;  // largest b in [0, B) with cost_before_user(b) <= tau
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) >> 1;
    if (cost_before_user(off, mid) <= tau) lo = mid; else hi = mid - 1;
  }
  if (user) *user = lo;
  return range_row(off, lo, N, tau);
}

// The CTA range that holds row r of user b (off[b] <= r < off[b + 1]): the
// largest c with R_c <= r, from b's offsets alone.
SA_HD int64_t cta_of_row(const int64_t* off, int64_t b, int64_t B, int64_t N, int64_t G,
                         int64_t r) {
  const int64_t C = N + kUserStartCost * B;
  int64_t X = cost_before_user(off, b) + kUserStartCost +
              kTileRows * ((r - off[b]) / kTileRows + 1);
  const int64_t next = cost_before_user(off, b + 1);
  if (X > next) X = next;
  int64_t c = (X * G + C - 1) / C - 1;  // largest c with floor(c C / G) < X
  if (c < 0) c = 0;
  return c > G - 1 ? G - 1 : c;
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
  // 0: one Q' for every user.  1: user b's rows are queried by its own Q'_b
  // (the tensor-core pass reads rows b * k_pad.. of its Q' tensor map, the
  // fp32 pass the k x d block at b * k * d).
  int user_queries;
  // 1: leave the header's flag words as they are (a later layer of a stacked
  // call, which adds its flags to the earlier layers'); 0: clear them.
  int keep_flags;
};

// 2-D bf16 tensor map over a row-major [rows][cols] array: boxes of 64
// columns (128 bytes) x box_rows rows, 128-byte swizzle, zero fill.  False if
// the driver's encoder is unavailable or rejects the shape.
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);
// The same with the box width and swizzle chosen: 64 columns with the
// 128-byte swizzle, or 16 columns (32 bytes) with the 32-byte swizzle.
bool make_tmap_bf16_box(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                        uint32_t box_cols, uint32_t box_rows, int swizzle_bytes);

// Action-side fusion (sa_action.cu): the width d and the device of a
// prepared producer, and the producer kernel X = E + SwiGLU-FFN([E; a]) for
// `rows` rows enqueued on `st` (flag bits OR-ed into *flags when not null).
void action_info(const sa_action_s* act, int* d, int* device);

// sa_sketch_forward with the choice of keeping the workspace header's flag
// words (a later call of a sequence that reports every call's flags).
sa_status sketch_forward_flags(sa_query q, const void* X, const int64_t* offsets, int64_t batch,
                               int64_t total_rows, float* X_tilde, float* mass, void* workspace,
                               size_t workspace_bytes, void* stream, bool keep_flags);
sa_status action_fuse_enqueue(const sa_action_s* act, const void* E, const uint8_t* types,
                              int64_t rows, void* X, uint32_t* flags, cudaStream_t st);

// ---------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error.

// Q' = (P W_Q) W_K^T * scale * log2(e); writes q_f32 [k][d] and, if q_bf16
// is not null, q_bf16 [k_pad][d] (rows >= k must already be zero).
cudaError_t launch_prepare_query(const void* P, const void* W_Q, const void* W_K, int k,
                                 int d, double scale, bool bf16_inputs, float* q_f32,
                                 uint16_t* q_bf16, cudaStream_t stream);

// M = W_Q W_K^T * scale * log2(e) (d x d, fp32), for per-user queries.
cudaError_t launch_prepare_projection(const void* W_Q, const void* W_K, int d, double scale,
                                      bool bf16_inputs, float* m_f32, cudaStream_t stream);

// Q'_b = Q_b M for b < batch: queries [batch][k][d] fp32 -> rows of k_rows
// (>= k; rows k.. zero) written to out_f32 and/or out_bf16 ([batch][k_rows][d]).
cudaError_t launch_user_query(const float* queries, const float* M, int64_t batch, int k,
                              int k_rows, int d, float* out_f32, uint16_t* out_bf16,
                              cudaStream_t stream);

// Tensor-core pass (bf16 X).  Returns cudaErrorInvalidValue for an
// unsupported (d, k_pad) pair.
cudaError_t launch_fused_bf16(const CUtensorMap& tmap_x, const CUtensorMap& tmap_q,
                              int k_pad, const PassArgs& a, int grid, cudaStream_t stream);
bool fused_bf16_supported(int d, int k_pad);

// Tensor-core pass for d = 64 or 128 and 129..1024 prototypes: `ranges`
// clusters of ncl = k_pad / 128 CTAs (2..8), each CTA a slice of 128
// prototypes.  tmap_q reads 128-row boxes of the padded Q' (k_pad x d, or
// batch * k_pad x d with per-user queries).
cudaError_t launch_fused_bf16_cluster(const CUtensorMap& tmap_x, const CUtensorMap& tmap_q,
                                      const PassArgs& a, int ranges, int ncl,
                                      cudaStream_t stream);
// How many such clusters fit on the GPU at once (0 if none or on error).
int fused_bf16_cluster_max_clusters(int d, int ncl);

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

struct sa_refine_s;

namespace sa {

// The update of a refinement layer after its SA step (sa_refine.cu):
// out = LN2(z + FFN(z)), z = LN1(prev + x_tilde / mass), for batch * k rows;
// prev is k x d shared by every user when prev_shared.  Timeouts are OR-ed
// into *flags (may be null).
cudaError_t launch_refine_update(const sa_refine_s* r, const float* prev, bool prev_shared,
                                 const float* x_tilde, const float* mass, int64_t batch, int k,
                                 float* out, uint32_t* flags, cudaStream_t st);
// Feature width d of a refinement handle.
int refine_width(const sa_refine_s* r);

// Backward pass (sa_backward.cu).  launch_backward runs the per-tile kernel:
// dX (bf16) for every row, and R_b = ln 2 * dL/dQ' for every user into
// p.out_x (users inside one CTA range) or p.part_x (split users; the finalize
// pass sums them).  tmap_q reads k_pad-row boxes of Q'' (shared) or of the
// per-call Q''_b array (p.user_queries); tmap_g reads k_pad-row boxes of
// G_b (bf16, batch * k_pad x d); g_pad is batch x k_pad fp32.
bool backward_supported(int d, int k_pad);
cudaError_t launch_backward(const CUtensorMap& tx, const CUtensorMap& tq, const CUtensorMap& tg,
                            int k_pad, const PassArgs& p, const float* g_pad, uint16_t* dX,
                            int grid, cudaStream_t st);
// G (batch x k x d) -> bf16 batch x k_pad x d (zero rows past k); g -> fp32
// batch x k_pad (zeros past k, or everywhere when g is null).
cudaError_t launch_bwd_prep(const float* G, const float* g, int64_t batch, int k, int km, int d,
                            uint16_t* Gb, float* gp, cudaStream_t st);
// out = sum over `batch` consecutive blocks of n floats of R.
cudaError_t launch_sum_users(const float* R, int64_t batch, int64_t n, float* out,
                             cudaStream_t st);
// C[b] = alpha op(A[b]) op(B[b]) (+ C[b]), row-major, fp64 accumulation, for
// b < batch (strides sa, sb, sc in floats).
cudaError_t launch_bwd_gemm(const float* A, int64_t sa, bool ta, const float* B, int64_t sb,
                            bool tb, float* C, int64_t sc, int m, int n, int l, double alpha,
                            bool accumulate, int64_t batch, cudaStream_t st);

}  // namespace sa
