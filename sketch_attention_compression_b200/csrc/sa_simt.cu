// fp32 SA pass on the CUDA cores.
//
// The fp32 path has to match an fp64 evaluation to 1e-4 of the sketch's
// largest entry.  tcgen05's tf32 mode keeps 10 mantissa bits, which cannot
// meet that, so this pass uses fp32 FMAs for the affinities and fp64
// accumulation for the sketch and the mass.  It follows the same row-range
// split and partial-slot scheme as the tensor-core pass (sa_internal.h), so
// the finalize kernel is shared.
//
// Per CTA (256 threads), per 32-row tile of one user:
//   1. the tile's rows (all d columns) are staged in shared memory;
//   2. thread j < k computes s_ji = q'_j . x_i for the 32 rows (Q' rows come
//      through the L1 cache; log2 e is folded into Q'; with per-user queries
//      the rows of the user's own Q'_b);
//   3. each warp normalises 4 rows over the k prototypes: exp2(s - max) /
//      sum (section 2.1: the normaliser runs over prototypes);
//   4. every thread accumulates its (prototype, column) outputs
//      X~_jc += a_ji x_ic in fp64, and thread j < k its mass m_j += a_ji.
// blockIdx.y selects a 64-column slice of the sketch; the affinities are
// recomputed per slice.
#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {
namespace {

constexpr int kRowsPerTile = 32;
constexpr int kThreadsSimt = 256;
constexpr int kColsPerCta = 64;
constexpr int kMaxAccPerThread = 256 / 4;  // k <= 256 prototypes over 4 thread rows

__global__ void __launch_bounds__(kThreadsSimt)
    simt_fp32_kernel(const float* __restrict__ qf, const float* __restrict__ X, const PassArgs a) {
  extern __shared__ float sh[];
  const int d = a.d;
  const int k = a.k;
  float* xs = sh;                          // [32][d]
  float* ss = sh + kRowsPerTile * d;       // [32][k]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t G = gridDim.x;
  const int64_t c = blockIdx.x;
  const int col0 = blockIdx.y * kColsPerCta;
  const int ncols = (d - col0) < kColsPerCta ? (d - col0) : kColsPerCta;
  const int64_t N = a.total_rows;
  // The device flags of this call start clear (block 0's first global
  // access; this pass sets no flag itself).
  if (c == 0 && blockIdx.y == 0 && tid == 0 && !a.keep_flags) {
    a.header->flags = 0u;
    a.header->timeout_flags = 0u;
  }
  const int64_t R0 = range_begin(a.offsets, a.batch, N, c, G);
  const int64_t R1 = range_begin(a.offsets, a.batch, N, c + 1, G);
  if (a.batch == 0 || R0 >= R1) return;
  const int64_t b0 = user_at_or_before(a.offsets, a.batch, R0);

  // output ownership: column (tid % 64), prototypes jr, jr+4, jr+8, ...
  const int oc = tid % kColsPerCta;
  const int jr = tid / kColsPerCta;
  const bool col_ok = oc < ncols;

  double acc[kMaxAccPerThread];
  double macc = 0.0;

  SegmentWalker w{a.offsets, a.batch, R0, R1, b0};
  int64_t user, s, e, lo, hi;
  while (w.next(user, s, e, lo, hi)) {
#pragma unroll
    for (int i = 0; i < kMaxAccPerThread; ++i) acc[i] = 0.0;
    macc = 0.0;
    for (int64_t r0 = s; r0 < e; r0 += kRowsPerTile) {
      const int nrows = static_cast<int>((e - r0) < kRowsPerTile ? (e - r0) : kRowsPerTile);
      __syncthreads();
      for (int idx = tid; idx < kRowsPerTile * d; idx += kThreadsSimt) {
        const int rr = idx / d;
        xs[idx] = rr < nrows ? X[(r0 + rr) * d + (idx - rr * d)] : 0.f;
      }
      __syncthreads();
      // 2. affinities
      if (tid < k) {
        float sacc[kRowsPerTile];
#pragma unroll
        for (int rr = 0; rr < kRowsPerTile; ++rr) sacc[rr] = 0.f;
        const float* qrow = qf + (a.user_queries ? user * k * d : 0) + static_cast<int64_t>(tid) * d;
        for (int f = 0; f < d; ++f) {
          const float qv = __ldg(qrow + f);
#pragma unroll
          for (int rr = 0; rr < kRowsPerTile; ++rr) sacc[rr] = fmaf(qv, xs[rr * d + f], sacc[rr]);
        }
#pragma unroll
        for (int rr = 0; rr < kRowsPerTile; ++rr) ss[rr * k + tid] = sacc[rr];
      }
      __syncthreads();
      // 3. softmax over prototypes, 4 rows per warp
      for (int rr = warp; rr < kRowsPerTile; rr += kThreadsSimt / 32) {
        float* srow = ss + rr * k;
        if (rr >= nrows) {
          for (int j = lane; j < k; j += 32) srow[j] = 0.f;
          continue;
        }
        float mx = -INFINITY;
        for (int j = lane; j < k; j += 32) mx = fmaxf(mx, srow[j]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        float sum = 0.f;
        for (int j = lane; j < k; j += 32) {
          const float ev = exp2f(srow[j] - mx);
          srow[j] = ev;
          sum += ev;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        for (int j = lane; j < k; j += 32) srow[j] = srow[j] / sum;
      }
      __syncthreads();
      // 4. accumulate
      if (col_ok) {
        for (int rr = 0; rr < nrows; ++rr) {
          const double xv = static_cast<double>(xs[rr * d + col0 + oc]);
          const float* prow = ss + rr * k;
#pragma unroll
          for (int i = 0; i < kMaxAccPerThread; ++i) {
            const int j = jr + 4 * i;
            if (j < k) acc[i] = fma(static_cast<double>(prow[j]), xv, acc[i]);
          }
        }
      }
      if (tid < k)
        for (int rr = 0; rr < nrows; ++rr) macc += static_cast<double>(ss[rr * k + tid]);
    }
    const int64_t slot = segment_slot(c, lo, hi, R0, R1);
    float* dx = slot < 0 ? a.out_x + user * k * d : a.part_x + slot * k * d;
    float* dm = slot < 0 ? a.out_m + user * k : a.part_m + slot * k;
    if (col_ok) {
#pragma unroll
      for (int i = 0; i < kMaxAccPerThread; ++i) {
        const int j = jr + 4 * i;
        if (j < k) dx[static_cast<int64_t>(j) * d + col0 + oc] = static_cast<float>(acc[i]);
      }
    }
    if (blockIdx.y == 0 && tid < k) dm[tid] = static_cast<float>(macc);
  }
}

}  // namespace

cudaError_t launch_simt_fp32(const float* q_f32, const float* X, const PassArgs& a, int grid,
                             cudaStream_t stream) {
  const int ychunks = (a.d + kColsPerCta - 1) / kColsPerCta;
  const size_t smem = static_cast<size_t>(kRowsPerTile) * (a.d + a.k) * sizeof(float);
  cudaError_t err = cudaFuncSetAttribute(simt_fp32_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  simt_fp32_kernel<<<dim3(grid, ychunks), kThreadsSimt, smem, stream>>>(q_f32, X, a);
  return cudaGetLastError();
}

}  // namespace sa
