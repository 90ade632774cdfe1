// Query precompute for SA.
//
// S = (P W_Q)(X W_K)^T * scale can be evaluated as X-row dot products with
// Q' = (P W_Q) W_K^T * scale, because
//   S_ji = scale * sum_f (P W_Q)_jf (X W_K)_if
//        = sum_e X_ie [ scale * sum_f (P W_Q)_jf (W_K)_ef ] = sum_e X_ie Q'_je.
// This is the matrix rearrangement the SequenceO1 notes describe for
// single-query cross-attention (section 1): the per-behaviour key
// projection X W_K is never formed.  log2(e) is folded in as well, so the
// sketch kernels evaluate the softmax with exp2.
//
// One CTA per prototype row j, d threads; fp64 accumulation (the work is
// k*d*(2d) multiply-adds, negligible next to one pass over X).
//
// Per-user queries (the SA step of a refinement layer, section 2.2 "Stacked
// Refinement" of the same notes) change only the left factor: with
// M = W_Q W_K^T * scale * log2(e), prepared once per weight set (the same
// kernel with P = I), each call forms Q'_b = Q_b M for every user's k x d
// query matrix Q_b in fp32 (user_query_kernel).
#include <cuda_bf16.h>

#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {
namespace {

__device__ __forceinline__ double load_in(const void* p, size_t i, bool bf16) {
  if (bf16) {
    const uint16_t b = static_cast<const uint16_t*>(p)[i];
    return static_cast<double>(__uint_as_float(static_cast<uint32_t>(b) << 16));
  }
  return static_cast<double>(static_cast<const float*>(p)[i]);
}

// Round a double to the nearest bf16 (ties to even) in one step.  Going
// through float first rounds twice; the only case where that differs is a
// float that lands exactly on a bf16 halfway point although the double did
// not, which is resolved here by the sign of the first rounding's error.
__device__ __forceinline__ uint16_t double_to_bf16_rne(double x) {
  const float f = static_cast<float>(x);
  uint32_t u = __float_as_uint(f);
  if ((u & 0xFFFFu) == 0x8000u && static_cast<double>(f) != x) {
    const bool above = fabs(x) > fabs(static_cast<double>(f));
    u = (u & 0xFFFF0000u) + (above ? 0x10000u : 0u);
  } else {
    u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
  }
  return static_cast<uint16_t>(u >> 16);
}

// P == nullptr stands for the d x d identity (then q_f32 receives M).
__global__ void prepare_query_kernel(const void* __restrict__ P, const void* __restrict__ W_Q,
                                     const void* __restrict__ W_K, int d, double qscale,
                                     bool bf16, float* __restrict__ q_f32,
                                     uint16_t* __restrict__ q_bf16) {
  extern __shared__ double sh[];  // p_row[d], m1[d]
  double* p_row = sh;
  double* m1 = sh + d;
  const int j = blockIdx.x;
  const int e = threadIdx.x;
  p_row[e] = P != nullptr ? load_in(P, static_cast<size_t>(j) * d + e, bf16) : (e == j ? 1.0 : 0.0);
  __syncthreads();
  // m1 = p_j W_Q   (row vector times matrix)
  double acc = 0.0;
  for (int f = 0; f < d; ++f) acc += p_row[f] * load_in(W_Q, static_cast<size_t>(f) * d + e, bf16);
  m1[e] = acc;
  __syncthreads();
  // q_je = sum_f m1_f W_K[e][f]   (times W_K^T)
  acc = 0.0;
  for (int f = 0; f < d; ++f) acc += m1[f] * load_in(W_K, static_cast<size_t>(e) * d + f, bf16);
  acc *= qscale;
  q_f32[static_cast<size_t>(j) * d + e] = static_cast<float>(acc);
  if (q_bf16 != nullptr) q_bf16[static_cast<size_t>(j) * d + e] = double_to_bf16_rne(acc);
}

// Q'_b = Q_b M for all users: out row (b, j) = sum_f Q[b][j][f] M[f][:],
// fp32 multiply-adds in f order.  Rows j in [k, k_rows) are zero (the
// padded prototypes of the bf16 copy).  A CTA of 256 threads computes 32
// rows x 64 columns: thread (ty, tx) owns rows 2ty, 2ty+1 and columns
// 4tx..4tx+3; Q and M pass through shared memory in 32-wide slices of f.
constexpr int kUqRows = 32, kUqCols = 64, kUqF = 32;

__global__ void __launch_bounds__(256)
    user_query_kernel(const float* __restrict__ Q, const float* __restrict__ M, int64_t B, int k,
                      int k_rows, int d, float* __restrict__ out_f32,
                      uint16_t* __restrict__ out_bf16) {
  __shared__ float qs[kUqRows][kUqF + 1];
  __shared__ float ms[kUqF][kUqCols];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kUqRows;
  const int col0 = blockIdx.y * kUqCols;
  const int64_t total = B * k_rows;
  // The pass that reads Q' may start its set-up now (it waits for this
  // grid's completion before reading anything).
  grid_dependency_launch();
  float acc[2][4] = {};
  for (int f0 = 0; f0 < d; f0 += kUqF) {
    for (int i = tid; i < kUqRows * kUqF; i += 256) {
      const int rr = i / kUqF, ff = i % kUqF;
      const int64_t R = row0 + rr;
      float v = 0.f;
      if (R < total) {
        const int64_t b = R / k_rows;
        const int j = static_cast<int>(R - b * k_rows);
        if (j < k) v = Q[(b * k + j) * d + f0 + ff];
      }
      qs[rr][ff] = v;
    }
    for (int i = tid; i < kUqF * kUqCols; i += 256) {
      const int ff = i / kUqCols, cc = i % kUqCols;
      ms[ff][cc] = M[static_cast<int64_t>(f0 + ff) * d + col0 + cc];
    }
    __syncthreads();
#pragma unroll 8
    for (int ff = 0; ff < kUqF; ++ff) {
      const float q0 = qs[2 * ty][ff], q1 = qs[2 * ty + 1][ff];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float mv = ms[ff][4 * tx + u];
        acc[0][u] = fmaf(q0, mv, acc[0][u]);
        acc[1][u] = fmaf(q1, mv, acc[1][u]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t R = row0 + 2 * ty + h;
    if (R >= total) continue;
    const int64_t o = R * d + col0 + 4 * tx;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (out_f32 != nullptr) out_f32[o + u] = acc[h][u];
      if (out_bf16 != nullptr) out_bf16[o + u] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[h][u]));
    }
  }
}

}  // namespace

cudaError_t launch_user_query(const float* queries, const float* M, int64_t batch, int k,
                              int k_rows, int d, float* out_f32, uint16_t* out_bf16,
                              cudaStream_t stream) {
  const int64_t rows = batch * k_rows;
  if (rows <= 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((rows + kUqRows - 1) / kUqRows),
                  static_cast<unsigned>(d / kUqCols));
  user_query_kernel<<<grid, 256, 0, stream>>>(queries, M, batch, k, k_rows, d, out_f32, out_bf16);
  return cudaGetLastError();
}

cudaError_t launch_prepare_projection(const void* W_Q, const void* W_K, int d, double scale,
                                      bool bf16_inputs, float* m_f32, cudaStream_t stream) {
  return launch_prepare_query(nullptr, W_Q, W_K, d, d, scale, bf16_inputs, m_f32, nullptr,
                              stream);
}

cudaError_t launch_prepare_query(const void* P, const void* W_Q, const void* W_K, int k,
                                 int d, double scale, bool bf16_inputs, float* q_f32,
                                 uint16_t* q_bf16, cudaStream_t stream) {
  const double log2e = 1.4426950408889634073599246810018921;  // 1 / ln 2
  prepare_query_kernel<<<k, d, 2 * d * sizeof(double), stream>>>(
      P, W_Q, W_K, d, scale * log2e, bf16_inputs, q_f32, q_bf16);
  return cudaGetLastError();
}

}  // namespace sa
