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
#include "sa_internal.h"

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

__global__ void prepare_query_kernel(const void* __restrict__ P, const void* __restrict__ W_Q,
                                     const void* __restrict__ W_K, int d, double qscale,
                                     bool bf16, float* __restrict__ q_f32,
                                     uint16_t* __restrict__ q_bf16) {
  extern __shared__ double sh[];  // p_row[d], m1[d]
  double* p_row = sh;
  double* m1 = sh + d;
  const int j = blockIdx.x;
  const int e = threadIdx.x;
  p_row[e] = load_in(P, static_cast<size_t>(j) * d + e, bf16);
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

}  // namespace

cudaError_t launch_prepare_query(const void* P, const void* W_Q, const void* W_K, int k,
                                 int d, double scale, bool bf16_inputs, float* q_f32,
                                 uint16_t* q_bf16, cudaStream_t stream) {
  const double log2e = 1.4426950408889634073599246810018921;  // 1 / ln 2
  prepare_query_kernel<<<k, d, 2 * d * sizeof(double), stream>>>(
      P, W_Q, W_K, d, scale * log2e, bf16_inputs, q_f32, q_bf16);
  return cudaGetLastError();
}

}  // namespace sa
