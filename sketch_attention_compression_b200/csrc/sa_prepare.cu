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

// Per-user query rows Q'_b = Q_b M for all users (fp32; a few MFLOP per
// call): out row (b, j) = sum_f Q[b][j][f] M[f][:], and rows j in
// [k, k_rows) are zero (the padded prototypes of the bf16 copy).  A CTA of
// 128 threads computes a tile of 32 rows x 64 columns: thread (ty, tx) owns
// rows 4ty..4ty+3 and columns 4tx..4tx+3, each an fmaf chain over f in
// ascending order.  The tile's 32 rows of Q (transposed: [f][row], so a
// thread's four row values are one 16-byte read) and 64 columns of M (all d
// of f) are staged in shared memory in one step, so the CTA waits for
// global memory once; per f a warp then reads 3 shared-memory wavefronts
// for 16 multiply-adds per thread.  The staging reads Q in 16-byte units
// when it is 16-byte aligned, else word by word, and finds a unit's user
// and row with one 32-bit division (rows stay below 2^31).
constexpr int kUqRows = 32, kUqCols = 64, kUqThreads = 128;
static_assert(kUqRows == 32, "the Q staging loop takes a unit's row from the low 5 bits");
static_assert(kUqCols == 64 && kUqThreads == 128, "16 x 8 threads own 4 x 4 outputs each");

size_t user_query_smem(int d) {
  return (static_cast<size_t>(d) * kUqRows + static_cast<size_t>(d) * kUqCols) * sizeof(float);
}

template <bool kVecQ>
__global__ void __launch_bounds__(kUqThreads)
    user_query_kernel(const float* __restrict__ Q, const float* __restrict__ M, uint32_t total,
                      int k, int k_rows, int d, float* __restrict__ out_f32,
                      uint16_t* __restrict__ out_bf16) {
  extern __shared__ __align__(16) float uq_sh[];
  float* qt = uq_sh;                 // [d][32]: qt[f][r] = Q row r of the tile, entry f
  float* ms = uq_sh + d * kUqRows;   // [d][64]
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const uint32_t row0 = blockIdx.x * kUqRows;
  const int col0 = blockIdx.y * kUqCols;
  // Launched as a programmatic dependent of the stream's previous kernel
  // (for back-to-back calls, the previous call's finalize, which already
  // waited for the fused pass that read the old Q'_b): nothing is read or
  // written before that kernel has completed.  The pass that reads Q'_b may
  // then start its own set-up (it waits for this grid before reading).
  grid_dependency_wait();
  grid_dependency_launch();
  // Q: a warp takes one 16-byte unit of 32 consecutive rows, so its
  // transposed stores are 32 consecutive words.
  const int d4 = d >> 2;
  for (int i = tid; i < kUqRows * d4; i += kUqThreads) {
    const int rr = i & (kUqRows - 1), u = i >> 5;
    const uint32_t R = row0 + static_cast<uint32_t>(rr);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (R < total) {
      const uint32_t b = R / static_cast<uint32_t>(k_rows);
      const int j = static_cast<int>(R - b * static_cast<uint32_t>(k_rows));
      if (j < k) {
        const float* src = Q + (static_cast<int64_t>(b) * k + j) * d + 4 * u;
        if constexpr (kVecQ) {
          v = *reinterpret_cast<const float4*>(src);
        } else {
          v = make_float4(src[0], src[1], src[2], src[3]);
        }
      }
    }
    qt[(4 * u + 0) * kUqRows + rr] = v.x;
    qt[(4 * u + 1) * kUqRows + rr] = v.y;
    qt[(4 * u + 2) * kUqRows + rr] = v.z;
    qt[(4 * u + 3) * kUqRows + rr] = v.w;
  }
  for (int i = tid; i < d * (kUqCols / 4); i += kUqThreads) {
    const int ff = i >> 4, u = i & 15;
    *reinterpret_cast<float4*>(ms + ff * kUqCols + 4 * u) =
        *reinterpret_cast<const float4*>(M + static_cast<int64_t>(ff) * d + col0 + 4 * u);
  }
  __syncthreads();
  float acc[4][4] = {};
#pragma unroll 4
  for (int ff = 0; ff < d; ++ff) {
    const float4 qv = *reinterpret_cast<const float4*>(qt + ff * kUqRows + 4 * ty);
    const float4 mv = *reinterpret_cast<const float4*>(ms + ff * kUqCols + 4 * tx);
    const float q[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      acc[r][0] = fmaf(q[r], mv.x, acc[r][0]);
      acc[r][1] = fmaf(q[r], mv.y, acc[r][1]);
      acc[r][2] = fmaf(q[r], mv.z, acc[r][2]);
      acc[r][3] = fmaf(q[r], mv.w, acc[r][3]);
    }
  }
  // Four consecutive columns: one 16-byte fp32 store, one 8-byte bf16 store
  // (the outputs are 16- and 8-byte aligned and d is a multiple of 64).
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const uint32_t R = row0 + static_cast<uint32_t>(4 * ty + r);
    if (R >= total) continue;
    const int64_t o = static_cast<int64_t>(R) * d + col0 + 4 * tx;
    if (out_f32 != nullptr)
      *reinterpret_cast<float4*>(out_f32 + o) = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    if (out_bf16 != nullptr)
      *reinterpret_cast<uint2*>(out_bf16 + o) =
          make_uint2(pack_bf16x2(acc[r][0], acc[r][1]), pack_bf16x2(acc[r][2], acc[r][3]));
  }
}

}  // namespace

cudaError_t launch_user_query(const float* queries, const float* M, int64_t batch, int k,
                              int k_rows, int d, float* out_f32, uint16_t* out_bf16,
                              cudaStream_t stream) {
  const int64_t rows = batch * k_rows;
  if (rows <= 0) return cudaSuccess;
  if (rows >= (int64_t{1} << 31) || d % kUqCols != 0 ||
      (reinterpret_cast<uintptr_t>(out_f32) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(out_bf16) & 7u) != 0)
    return cudaErrorInvalidValue;
  const bool vec = (reinterpret_cast<uintptr_t>(queries) & 15u) == 0;
  auto kern = vec ? user_query_kernel<true> : user_query_kernel<false>;
  const dim3 grid(static_cast<unsigned>((rows + kUqRows - 1) / kUqRows),
                  static_cast<unsigned>(d / kUqCols));
  const size_t smem = user_query_smem(d);
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kUqThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, queries, M, static_cast<uint32_t>(rows), k, k_rows, d,
                            out_f32, out_bf16);
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
