// Mass-normalised sketch: X~_bj / m_bj, 0 where m_bj == 0.
//
// Section 2.1 of the SequenceO1 reading notes returns the sketch as a
// weighted sum; with the masses m_bj = sum_i A_ji the same sketch becomes a
// weighted mean of the user's rows, the form a refinement layer (section
// 2.2) can query with.  An empty prototype (m = 0: an empty user, or fp
// underflow) gets a zero row.
//
// Element-wise over B x k rows of d floats, HBM-bound: one thread per
// float4, the row's mass read once per thread (from L1/L2).
#include "sa.h"

namespace {

__global__ void mass_normalise_kernel(const float4* __restrict__ x, const float* __restrict__ m,
                                      int64_t rows, int d4, float4* __restrict__ out) {
  const int64_t n = rows * d4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float mj = m[i / d4];
    const float4 v = x[i];
    out[i] = mj > 0.f ? make_float4(v.x / mj, v.y / mj, v.z / mj, v.w / mj)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

}  // namespace

extern "C" sa_status sa_mass_normalise(const float* X_tilde, const float* mass, int64_t batch,
                                       int k, int d, float* out, void* stream) {
  if (batch < 0 || k < 1 || d < 4 || d % 4 != 0) return SA_ERR_INVALID_ARG;
  if (batch == 0) return SA_OK;
  if (X_tilde == nullptr || mass == nullptr || out == nullptr) return SA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(X_tilde) % 16 != 0 || reinterpret_cast<uintptr_t>(out) % 16 != 0 ||
      reinterpret_cast<uintptr_t>(mass) % 4 != 0)
    return SA_ERR_INVALID_ARG;
  const int64_t rows = batch * k;
  const int64_t n = rows * (d / 4);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return SA_ERR_CUDA;
  const int64_t want = (n + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
  mass_normalise_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float4*>(X_tilde), mass, rows, d / 4, reinterpret_cast<float4*>(out));
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}
