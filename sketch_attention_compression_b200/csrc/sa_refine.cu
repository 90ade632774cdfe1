// The update of a stacked refinement layer after its SA step (section 2.2
// "Stacked Refinement" of the SequenceO1 reading notes,
// "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模").
//
// For every (user b, prototype j) row of width d:
//   z   = LN1(prev_bj + X~_bj / m_bj)           (X~/m: 0 where m_bj = 0)
//   out = LN2(z + (SiLU(z W1) * (z W3)) W2)
// LN over the feature axis with gain and shift, biased variance, eps 1e-5;
// W1, W3 are d x h and W2 is h x d (a SwiGLU feed-forward network, no
// biases).  The page lost the layer's formulas; this is the reading that its
// text supports: the aggregation added to the previous state and
// normalised, then a residual feed-forward network and a second norm.  The
// aggregation enters as the mass-normalised sketch (a weighted mean of the
// user's rows), whose scale does not grow with the history length.
//
// One CTA of 128 threads per 128-row tile; thread t owns row t of the tile
// (TMEM lane t).  The FFN runs on the tensor cores in 128-wide chunks of
// the hidden width:
//   H_c = z W1_c, G_c = z W3_c       M=128 rows, N=128, K=d   (TMEM cols 0, 128)
//   U_c = SiLU(H_c) * G_c            thread-local, bf16 into shared memory
//   Y  += U_c W2_c                   M=128 rows, N=d, K=128    (TMEM col 256)
// z and U are the MMAs' K-major A operands (bf16, 128-byte swizzle); the
// weight chunks arrive by TMA as K-major B operands (W1^T, W3^T: h x d;
// W2^T: d x h, bf16 copies made once by sa_prepare_refine).  The work is
// 2 (2 h d + h d) flop per row, small next to the SA pass over X, so the
// tile runs its steps in order rather than overlapping them.
#include <cuda_bf16.h>

#include <new>

#include "sa.h"
#include "sa_internal.h"
#include "sa_ptx.cuh"

struct sa_refine_s {
  int device;
  int sms;
  int d;
  int h;
  float* params;     // gamma1, beta1, gamma2, beta2: 4 x d fp32
  uint16_t* w13t;    // W1^T then W3^T: 2 x h x d bf16
  uint16_t* w2t;     // W2^T: d x h bf16
  CUtensorMap tm_w1, tm_w3, tm_w2;
};

namespace sa {
namespace {

constexpr int kRefThreads = 128;
constexpr float kLnEps = 1e-5f;

struct RefineArgs {
  const float* prev;     // [rows][d], or [k][d] when prev_shared
  int prev_shared;
  const float* x_tilde;  // [rows][d]
  const float* mass;     // [rows]
  const float* params;   // gamma1, beta1, gamma2, beta2
  float* out;            // [rows][d]
  int64_t rows;          // batch * k
  int k;
  int h;
  uint32_t* flags;       // timeout bits (may be null)
};

template <int D>
struct RefPlan {
  static constexpr int kBox = 128 * 128;         // 128 rows x 64 bf16
  static constexpr int kW2Box = D * 128;         // D rows x 64 bf16
  static constexpr int kZ = 0;                   // z: D / 64 boxes
  static constexpr int kW1 = kZ + (D / 64) * kBox;
  static constexpr int kW3 = kW1 + (D / 64) * kBox;
  static constexpr int kW2 = kW3 + (D / 64) * kBox;  // two boxes (hidden columns 0-63, 64-127)
  static constexpr int kU = kW2 + 2 * kW2Box;         // two boxes
  static constexpr int kBars = kU + 2 * kBox;
  static constexpr int kSmem = kBars + 256;
  static constexpr uint32_t kChunkBytes = 3u * 128u * D * 2u;
  static_assert(kSmem <= 232448, "shared memory budget");
};

// Offset of a K-step (16 columns) in a K-major, 128-byte-swizzled operand
// made of 64-column boxes `box` bytes apart, in descriptor units (16 B).
__device__ __forceinline__ uint64_t kstep(int ks, int box) {
  return static_cast<uint64_t>(((ks >> 2) * box + (ks & 3) * 32) >> 4);
}

// Byte offset of 16-byte unit u of row r in a 128-row box, 128-byte swizzle.
__device__ __forceinline__ uint32_t swz(int r, int u) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4);
}

template <int D>
__device__ __forceinline__ void ln_row(float (&v)[D], const float* gamma, const float* beta) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < D; ++i) s += v[i];
  const float mu = s / D;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < D; ++i) {
    const float c = v[i] - mu;
    q += c * c;
  }
  const float rstd = 1.0f / sqrtf(q / D + kLnEps);
#pragma unroll
  for (int i = 0; i < D; ++i) v[i] = (v[i] - mu) * rstd * gamma[i] + beta[i];
}

template <int D>
__global__ void __launch_bounds__(kRefThreads, 1)
    refine_update_kernel(const __grid_constant__ CUtensorMap tm_w1,
                         const __grid_constant__ CUtensorMap tm_w3,
                         const __grid_constant__ CUtensorMap tm_w2, const RefineArgs a) {
  using Pl = RefPlan<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5;
  if ((smem_u32(smem) & 1023u) != 0u) {  // the swizzled operands need 1024-byte alignment
    if (tid == 0 && a.flags != nullptr) atomicOr(a.flags, DEVFLAG_SMEM_ALIGN);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Pl::kBars);
  uint64_t* w_full = bars;      // a chunk of the weights has landed
  uint64_t* mma1 = bars + 1;    // H_c and G_c are in TMEM
  uint64_t* mma2 = bars + 2;    // Y += U_c W2_c has completed
  uint64_t* drain = bars + 3;   // abort path: every MMA issued so far has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  uint32_t* local_flags = tmem_slot + 2;  // timeout bits when the caller passes no flag word
  if (tid == 0) {
    mbar_init(w_full, 1);
    mbar_init(mma1, 1);
    mbar_init(mma2, 1);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    *local_flags = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  uint32_t* sticky = a.flags != nullptr ? a.flags : local_flags;
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const int chunks = a.h / 128;
  const float* g1 = a.params;
  const float* b1 = a.params + D;
  const float* g2 = a.params + 2 * D;
  const float* b2 = a.params + 3 * D;
  constexpr uint32_t idesc_h = idesc_bf16_f32(128, 128, 0, 0);
  constexpr uint32_t idesc_y = idesc_bf16_f32(128, D, 0, 0);
  const uint64_t dz = smem_desc(sbase + Pl::kZ, 16, 1024, 2);
  const uint64_t dw1 = smem_desc(sbase + Pl::kW1, 16, 1024, 2);
  const uint64_t dw3 = smem_desc(sbase + Pl::kW3, 16, 1024, 2);
  const uint64_t dw2 = smem_desc(sbase + Pl::kW2, 16, 1024, 2);
  const uint64_t du = smem_desc(sbase + Pl::kU, 16, 1024, 2);

  auto load_chunk = [&](int c) {  // thread 0
    mbar_arrive_expect_tx(w_full, Pl::kChunkBytes);
#pragma unroll
    for (int b = 0; b < D / 64; ++b) {
      tma_load_2d(smem + Pl::kW1 + b * Pl::kBox, &tm_w1, w_full, b * 64, c * 128);
      tma_load_2d(smem + Pl::kW3 + b * Pl::kBox, &tm_w3, w_full, b * 64, c * 128);
    }
#pragma unroll
    for (int b = 0; b < 2; ++b)
      tma_load_2d(smem + Pl::kW2 + b * Pl::kW2Box, &tm_w2, w_full, c * 128 + b * 64, 0);
  };

  uint32_t it = 0;         // chunk iterations so far (phase of all three barriers)
  uint32_t loads = 0;      // thread 0: chunk loads issued
  for (int64_t tile = blockIdx.x; tile * 128 < a.rows; tile += gridDim.x) {
    const int64_t r = tile * 128 + tid;
    const bool valid = r < a.rows;
    if (tid == 0 && !*abort_flag) {
      load_chunk(0);
      ++loads;
    }
    // z = LN1(prev + X~ / m), rounded to bf16 into the A operand.
    float z[D];
    if (valid) {
      const float* pv = a.prev + (a.prev_shared ? (r % a.k) : r) * D;
      const float* xv = a.x_tilde + r * D;
      const float mr = a.mass[r];
      const float inv = mr > 0.f ? 1.0f / mr : 0.f;
#pragma unroll
      for (int i = 0; i < D; i += 4) {
        const float4 p4 = *reinterpret_cast<const float4*>(pv + i);
        const float4 x4 = *reinterpret_cast<const float4*>(xv + i);
        z[i] = p4.x + x4.x * inv;
        z[i + 1] = p4.y + x4.y * inv;
        z[i + 2] = p4.z + x4.z * inv;
        z[i + 3] = p4.w + x4.w * inv;
      }
      ln_row<D>(z, g1, b1);
    } else {
#pragma unroll
      for (int i = 0; i < D; ++i) z[i] = 0.f;
    }
#pragma unroll
    for (int b = 0; b < D / 64; ++b)
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = b * 64 + u * 8;
        st_shared_v4(sbase + Pl::kZ + b * Pl::kBox + swz(tid, u), pack_bf16x2(z[i], z[i + 1]),
                     pack_bf16x2(z[i + 2], z[i + 3]), pack_bf16x2(z[i + 4], z[i + 5]),
                     pack_bf16x2(z[i + 6], z[i + 7]));
      }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    for (int c = 0; c < chunks; ++c, ++it) {
      if (tid == 0 && !*abort_flag && mbar_wait(w_full, it & 1u, abort_flag, sticky)) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_bf16_ss(tmem, dz + kstep(ks, Pl::kBox), dw1 + kstep(ks, Pl::kBox), idesc_h,
                      ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_bf16_ss(tmem + 128, dz + kstep(ks, Pl::kBox), dw3 + kstep(ks, Pl::kBox), idesc_h,
                      ks > 0 ? 1u : 0u);
        mma_commit(mma1);
      }
      // U_c = SiLU(H_c) * G_c for this thread's row, 32 columns at a time.
      if (!*abort_flag && mbar_wait(mma1, it & 1u, abort_flag, sticky)) {
        tc_fence_after();
#pragma unroll 1
        for (int p = 0; p < 4; ++p) {
          uint32_t hv[32], gv[32];
          tmem_ld32(lane_addr + p * 32, hv);
          tmem_ld32(lane_addr + 128 + p * 32, gv);
          tmem_wait_ld();
          tmem_pin32(hv);
          tmem_pin32(gv);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = u * 8 + 2 * e;
              const float x0 = __uint_as_float(hv[i]), x1 = __uint_as_float(hv[i + 1]);
              const float u0 = x0 / (1.0f + __expf(-x0)) * __uint_as_float(gv[i]);
              const float u1 = x1 / (1.0f + __expf(-x1)) * __uint_as_float(gv[i + 1]);
              w[e] = pack_bf16x2(u0, u1);
            }
            st_shared_v4(sbase + Pl::kU + (p >> 1) * Pl::kBox + swz(tid, (p & 1) * 4 + u), w[0],
                         w[1], w[2], w[3]);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0 && !*abort_flag) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_bf16_ss(tmem + 256, du + kstep(ks, Pl::kBox), dw2 + kstep(ks, Pl::kW2Box), idesc_y,
                      (c > 0 || ks > 0) ? 1u : 0u);
        mma_commit(mma2);
        // The next chunk's weights may replace these once Y's MMAs (the
        // last readers of the buffers) have completed.
        if (c + 1 < chunks && mbar_wait(mma2, it & 1u, abort_flag, sticky)) {
          load_chunk(c + 1);
          ++loads;
        }
      }
    }
    // out = LN2(z + Y).
    if (!*abort_flag && mbar_wait(mma2, (it - 1u) & 1u, abort_flag, sticky)) {
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t yv[32];
        tmem_ld32(lane_addr + 256 + cc * 32, yv);
        tmem_wait_ld();
        tmem_pin32(yv);
#pragma unroll
        for (int i = 0; i < 32; ++i) z[cc * 32 + i] += __uint_as_float(yv[i]);
      }
      if (valid) {
        ln_row<D>(z, g2, b2);
        float* ov = a.out + r * D;
#pragma unroll
        for (int i = 0; i < D; i += 4)
          *reinterpret_cast<float4*>(ov + i) = make_float4(z[i], z[i + 1], z[i + 2], z[i + 3]);
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (*abort_flag && tid == 0) {
    // A wait gave up: let the copies and MMAs already issued finish before
    // the tensor memory is released.
    if (loads > 0) mbar_wait_bounded(w_full, (loads - 1) & 1u);
    mma_commit(drain);
    mbar_wait_bounded(drain, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// W^T in bf16 (round to nearest even): out[c][i] = W[i][c] for W rows x cols.
__global__ void transpose_bf16_kernel(const float* __restrict__ W, int rows, int cols,
                                      uint16_t* __restrict__ out) {
  const int64_t n = static_cast<int64_t>(rows) * cols;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t c = e / rows, i = e % rows;
    out[e] = __bfloat16_as_ushort(__float2bfloat16_rn(W[i * cols + c]));
  }
}

template <int D>
cudaError_t launch_update(const sa_refine_s* r, const RefineArgs& a, cudaStream_t st) {
  using Pl = RefPlan<D>;
  cudaError_t err = cudaFuncSetAttribute(refine_update_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Pl::kSmem);
  if (err != cudaSuccess) return err;
  const int64_t tiles = (a.rows + 127) / 128;
  const unsigned grid = static_cast<unsigned>(tiles < r->sms ? tiles : r->sms);
  refine_update_kernel<D><<<grid, kRefThreads, Pl::kSmem, st>>>(r->tm_w1, r->tm_w3, r->tm_w2, a);
  return cudaGetLastError();
}

bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

cudaError_t launch_refine_update(const sa_refine_s* r, const float* prev, bool prev_shared,
                                 const float* x_tilde, const float* mass, int64_t batch, int k,
                                 float* out, uint32_t* flags, cudaStream_t st) {
  RefineArgs a;
  a.prev = prev;
  a.prev_shared = prev_shared ? 1 : 0;
  a.x_tilde = x_tilde;
  a.mass = mass;
  a.params = r->params;
  a.out = out;
  a.rows = batch * k;
  a.k = k;
  a.h = r->h;
  a.flags = flags;
  if (a.rows == 0) return cudaSuccess;
  return r->d == 64 ? launch_update<64>(r, a, st) : launch_update<128>(r, a, st);
}

int refine_width(const sa_refine_s* r) { return r->d; }

}  // namespace sa

extern "C" {

sa_status sa_prepare_refine(const float* W1, const float* W3, const float* W2,
                            const float* gamma1, const float* beta1, const float* gamma2,
                            const float* beta2, int d, int h, void* stream, sa_refine* out) {
  if (out == nullptr) return SA_ERR_INVALID_ARG;
  *out = nullptr;
  if (W1 == nullptr || W3 == nullptr || W2 == nullptr || gamma1 == nullptr || beta1 == nullptr ||
      gamma2 == nullptr || beta2 == nullptr)
    return SA_ERR_INVALID_ARG;
  if (h < 128 || h > 4096 || h % 128 != 0) return SA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return d == 256 ? SA_ERR_UNSUPPORTED : SA_ERR_INVALID_ARG;
  if (!sa::aligned_to(W1, 4) || !sa::aligned_to(W3, 4) || !sa::aligned_to(W2, 4) ||
      !sa::aligned_to(gamma1, 4) || !sa::aligned_to(beta1, 4) || !sa::aligned_to(gamma2, 4) ||
      !sa::aligned_to(beta2, 4))
    return SA_ERR_INVALID_ARG;
  int dev = 0, major = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return SA_ERR_CUDA;
  if (major != 10) return SA_ERR_UNSUPPORTED;
  sa_refine_s* r = new (std::nothrow) sa_refine_s;
  if (r == nullptr) return SA_ERR_CUDA;
  r->device = dev;
  r->sms = sms;
  r->d = d;
  r->h = h;
  r->params = nullptr;
  r->w13t = nullptr;
  r->w2t = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t hd = static_cast<size_t>(h) * d;
  bool ok = cudaMalloc(&r->params, 4 * d * sizeof(float)) == cudaSuccess &&
            cudaMalloc(&r->w13t, 2 * hd * sizeof(uint16_t)) == cudaSuccess &&
            cudaMalloc(&r->w2t, hd * sizeof(uint16_t)) == cudaSuccess;
  const float* src[4] = {gamma1, beta1, gamma2, beta2};
  for (int i = 0; ok && i < 4; ++i)
    ok = cudaMemcpyAsync(r->params + i * d, src[i], d * sizeof(float), cudaMemcpyDeviceToDevice,
                         st) == cudaSuccess;
  if (ok) {
    const unsigned grid = static_cast<unsigned>((hd + 255) / 256 < 4096 ? (hd + 255) / 256 : 4096);
    sa::transpose_bf16_kernel<<<grid, 256, 0, st>>>(W1, d, h, r->w13t);
    sa::transpose_bf16_kernel<<<grid, 256, 0, st>>>(W3, d, h, r->w13t + hd);
    sa::transpose_bf16_kernel<<<grid, 256, 0, st>>>(W2, h, d, r->w2t);
    ok = cudaGetLastError() == cudaSuccess;
  }
  ok = ok && sa::make_tmap_bf16(&r->tm_w1, r->w13t, h, d, 128) &&
       sa::make_tmap_bf16(&r->tm_w3, r->w13t + hd, h, d, 128) &&
       sa::make_tmap_bf16(&r->tm_w2, r->w2t, d, h, static_cast<uint32_t>(d));
  if (!ok) {
    cudaFree(r->params);
    cudaFree(r->w13t);
    cudaFree(r->w2t);
    delete r;
    return SA_ERR_CUDA;
  }
  *out = r;
  return SA_OK;
}

void sa_refine_free(sa_refine r) {
  if (r == nullptr) return;
  cudaFree(r->params);
  cudaFree(r->w13t);
  cudaFree(r->w2t);
  delete r;
}

sa_status sa_refine_update(sa_refine r, const float* prev, int prev_shared, const float* X_tilde,
                           const float* mass, int64_t batch, int k, float* out,
                           uint32_t* device_flags, void* stream) {
  if (r == nullptr || batch < 0 || k < 1) return SA_ERR_INVALID_ARG;
  if (batch == 0) return SA_OK;
  if (prev == nullptr || X_tilde == nullptr || mass == nullptr || out == nullptr)
    return SA_ERR_INVALID_ARG;
  if (!sa::aligned_to(prev, 16) || !sa::aligned_to(X_tilde, 16) || !sa::aligned_to(out, 16) ||
      !sa::aligned_to(mass, 4) || !sa::aligned_to(device_flags, 4))
    return SA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != r->device) return SA_ERR_INVALID_ARG;
  return sa::launch_refine_update(r, prev, prev_shared != 0, X_tilde, mass, batch, k, out,
                                  device_flags, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SA_OK
             : SA_ERR_CUDA;
}

}  // extern "C"
