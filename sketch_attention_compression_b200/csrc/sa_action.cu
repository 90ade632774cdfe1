// Action-side fusion, the producer of the history matrix X (section 2.2 of
// the SequenceO1 reading notes, "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模",
// "Stacked Refinement 与动作侧融合"):
//
//   x_i = e_i + (SiLU(z_i W1) * (z_i W3)) W2,   z_i = [e_i ; a_i],
//
// e_i the item embedding of behaviour i (d wide, bf16), a_i the row of the
// action-type table its type id selects, W1, W3 (d + d_a) x h, W2 h x d, no
// biases.  Because a_i takes one of n_types values, [e ; a] W1 splits into
// e W1_e + T1[type] with T1 = table W1_a (n_types x h), made once; the
// kernel adds T1[type] on the tensor cores as one extra K-step whose A
// operand is the one-hot row of the type (K = 16, so n_types <= 16).  The
// concatenation is never formed and the K of the big products is d.
//
// Kernel: persistent, one CTA per SM, pairs of 128-row tiles (slots A and
// B), the hidden width in chunks of 64.  Warp 0 issues TMA loads (E tiles;
// per chunk W1_e^T, W3_e^T, W2^T and the T1, T3 columns, into a two-stage
// ring whose W1/W3 and W2 parts have their own barriers, so each is
// refilled as soon as both slots have read it); warp 1 issues the MMAs;
// warps 2-9 gate slot A and warps 10-17 slot B, so that the two slots'
// epilogues overlap.  Per slot and chunk c:
//   [U | V] = E [W1_c | W3_c] + onehot [T1_c | T3_c]   M 128, N 128 (TMEM)
//   G = SiLU(U) * V                   epilogue: bf16 pairs back into TMEM
//   Y += G W2_c                       M 128, N d, K 64, A from TMEM (TMEM)
// U and V are one product (N = 128) so that each K-step reads the E slice
// from shared memory once, and G never passes through shared memory: at
// these shapes the shared-memory operand traffic, not the tensor cores, sets
// the pace.
// The residual is a product too: after the first chunk, Y += E I_16 slice
// by slice (M 128, N 16, K 16 per 16 columns of E), from the E tile already
// in shared memory, so that the epilogue only rounds Y to bf16 and stores
// it.  The two slots alternate on the tensor cores, which run one slot's
// products while the other slot's epilogue gates.  TMEM: slot r holds U at
// 256 r, V at 256 r + 64, Y at 256 r + 128.
// SiLU(u) = u sigma(u) with sigma(u) = (1 + tanh(u / 2)) / 2, one MUFU
// operation per element.
#include <cuda_bf16.h>

#include <new>

#include "sa.h"
#include "sa_internal.h"
#include "sa_ptx.cuh"

struct sa_action_s {
  int device;
  int sms;
  int d;
  int h;
  int n_types;
  uint16_t* w13t;  // W1_e^T then W3_e^T: 2 x h x d bf16
  uint16_t* w2t;   // W2^T: d x h bf16
  uint16_t* t13t;  // T1^T then T3^T: 2 x h x 16 bf16 (types >= n_types are 0)
  CUtensorMap tm_w1, tm_w3, tm_w2, tm_t1, tm_t3;
};

namespace sa {
namespace {

constexpr int kActThreads = 576;  // warp 0 TMA, warp 1 MMA, warps 2-9 and 10-17 epilogue
constexpr int kHc = 64;           // hidden columns per chunk
constexpr int kMaxTypes = 16;

template <int D>
struct ActPlan {
  static constexpr int kEBox = 128 * 128;      // 128 rows x 64 bf16
  static constexpr int kE = 0;                 // 2 slots x D/64 boxes
  static constexpr int kESlot = (D / 64) * kEBox;
  static constexpr int kW = kE + 2 * kESlot;   // 2 weight stages
  static constexpr int kWBox = kHc * 128;      // 64 rows x 64 bf16
  // Inside a stage: per 64 columns of K, the W1 box then the W3 box, so that
  // [W1_c ; W3_c] is one 128-row B operand and U, V one N = 128 product.
  static constexpr int kW13 = 0;
  static constexpr int kW13Box = 2 * kWBox;
  static constexpr int kW2 = kW13 + (D / 64) * kW13Box;  // D rows x 64 bf16
  static constexpr int kT1 = kW2 + D * 128;           // 64 rows x 16 bf16, 32-byte swizzle
  static constexpr int kT3 = kT1 + kHc * 32;
  static constexpr int kStage = kT3 + kHc * 32;
  static constexpr uint32_t kW13Bytes = 2 * (D / 64) * kWBox + 2 * kHc * 32;
  static constexpr uint32_t kW2Bytes = D * 128;
  static constexpr uint32_t kEBytes = kESlot;
  static constexpr int kOH = kW + 2 * kStage;  // 2 slots x 128 rows x 32 B
  static constexpr int kI = kOH + 2 * 128 * 32;  // I_16 (16 x 16 bf16, 32-byte swizzle)
  // Store staging: per epilogue warp 32 rows x 32 columns of X (bf16).
  static constexpr int kStg = kI + 1024;
  static constexpr int kStgWarp = 32 * 64;
  static constexpr int kBars = kStg + 16 * kStgWarp;
  // At least 116 KB, so that one CTA holds an SM (it allocates all of TMEM).
  static constexpr int kSmem = kBars + 256 > 118784 ? kBars + 256 : 118784;
  static_assert(kStage % 1024 == 0, "stage alignment");
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct ActArgs {
  const uint8_t* types;    // [rows]
  uint16_t* X;             // [rows][d] bf16 out
  int64_t rows;
  int64_t pairs;           // ceil(ceil(rows / 128) / 2)
  int chunks;              // h / 64
  int n_types;
  uint32_t* flags;         // may be null
};

__device__ __forceinline__ uint32_t swz32(int r, int u) {
  return r * 32 + ((u ^ ((r >> 2) & 1)) << 4);
}

__device__ __forceinline__ uint64_t kstep(int ks, int box) {
  return static_cast<uint64_t>(((ks >> 2) * box + (ks & 3) * 32) >> 4);
}

__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t gate_pair(float u0, float v0, float u1, float v1) {
  // SiLU(u) v = (u v / 2)(1 + tanh(u / 2))
  const float h0 = 0.5f * u0, h1 = 0.5f * u1;
  const float w0 = h0 * v0, w1 = h1 * v1;
  return pack_bf16x2(fmaf(w0, tanh_fast(h0), w0), fmaf(w1, tanh_fast(h1), w1));
}

template <int D>
__global__ void __launch_bounds__(kActThreads, 1)
    action_fuse_kernel(const __grid_constant__ CUtensorMap tm_e,
                       const __grid_constant__ CUtensorMap tm_w1,
                       const __grid_constant__ CUtensorMap tm_w3,
                       const __grid_constant__ CUtensorMap tm_w2,
                       const __grid_constant__ CUtensorMap tm_t1,
                       const __grid_constant__ CUtensorMap tm_t3, const ActArgs a) {
  using Pl = ActPlan<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (tid == 0 && a.flags != nullptr) atomicOr(a.flags, DEVFLAG_SMEM_ALIGN);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Pl::kBars);
  uint64_t* e_full = bars + 0;     // [2]
  uint64_t* e_empty = bars + 2;    // [2]
  uint64_t* oh_full = bars + 4;    // [2]
  uint64_t* uv_full = bars + 6;    // [2]
  uint64_t* epi_done = bars + 8;   // [2]
  uint64_t* y_full = bars + 10;    // [2]
  uint64_t* y_empty = bars + 12;   // [2]
  uint64_t* w13_full = bars + 14;  // [2] W1, W3, T1, T3 of a chunk have landed
  uint64_t* w13_empty = bars + 16; // [2] ... and both slots' U, V products have read them
  uint64_t* w2_full = bars + 18;   // [2] W2 of a chunk has landed
  uint64_t* w2_empty = bars + 20;  // [2] ... and both slots' Y products have read it
  uint64_t* drain = bars + 22;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 23);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  uint32_t* local_flags = tmem_slot + 2;
  if (tid == 0) {
    for (int r = 0; r < 2; ++r) {
      mbar_init(e_full + r, 1);
      mbar_init(e_empty + r, 1);
      mbar_init(oh_full + r, 8);
      mbar_init(uv_full + r, 1);
      mbar_init(epi_done + r, 8);
      mbar_init(y_full + r, 1);
      mbar_init(y_empty + r, 8);
      mbar_init(w13_full + r, 1);
      mbar_init(w13_empty + r, 1);
      mbar_init(w2_full + r, 1);
      mbar_init(w2_empty + r, 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    *local_flags = 0u;
    fence_mbar_init();
  }
  if (warp == 2 && lane < 16) {
    // I_16, the B operand that adds the residual e to Y (one 16-column slice
    // per K-step of E).
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      w[k] = ((lane & 7) >> 1) == (k & 3) && (lane >> 3) == (k >> 2)
                 ? ((lane & 1) ? 0x3F800000u : 0x00003F80u)
                 : 0u;
    st_shared_v4(sbase + Pl::kI + swz32(lane, 0), w[0], w[1], w[2], w[3]);
    st_shared_v4(sbase + Pl::kI + swz32(lane, 1), w[4], w[5], w[6], w[7]);
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  uint32_t* sticky = a.flags != nullptr ? a.flags : local_flags;
  const uint32_t tmem = *tmem_slot;
  const int C = a.chunks;
  const int64_t first = blockIdx.x, step = gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t g = 0;          // chunks whose W2 part is issued
      uint32_t g13 = 0;        // chunks whose W1/W3 part is issued
      uint32_t ep[2] = {0, 0};  // phases of e_full started per slot
      bool e_load[2] = {false, false};  // the latest of them is a TMA load
      bool ok = true;
      for (int64_t p = first, i = 0; ok && p < a.pairs; p += step, ++i) {
        for (int r = 0; r < 2 && ok; ++r) {
          if (i > 0 && !mbar_wait(e_empty + r, (i - 1) & 1, abort_flag, sticky)) {
            ok = false;
            break;
          }
          const int64_t y = (2 * p + r) * 128;
          ++ep[r];
          e_load[r] = y < a.rows;
          if (!e_load[r]) {  // the odd tile past the end: nothing to load, no row is stored
            mbar_arrive(e_full + r);
            continue;
          }
          mbar_arrive_expect_tx(e_full + r, Pl::kEBytes);
#pragma unroll
          for (int b = 0; b < D / 64; ++b)
            tma_load_2d(smem + Pl::kE + r * Pl::kESlot + b * Pl::kEBox, &tm_e, e_full + r, b * 64,
                        static_cast<int32_t>(y));
        }
        for (int c = 0; c < C && ok; ++c, ++g) {
          // Stage g & 1 is reused by chunk g: its W1/W3 part once both U, V
          // products of chunk g - 2 are done, its W2 part once both Y
          // products of chunk g - 2 are done (half a chunk later), so each
          // part loads as early as it can.
          const int s = g & 1;
          uint8_t* st = smem + Pl::kW + s * Pl::kStage;
          if (g >= 2 && !mbar_wait(w13_empty + s, ((g >> 1) + 1) & 1, abort_flag, sticky)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(w13_full + s, Pl::kW13Bytes);
#pragma unroll
          for (int b = 0; b < D / 64; ++b) {
            tma_load_2d(st + Pl::kW13 + b * Pl::kW13Box, &tm_w1, w13_full + s, b * 64, c * kHc);
            tma_load_2d(st + Pl::kW13 + b * Pl::kW13Box + Pl::kWBox, &tm_w3, w13_full + s, b * 64,
                        c * kHc);
          }
          tma_load_2d(st + Pl::kT1, &tm_t1, w13_full + s, 0, c * kHc);
          tma_load_2d(st + Pl::kT3, &tm_t3, w13_full + s, 0, c * kHc);
          ++g13;
          if (g >= 2 && !mbar_wait(w2_empty + s, ((g >> 1) + 1) & 1, abort_flag, sticky)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(w2_full + s, Pl::kW2Bytes);
          tma_load_2d(st + Pl::kW2, &tm_w2, w2_full + s, c * kHc, 0);
        }
      }
      if (!ok) {
        // Let the copies in flight land before the CTA releases its memory:
        // the last phases armed on each full barrier.
        for (uint32_t k = (g13 >= 2 ? g13 - 2 : 0); k < g13; ++k)
          mbar_wait_bounded(w13_full + (k & 1), (k >> 1) & 1);
        for (uint32_t k = (g >= 2 ? g - 2 : 0); k < g; ++k)
          mbar_wait_bounded(w2_full + (k & 1), (k >> 1) & 1);
        for (int r = 0; r < 2; ++r)
          if (e_load[r]) mbar_wait_bounded(e_full + r, (ep[r] - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_uv = idesc_bf16_f32(128, 2 * kHc, 0, 0);
      constexpr uint32_t idesc_y = idesc_bf16_f32(128, D, 0, 0);
      constexpr uint32_t idesc_i = idesc_bf16_f32(128, 16, 0, 0);
      uint32_t g = 0;
      bool ok = true;
      auto mma1 = [&](int r, uint32_t gc) {
        const uint32_t st = sbase + Pl::kW + (gc & 1) * Pl::kStage;
        const uint64_t de = smem_desc(sbase + Pl::kE + r * Pl::kESlot, 16, 1024, 2);
        const uint64_t d13 = smem_desc(st + Pl::kW13, 16, 1024, 2);
        const uint32_t tu = tmem + r * 256;  // U in columns 0-63, V in 64-127
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_bf16_ss(tu, de + kstep(ks, Pl::kEBox), d13 + kstep(ks, Pl::kW13Box), idesc_uv,
                      ks > 0 ? 1u : 0u);
        // The action term: onehot(type) (K = 16) times [T1_c ; T3_c].
        const uint64_t doh = smem_desc(sbase + Pl::kOH + r * 4096, 16, 256, 6);
        mma_bf16_ss(tu, doh, smem_desc(st + Pl::kT1, 16, 256, 6), idesc_uv, 1u);
      };
      // Y[:, 16 ks .. 16 ks + 16) += E[:, 16 ks .. 16 ks + 16) I_16: the residual.
      auto residual = [&](int r) {
        const uint64_t de = smem_desc(sbase + Pl::kE + r * Pl::kESlot, 16, 1024, 2);
        const uint64_t di = smem_desc(sbase + Pl::kI, 16, 256, 6);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_bf16_ss(tmem + r * 256 + 128 + ks * 16, de + kstep(ks, Pl::kEBox), di, idesc_i, 1u);
      };
      // Y += G W2_c with G read from TMEM: hidden columns 32 h .. 32 h + 31
      // are bf16 pairs in U's columns 32 h .. 32 h + 15 (h = 0, 1).
      auto mma2 = [&](int r, uint32_t gc, bool acc) {
        const uint32_t st = sbase + Pl::kW + (gc & 1) * Pl::kStage;
        const uint64_t d2 = smem_desc(st + Pl::kW2, 16, 1024, 2);
#pragma unroll
        for (int ks = 0; ks < kHc / 16; ++ks)
          mma_bf16_ts(tmem + r * 256 + 128, tmem + r * 256 + (ks >> 1) * 32 + (ks & 1) * 8,
                      d2 + kstep(ks, D * 128),
                      idesc_y, (acc || ks > 0) ? 1u : 0u);
      };
      for (int64_t p = first, i = 0; ok && p < a.pairs; p += step, ++i) {
        const uint32_t g0 = g;
        for (int r = 0; r < 2 && ok; ++r)
          ok = mbar_wait(e_full + r, i & 1, abort_flag, sticky) &&
               mbar_wait(oh_full + r, i & 1, abort_flag, sticky);
        if (!ok || !mbar_wait(w13_full + (g0 & 1), (g0 >> 1) & 1, abort_flag, sticky)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int r = 0; r < 2; ++r) {
          mma1(r, g0);
          mma_commit(uv_full + r);
        }
        mma_commit(w13_empty + (g0 & 1));
        for (int c = 0; c < C && ok; ++c) {
          const uint32_t gc = g0 + c;
          for (int r = 0; r < 2 && ok; ++r) {
            if (!mbar_wait(epi_done + r, gc & 1, abort_flag, sticky) ||
                (c == 0 && i > 0 && !mbar_wait(y_empty + r, (i - 1) & 1, abort_flag, sticky)) ||
                (r == 0 && !mbar_wait(w2_full + (gc & 1), (gc >> 1) & 1, abort_flag, sticky))) {
              ok = false;
              break;
            }
            tc_fence_after();
            mma2(r, gc, c > 0);
            if (r == 1) mma_commit(w2_empty + (gc & 1));
            if (c == 0) {
              residual(r);
              if (C == 1) mma_commit(e_empty + r);
            }
            if (c == C - 1) mma_commit(y_full + r);
            if (c + 1 < C) {
              if (r == 0 && !mbar_wait(w13_full + ((gc + 1) & 1), ((gc + 1) >> 1) & 1, abort_flag,
                                       sticky)) {
                ok = false;
                break;
              }
              tc_fence_after();
              mma1(r, gc + 1);
              mma_commit(uv_full + r);
              if (r == 1) mma_commit(w13_empty + ((gc + 1) & 1));
              if (c + 1 == C - 1) mma_commit(e_empty + r);
            }
          }
        }
        g = g0 + C;
      }
      if (!ok) {
        mma_commit(drain);
        mbar_wait_bounded(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int slot = (warp - 2) >> 3;        // warps 2-9 gate slot A, warps 10-17 slot B
    const int q = warp & 3;                  // TMEM lane quadrant
    const int half = ((warp - 2) >> 2) & 1;  // which 32 of the chunk's 64 columns
    const int row = q * 32 + lane;       // row of the tile, TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    bool ok = true;
    // The type id of this thread's row in slot r of pair p (-1 past the end).
    // Loaded a pair ahead of its use, so its latency is hidden.
    auto load_type = [&](int r, int64_t p) -> int {
      const int64_t gr = (2 * p + r) * 128 + row;
      return (half == 0 && p < a.pairs && gr < a.rows) ? static_cast<int>(__ldg(a.types + gr)) : -1;
    };
    auto build_onehot = [&](int r, int t) {
      if (half == 0) {
        if (t >= a.n_types) {
          atomicOr(sticky, DEVFLAG_ACTION_TYPE);
          t = -1;
        }
        uint32_t w[8];  // bf16 1.0 in column t, zeros elsewhere
#pragma unroll
        for (int k = 0; k < 8; ++k)
          w[k] = (t >= 0 && (t >> 1) == k) ? ((t & 1) ? 0x3F800000u : 0x00003F80u) : 0u;
        const uint32_t base = sbase + Pl::kOH + r * 4096;
        st_shared_v4(base + swz32(row, 0), w[0], w[1], w[2], w[3]);
        st_shared_v4(base + swz32(row, 1), w[4], w[5], w[6], w[7]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(oh_full + r);
    };
    const int r = slot;
    uint32_t g = 0;
    for (int64_t p = first, i = 0; ok && p < a.pairs; p += step, ++i) {
      if (i == 0) build_onehot(r, load_type(r, p));
      const int64_t pn = p + step;
      const int tn = load_type(r, pn);
      for (int c = 0; c < C; ++c, ++g) {
        if (!mbar_wait(uv_full + r, g & 1, abort_flag, sticky)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t u[32], v[32];
        tmem_ld32(lane_base + r * 256 + half * 32, u);
        tmem_ld32(lane_base + r * 256 + 64 + half * 32, v);
        tmem_wait_ld();
        tmem_pin32(u);
        tmem_pin32(v);
        // G (this thread's 32 hidden columns as 16 bf16 pairs) goes over the
        // first half of the U columns this thread read, where the Y product
        // reads it as its A operand.
        uint32_t o[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          o[e] = gate_pair(__uint_as_float(u[2 * e]), __uint_as_float(v[2 * e]),
                           __uint_as_float(u[2 * e + 1]), __uint_as_float(v[2 * e + 1]));
        tmem_st16(lane_base + r * 256 + half * 32, o);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(epi_done + r);
        // The last chunk's U, V were this slot's last use of its one-hot
        // rows: build the next pair's now, while the products finish.
        if (c == C - 1 && pn < a.pairs) build_onehot(r, tn);
      }
      if (!ok || !mbar_wait(y_full + r, i & 1, abort_flag, sticky)) {
        ok = false;
        break;
      }
      tc_fence_after();
      constexpr int kCols = D / 2;  // this thread's half of the row
      const int64_t gr0 = (2 * p + r) * 128;
      // Each 32-column chunk goes through the warp's own staging area (row
      // i at 64 i bytes, its four 16-byte units rotated by i / 2 so that a
      // warp's stores spread over the banks), and out as whole 64-byte row
      // pieces, 8 rows per warp store, instead of 16 bytes of 32 rows.
      const uint32_t stg = sbase + Pl::kStg + (warp - 2) * Pl::kStgWarp;
#pragma unroll
      for (int cc = 0; cc < kCols / 32; ++cc) {
        uint32_t y[32];
        tmem_ld32(lane_base + r * 256 + 128 + half * kCols + cc * 32, y);
        tmem_wait_ld();
        tmem_pin32(y);
        if (cc == kCols / 32 - 1) {
          // Y (which already holds e) is in registers: the slot's TMEM is free.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(y_empty + r);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          st_shared_v4(stg + lane * 64 + (((j + (lane >> 1)) & 3) << 4),
                       pack_bf16x2(__uint_as_float(y[8 * j]), __uint_as_float(y[8 * j + 1])),
                       pack_bf16x2(__uint_as_float(y[8 * j + 2]), __uint_as_float(y[8 * j + 3])),
                       pack_bf16x2(__uint_as_float(y[8 * j + 4]), __uint_as_float(y[8 * j + 5])),
                       pack_bf16x2(__uint_as_float(y[8 * j + 6]), __uint_as_float(y[8 * j + 7])));
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int i = it * 8 + (lane >> 2), j = lane & 3;  // staged row i, unit j
          const int64_t gr = gr0 + q * 32 + i;
          if (gr < a.rows) {
            uint32_t v0, v1, v2, v3;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v0), "=r"(v1), "=r"(v2), "=r"(v3)
                         : "r"(stg + i * 64 + (((j + (i >> 1)) & 3) << 4)));
            *reinterpret_cast<uint4*>(a.X + gr * D + half * kCols + cc * 32 + j * 8) =
                make_uint4(v0, v1, v2, v3);
          }
        }
        __syncwarp();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

__global__ void action_prepare_kernel(const float* __restrict__ W1, const float* __restrict__ W3,
                                      const float* __restrict__ W2, const float* __restrict__ table,
                                      int d, int da, int h, int n_types, uint16_t* __restrict__ w13t,
                                      uint16_t* __restrict__ w2t, uint16_t* __restrict__ t13t) {
  const int64_t n_w = static_cast<int64_t>(h) * d;
  const int64_t n_t = static_cast<int64_t>(h) * kMaxTypes;
  const int64_t total = 3 * n_w + 2 * n_t;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (e < 2 * n_w) {  // W1_e^T, W3_e^T: [j][i] = W[i][j], i < d
      const float* W = e < n_w ? W1 : W3;
      const int64_t f = e % n_w, j = f / d, i = f % d;
      w13t[e] = __bfloat16_as_ushort(__float2bfloat16_rn(W[i * h + j]));
    } else if (e < 3 * n_w) {  // W2^T: [c][j] = W2[j][c]
      const int64_t f = e - 2 * n_w, c = f / h, j = f % h;
      w2t[f] = __bfloat16_as_ushort(__float2bfloat16_rn(W2[j * d + c]));
    } else {  // T^T: [j][t] = sum_i table[t][i] W[d + i][j]
      const int64_t f = e - 3 * n_w;
      const float* W = f < n_t ? W1 : W3;
      const int64_t g = f % n_t, j = g / kMaxTypes, t = g % kMaxTypes;
      float s = 0.f;
      if (t < n_types)
        for (int i = 0; i < da; ++i) s = fmaf(table[t * da + i], W[(d + i) * static_cast<int64_t>(h) + j], s);
      t13t[f] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
    }
  }
}

template <int D>
cudaError_t launch_action(const sa_action_s* act, const CUtensorMap& tm_e, const ActArgs& args,
                          cudaStream_t st) {
  using Pl = ActPlan<D>;
  cudaError_t err = cudaFuncSetAttribute(action_fuse_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Pl::kSmem);
  if (err != cudaSuccess) return err;
  const int64_t grid = args.pairs < act->sms ? args.pairs : act->sms;
  action_fuse_kernel<D><<<static_cast<unsigned>(grid), kActThreads, Pl::kSmem, st>>>(
      tm_e, act->tm_w1, act->tm_w3, act->tm_w2, act->tm_t1, act->tm_t3, args);
  return cudaGetLastError();
}

bool al(const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

}  // namespace

void action_info(const sa_action_s* act, int* d, int* device) {
  *d = act->d;
  *device = act->device;
}

sa_status action_fuse_enqueue(const sa_action_s* act, const void* E, const uint8_t* types,
                              int64_t rows, void* X, uint32_t* flags, cudaStream_t st) {
  CUtensorMap tm_e;
  if (!make_tmap_bf16(&tm_e, E, static_cast<uint64_t>(rows), static_cast<uint64_t>(act->d), 128))
    return SA_ERR_CUDA;
  ActArgs args;
  args.types = types;
  args.X = static_cast<uint16_t*>(X);
  args.rows = rows;
  args.pairs = ((rows + 127) / 128 + 1) / 2;
  args.chunks = act->h / kHc;
  args.n_types = act->n_types;
  args.flags = flags;
  const cudaError_t err = act->d == 64 ? launch_action<64>(act, tm_e, args, st)
                                       : launch_action<128>(act, tm_e, args, st);
  return err == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

}  // namespace sa

extern "C" {

sa_status sa_prepare_action(const float* W1, const float* W3, const float* W2,
                            const float* action_table, int d, int d_a, int h, int n_types,
                            void* stream, sa_action* out) {
  if (out == nullptr) return SA_ERR_INVALID_ARG;
  *out = nullptr;
  if (W1 == nullptr || W3 == nullptr || W2 == nullptr || action_table == nullptr ||
      !sa::al(W1, 4) || !sa::al(W3, 4) || !sa::al(W2, 4) || !sa::al(action_table, 4))
    return SA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || d_a < 1 || d_a > 4096 || h < sa::kHc || h > 4096 ||
      h % sa::kHc != 0 || n_types < 1 || n_types > sa::kMaxTypes)
    return SA_ERR_INVALID_ARG;
  int dev = 0, major = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return SA_ERR_CUDA;
  if (major != 10) return SA_ERR_UNSUPPORTED;
  sa_action_s* act = new (std::nothrow) sa_action_s;
  if (act == nullptr) return SA_ERR_CUDA;
  act->device = dev;
  act->sms = sms;
  act->d = d;
  act->h = h;
  act->n_types = n_types;
  act->w13t = act->w2t = act->t13t = nullptr;
  const size_t hd = static_cast<size_t>(h) * d;
  const size_t ht = static_cast<size_t>(h) * sa::kMaxTypes;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool ok = cudaMalloc(&act->w13t, 2 * hd * 2) == cudaSuccess &&
            cudaMalloc(&act->w2t, hd * 2) == cudaSuccess &&
            cudaMalloc(&act->t13t, 2 * ht * 2) == cudaSuccess;
  if (ok) {
    sa::action_prepare_kernel<<<256, 256, 0, st>>>(W1, W3, W2, action_table, d, d_a, h, n_types,
                                                    act->w13t, act->w2t, act->t13t);
    ok = cudaGetLastError() == cudaSuccess &&
         sa::make_tmap_bf16_box(&act->tm_w1, act->w13t, h, d, 64, sa::kHc, 128) &&
         sa::make_tmap_bf16_box(&act->tm_w3, act->w13t + hd, h, d, 64, sa::kHc, 128) &&
         sa::make_tmap_bf16_box(&act->tm_w2, act->w2t, d, h, 64, d, 128) &&
         sa::make_tmap_bf16_box(&act->tm_t1, act->t13t, h, sa::kMaxTypes, 16, sa::kHc, 32) &&
         sa::make_tmap_bf16_box(&act->tm_t3, act->t13t + ht, h, sa::kMaxTypes, 16, sa::kHc, 32);
  }
  if (!ok) {
    cudaFree(act->w13t);
    cudaFree(act->w2t);
    cudaFree(act->t13t);
    delete act;
    return SA_ERR_CUDA;
  }
  *out = act;
  return SA_OK;
}

void sa_action_free(sa_action act) {
  if (act == nullptr) return;
  // Producer kernels enqueued earlier may still read the weights: wait for
  // the producer's device (made current for this call only).
  int prev = -1;
  const bool switched = cudaGetDevice(&prev) == cudaSuccess && prev != act->device &&
                        cudaSetDevice(act->device) == cudaSuccess;
  cudaDeviceSynchronize();
  cudaFree(act->w13t);
  cudaFree(act->w2t);
  cudaFree(act->t13t);
  if (switched) cudaSetDevice(prev);
  delete act;
}

sa_status sa_action_fuse(sa_action act, const void* E, const uint8_t* types, int64_t rows, void* X,
                         uint32_t* device_flags, void* stream) {
  if (act == nullptr || rows < 0 || rows >= (int64_t{1} << 31) - 256) return SA_ERR_INVALID_ARG;
  if (rows == 0) return SA_OK;
  if (E == nullptr || types == nullptr || X == nullptr || !sa::al(E, 16) || !sa::al(X, 16) ||
      !sa::al(device_flags, 4))
    return SA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != act->device) return SA_ERR_INVALID_ARG;
  return sa::action_fuse_enqueue(act, E, types, rows, X, device_flags,
                                 static_cast<cudaStream_t>(stream));
}

}  // extern "C"
