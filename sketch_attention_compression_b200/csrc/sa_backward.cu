// Backward pass of one SA layer on sm_100a (tcgen05 + TMEM + TMA).
//
// Section 2.2 of the SequenceO1 reading notes
// ("SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模") trains the compression
// module end to end through the ranking loss; the page prints no backward,
// so the gradients follow from section 2.1's forward by the chain rule.  In
// the form the forward pass evaluates (S = Q' X^T with Q' = P W_Q W_K^T *
// scale; A the softmax of S over the prototype axis; X~ = A X, m = A 1), for
// a user's upstream gradients G = dL/dX~ (k x d) and g = dL/dm (k):
//   dA  = G X^T + g 1^T
//   dS  = A * (dA - 1 c^T),   c_i = sum_j A_ji dA_ji
//   dX  = A^T G + dS^T Q'
//   R   = dS X = dL/dQ'
// and, from R, dP = scale R W_K W_Q^T, dW_Q = scale P^T R W_K,
// dW_K = scale R^T P W_Q (per-user queries: dQ_b in dP's place).
//
// Per 128-row tile X_t of a user the pass recomputes the forward's softmax
// (no activations are stored) and runs, with the transposed affinities on
// the TMEM lanes as in the forward:
//   MMA1  S^T_t  = X_t Q''^T       M=128 rows, N=k_pad, K=d    (TMEM, fp32)
//   MMA1' dA^T_t = X_t G_b^T       M=128 rows, N=k_pad, K=d    (TMEM, fp32)
//   thread per row: A (exp2 softmax, Q'' = Q' log2 e), c_i, dS' = dS ln 2,
//         both rounded to bf16 into one shared-memory tile [A | dS']
//   MMA3  dX_t   = [A | dS'] [G_b ; Q'']    M=128 rows, N=d, K=2 k_pad
//   MMA4  R_b   += dS'^T X_t                M=k_pad, N=d, K=128 rows
// (dS' Q'' = dS Q', because Q'' = Q' log2 e; R_b collects ln 2 dL/dQ'.)  The
// tile [A | dS'] is the K-major A operand of MMA3 (rows x prototypes) and,
// through a second descriptor, the MN-major A operand of MMA4 (prototypes x
// rows); G_b and Q'' are K-major B operands of MMA1/1' and MN-major B
// operands of MMA3; the X tile is the K-major A of MMA1/1' and the MN-major
// B of MMA4.  TMEM at k = d = 128 holds S^T, dA^T, dX and R: 512 columns.
//
// Rows are split over CTAs as in the forward (sa_internal.h); a user that
// crosses CTA ranges writes R to partial slots that the forward's finalize
// pass sums in a fixed order.  The parameter gradients are small GEMMs over
// R (bwd_gemm_kernel).
#include <cuda_bf16.h>

#include "sa.h"
#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {
namespace {

constexpr int kBwdThreads = 384;  // warps 0-3 roles, 4-11 the softmax group (two warps per row)
constexpr int kBwdStages = 2;
constexpr float kLn2 = 0.6931471805599453f;

template <int D, int KM>
struct BwdPlan {
  static constexpr int kQBox = KM * 128;          // KM rows x 64 bf16
  static constexpr int kXBox = 128 * 128;         // 128 rows x 64 bf16
  static constexpr int kQ = 0;                    // Q'': D / 64 boxes
  static constexpr int kG = kQ + (D / 64) * kQBox;
  static constexpr int kX = kG + (D / 64) * kQBox;          // stages, D / 64 boxes each
  static constexpr int kAS = kX + kBwdStages * (D / 64) * kXBox;  // [A | dS']: 2 KM / 64 boxes
  static constexpr int kGv = kAS + (2 * KM / 64) * kXBox;   // g_b: KM floats
  // Row statistics the two halves of a row swap: [tile parity][half][row]
  // (max, sum of exponentials, sum of exponentials times dA + g, unused).
  static constexpr int kXch = kGv + KM * 4;
  static constexpr int kBars = kXch + 2 * 2 * 128 * 16;
  static constexpr int kSmem = kBars + 256;
  static_assert(kSmem <= 232448, "shared memory budget");
  static constexpr uint32_t kColS = 0, kColDA = KM, kColDX = 2 * KM, kColR = 2 * KM + D;
  static_assert(2 * KM + 2 * D <= 512, "TMEM budget");
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity,
                                          volatile uint32_t* abort_flag, uint32_t* sticky) {
  const bool ok = mbar_wait(bar, parity, abort_flag, sticky);
  return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ void warp_arrive(uint64_t* bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// TMA store of a 2-D box from shared memory (bulk async-group completion),
// and the waits on this thread's outstanding stores.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t x,
                                             int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The stores no longer read shared memory (the source may be overwritten).
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// The stores have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Byte offset of 16-byte unit u of row r in a 128-byte-swizzled box.
__device__ __forceinline__ uint32_t swz(int r, int u) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4);
}

struct BwdArgs {
  PassArgs p;             // offsets, batch, rows, k, d, R -> out_x / part_x, masses -> out_m
  const float* g_pad;     // [batch][KM] (zeros past k)
  uint16_t* dX;           // [N][d] bf16
};

template <int D, int KM, bool FULL>
__global__ void __launch_bounds__(kBwdThreads, 1)
    sa_backward_kernel(const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_g,
                       const __grid_constant__ CUtensorMap tm_dx, const BwdArgs ba) {
  using Pl = BwdPlan<D, KM>;
  constexpr int S = kBwdStages;
  const PassArgs& a = ba.p;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      a.header->flags = 0u;
      a.header->timeout_flags = DEVFLAG_SMEM_ALIGN;
    }
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Pl::kBars);
  uint64_t* x_full = bars;            // [S]
  uint64_t* x_empty = bars + S;       // [S]
  uint64_t* q_full = bars + 2 * S;    // Q'' loaded (once)
  uint64_t* gq_full = q_full + 1;     // this segment's G_b and g_b loaded (TMA + one arrival)
  uint64_t* g_empty = gq_full + 1;    // MMAs done with the segment's G_b, g_b
  uint64_t* s_full = g_empty + 1;     // S^T and dA^T in TMEM
  uint64_t* s_empty = s_full + 1;     // ... read by the softmax group
  uint64_t* p_full = s_empty + 1;     // [A | dS'] stored
  uint64_t* dx_full = p_full + 1;     // dX_t in TMEM (MMA3 done; the tile's MMAs issued)
  uint64_t* dx_empty = dx_full + 1;   // dX_t drained
  uint64_t* r_full = dx_empty + 1;    // [2] by segment parity: R complete
  uint64_t* r_empty = r_full + 2;     // R drained
  uint64_t* xch_full = r_empty + 1;   // [2] by tile parity: both halves' row statistics stored
  uint64_t* as_empty = xch_full + 2;  // MMA3 and MMA4 of a tile have read [A | dS']
  uint64_t* drain = as_empty + 1;     // abort path: the issuer's MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  int64_t* range_slot = reinterpret_cast<int64_t*>(tmem_slot + 2);  // R0, R1, b0
  float* g_s = reinterpret_cast<float*>(smem + Pl::kGv);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t c = blockIdx.x;
  const int64_t N = a.total_rows;
  uint32_t* sticky = &a.header->timeout_flags;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(gq_full, 2);
    mbar_init(g_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(s_empty, 8);
    mbar_init(p_full, 8);
    mbar_init(dx_full, 1);
    mbar_init(dx_empty, 8);
    mbar_init(&r_full[0], 1);
    mbar_init(&r_full[1], 1);
    mbar_init(r_empty, 8);
    mbar_init(&xch_full[0], 8);
    mbar_init(&xch_full[1], 8);
    mbar_init(as_empty, 1);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && !a.keep_flags) {
    a.header->flags = 0u;
    a.header->timeout_flags = 0u;
  }
  if (warp == 0) {
    int64_t b0v, b1v;
    const int64_t r0 = warp_range_begin(a.offsets, a.batch, N, c, G, lane, &b0v);
    const int64_t r1 = warp_range_begin(a.offsets, a.batch, N, c + 1, G, lane, &b1v);
    if (lane == 0) {
      range_slot[0] = r0;
      range_slot[1] = r1;
      range_slot[2] = r0 < r1 ? b0v : a.batch;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t R0 = range_slot[0], R1 = range_slot[1], b0 = range_slot[2];
  const int k = a.k;

  uint32_t tiles_issued = 0, g_loads = 0;
  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      if (!a.user_queries) {
        mbar_arrive_expect_tx(q_full, KM * D * 2);
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_2d(smem + Pl::kQ + cb * Pl::kQBox, &tm_q, q_full, cb * 64, 0);
      }
      const uint64_t pol = policy_evict_first();
      TileCursor cur{SegmentWalker{a.offsets, a.batch, R0, R1, b0}};
      int64_t r;
      uint32_t t = 0;
      while (cur.next(r)) {
        const int st = t % S;
        if (!mbar_wait(&x_empty[st], ((t / S) & 1u) ^ 1u, abort_flag, sticky)) break;
        mbar_arrive_expect_tx(&x_full[st], kTileRows * D * 2);
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_2d_hint(smem + Pl::kX + (st * (D / 64) + cb) * Pl::kXBox, &tm_x, &x_full[st],
                           cb * 64, static_cast<int32_t>(r), pol);
        ++t;
      }
      tiles_issued = t;
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------------- G_b, g_b loader
    SegmentWalker w{a.offsets, a.batch, R0, R1, b0};
    int64_t user, s, e, lo, hi;
    uint32_t gi = 0;
    while (w.next(user, s, e, lo, hi)) {
      if (gi > 0 && !warp_wait(g_empty, (gi - 1) & 1u, abort_flag, sticky)) break;
      if (lane == 0) {
        // G_b, and with per-user queries this user's Q''_b (rows user * KM..
        // of the per-call array; the shared Q'' is loaded once instead).
        mbar_arrive_expect_tx(gq_full, (a.user_queries ? 2 : 1) * KM * D * 2);
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
          tma_load_2d(smem + Pl::kG + cb * Pl::kQBox, &tm_g, gq_full, cb * 64,
                      static_cast<int32_t>(user * KM));
          if (a.user_queries)
            tma_load_2d(smem + Pl::kQ + cb * Pl::kQBox, &tm_q, gq_full, cb * 64,
                        static_cast<int32_t>(user * KM));
        }
      }
      for (int j = lane; j < KM; j += 32) g_s[j] = ba.g_pad[user * KM + j];
      warp_arrive(gq_full, lane);
      ++gi;
    }
    g_loads = gi;
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint64_t xk = smem_desc(sbase + Pl::kX, 16, 1024, 2);       // X as K-major A
      const uint64_t qk = smem_desc(sbase + Pl::kQ, 16, 1024, 2);       // Q'' as K-major B
      const uint64_t gk = smem_desc(sbase + Pl::kG, 16, 1024, 2);       // G_b as K-major B
      const uint64_t ask = smem_desc(sbase + Pl::kAS, 16, 1024, 2);     // [A | dS'] K-major A
      const uint64_t gmn = smem_desc(sbase + Pl::kG, Pl::kQBox, 1024, 2);  // G_b MN-major B
      const uint64_t qmn = smem_desc(sbase + Pl::kQ, Pl::kQBox, 1024, 2);  // Q'' MN-major B
      const uint64_t dsmn =                                                // dS' MN-major A
          smem_desc(sbase + Pl::kAS + (KM / 64) * Pl::kXBox, Pl::kXBox, 1024, 2);
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTileRows, KM, 0, 0);
      constexpr uint32_t idesc_dx = idesc_bf16_f32(kTileRows, D, 0, 1);
      constexpr uint32_t idesc_r = idesc_bf16_f32(KM, D, 1, 1);
      bool ok = a.user_queries || mbar_wait(q_full, 0, abort_flag, sticky);
      SegmentWalker w{a.offsets, a.batch, R0, R1, b0};
      int64_t user, s, e, lo, hi;
      uint32_t t = 0, seg = 0;
      // MMA1 and MMA1' of tile t + 1 are issued as soon as the softmax has
      // read tile t's S^T and dA^T out of TMEM (and before tile t's MMA3 and
      // MMA4, which wait for the softmax to finish), so they run under the
      // softmax of tile t.  A segment's first tile waits for its G_b (and
      // Q''_b), which reuse the previous segment's buffers: no look-ahead
      // across a segment boundary.
      auto issue_s = [&](uint32_t tt) {
        const uint64_t xs = xk + (((tt % S) * (D / 64) * Pl::kXBox) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t ao = ((ks >> 2) * Pl::kXBox + (ks & 3) * 32) >> 4;
          const uint64_t bo = ((ks >> 2) * Pl::kQBox + (ks & 3) * 32) >> 4;
          mma_bf16_ss(tmem + Pl::kColS, xs + ao, qk + bo, idesc_s, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t ao = ((ks >> 2) * Pl::kXBox + (ks & 3) * 32) >> 4;
          const uint64_t bo = ((ks >> 2) * Pl::kQBox + (ks & 3) * 32) >> 4;
          mma_bf16_ss(tmem + Pl::kColDA, xs + ao, gk + bo, idesc_s, ks > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
      };
      bool s_ahead = false;  // MMA1/MMA1' of tile t already issued
      while (ok && w.next(user, s, e, lo, hi)) {
        for (int64_t r = s; r < e; r += kTileRows, ++t) {
          const int st = t % S;
          const bool first = r == s, last = r + kTileRows >= e;
          if (!s_ahead) {
            if ((first && !mbar_wait(gq_full, seg & 1u, abort_flag, sticky)) ||
                !mbar_wait(&x_full[st], (t / S) & 1u, abort_flag, sticky) ||
                (t > 0 && !mbar_wait(s_empty, (t - 1) & 1u, abort_flag, sticky))) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(t);
          }
          s_ahead = false;
          if (!last) {
            if (!mbar_wait(&x_full[(t + 1) % S], ((t + 1) / S) & 1u, abort_flag, sticky) ||
                !mbar_wait(s_empty, t & 1u, abort_flag, sticky)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(t + 1);
            s_ahead = true;
          }
          if (!mbar_wait(p_full, t & 1u, abort_flag, sticky) ||
              (t > 0 && !mbar_wait(dx_empty, (t - 1) & 1u, abort_flag, sticky)) ||
              (first && !mbar_wait(r_empty, (seg & 1u) ^ 1u, abort_flag, sticky))) {
            ok = false;
            break;
          }
          tc_fence_after();
          // MMA3: dX = A G_b + dS' Q'' over K = 2 KM prototypes
#pragma unroll
          for (int ks = 0; ks < 2 * KM / 16; ++ks) {
            const int kk = ks % (KM / 16);
            const uint64_t ao = ((ks >> 2) * Pl::kXBox + (ks & 3) * 32) >> 4;
            const uint64_t bo = (kk * 2048) >> 4;
            mma_bf16_ss(tmem + Pl::kColDX, ask + ao, (ks < KM / 16 ? gmn : qmn) + bo, idesc_dx,
                        ks > 0 ? 1u : 0u);
          }
          mma_commit(dx_full);
          // MMA4: R += dS'^T X_t over the tile's rows
          const uint64_t xmn =
              smem_desc(sbase + Pl::kX + st * (D / 64) * Pl::kXBox, Pl::kXBox, 1024, 2);
#pragma unroll
          for (int ks = 0; ks < kTileRows / 16; ++ks)
            mma_bf16_ss(tmem + Pl::kColR, dsmn + ((ks * 2048) >> 4), xmn + ((ks * 2048) >> 4),
                        idesc_r, (!first || ks > 0) ? 1u : 0u);
          mma_commit(&x_empty[st]);
          mma_commit(as_empty);
          if (last) {
            mma_commit(&r_full[seg & 1u]);
            mma_commit(g_empty);
          }
        }
        ++seg;
      }
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax, dS, drains
    // Two warps per TMEM lane quarter: warp half hf takes prototypes
    // [hf KM/2, (hf + 1) KM/2) of its 32 rows, and the two halves of a row
    // swap (max, sum of exponentials, sum of exponentials times (dA + g))
    // once per tile through shared memory, behind a bounded mbarrier wait.
    const int q = warp & 3;
    const int hf = (warp - 4) >> 2;
    // d = k = 128: whole tiles of dX leave by TMA store from the staging rows.
    constexpr bool kTmaDx = KM == 128 && D == 128;
    const int row = q * 32 + lane;
    constexpr int HW = KM / 2, HC = HW / 32;
    const int j0 = hf * HW;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    float4* xch = reinterpret_cast<float4*>(smem + Pl::kXch);
    SegmentWalker w{a.offsets, a.batch, R0, R1, b0};
    // Software-pipelined over tiles: while MMA3 and MMA4 of tile t run, the
    // group already loads tile t + 1's logits and takes their exponentials;
    // only then does it drain dX_t.  (The issuer has started MMA1 of tile
    // t + 1 once the group released tile t's S^T and dA^T.)
    uint32_t sv[HC][32];   // the current tile's exponentials (as float bits)
    float mx = -INFINITY, z = 0.f;
    // Loads this half's logits of the tile now in S^T and takes its
    // maximum and exponentials (exp2 softmax: Q'' carries log2 e).
    auto load_exps = [&]() {
#pragma unroll
      for (int cc = 0; cc < HC; ++cc) tmem_ld32(lane_addr + Pl::kColS + j0 + cc * 32, sv[cc]);
      tmem_wait_ld();
#pragma unroll
      for (int cc = 0; cc < HC; ++cc) tmem_pin32(sv[cc]);
      mx = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < HC; ++cc)
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (FULL || j0 + cc * 32 + i < k) mx = fmaxf(mx, __uint_as_float(sv[cc][i]));
      z = 0.f;
#pragma unroll
      for (int cc = 0; cc < HC; ++cc)
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float ev =
              (FULL || j0 + cc * 32 + i < k) ? ex2_approx(__uint_as_float(sv[cc][i]) - mx) : 0.f;
          sv[cc][i] = __float_as_uint(ev);
          z += ev;
        }
    };
    int64_t user, s, e, lo, hi;
    bool ok = w.next(user, s, e, lo, hi);
    int64_t r = s;
    uint32_t t = 0, seg = 0;
    bool have_s = false;
    while (ok) {
      const bool first = r == s, last = r + kTileRows >= e;
      const int nrows = static_cast<int>((e - r) < kTileRows ? (e - r) : kTileRows);
      const bool valid = row < nrows;
      const int st = t % S;
      if (!have_s) {
        if ((first && !warp_wait(gq_full, seg & 1u, abort_flag, sticky)) ||
            !warp_wait(s_full, t & 1u, abort_flag, sticky)) {
          ok = false;
          break;
        }
        tc_fence_after();
        load_exps();
      }
      // dA of this half (dv becomes dA + g, g_b read four at a time); then
      // S^T and dA^T are free for the next tile's MMA1.
      uint32_t dv[HC][32];
#pragma unroll
      for (int cc = 0; cc < HC; ++cc) tmem_ld32(lane_addr + Pl::kColDA + j0 + cc * 32, dv[cc]);
      tmem_wait_ld();
#pragma unroll
      for (int cc = 0; cc < HC; ++cc) tmem_pin32(dv[cc]);
      tc_fence_before();
      warp_arrive(s_empty, lane);
      float wsum = 0.f;
#pragma unroll
      for (int cc = 0; cc < HC; ++cc) {
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 g4 = reinterpret_cast<const float4*>(g_s + j0 + cc * 32)[i4];
          const float gg[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
          for (int i1 = 0; i1 < 4; ++i1) {
            const int i = i4 * 4 + i1;
            const float dg = __uint_as_float(dv[cc][i]) + gg[i1];
            dv[cc][i] = __float_as_uint(dg);
            wsum = fmaf(__uint_as_float(sv[cc][i]), dg, wsum);
          }
        }
      }
      const uint32_t par = t & 1u;
      xch[(par * 2 + hf) * 128 + row] = make_float4(mx, z, wsum, 0.f);
      warp_arrive(&xch_full[par], lane);
      if (!warp_wait(&xch_full[par], (t >> 1) & 1u, abort_flag, sticky)) {
        ok = false;
        break;
      }
      const float4 o = xch[(par * 2 + (hf ^ 1)) * 128 + row];
      // Combine: M = max of both halves; a half with no prototype has max
      // -inf and contributes nothing.
      const float M = fmaxf(mx, o.x);
      const float sa_own = mx == -INFINITY ? 0.f : ex2_approx(mx - M);
      const float sa_oth = o.x == -INFINITY ? 0.f : ex2_approx(o.x - M);
      const float Z = z * sa_own + o.y * sa_oth;
      const float inv = valid ? 1.0f / Z : 0.f;
      const float scale = sa_own * inv;
      const float cs = (wsum * sa_own + o.z * sa_oth) * inv;
      // The shared tile is free once the previous tile's MMA3 and MMA4
      // have read it.
      if (t > 0 && !warp_wait(as_empty, (t - 1) & 1u, abort_flag, sticky)) {
        ok = false;
        break;
      }
      // This warp's dX store of the previous tile may still read its staging
      // rows (in the box about to be written).
      if (kTmaDx) {
        if (lane == 0) bulk_wait_read();
        __syncwarp();
      }
      // A and dS' = ln2 A (dA + g - c) of this half, into the shared tile
      // (A in the first KM / 64 boxes, dS' in the others).
#pragma unroll
      for (int cc = 0; cc < HC; ++cc) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t wa[4], wd[4];
#pragma unroll
          for (int ee = 0; ee < 4; ++ee) {
            const int i = u * 8 + 2 * ee;
            const float a0 = valid ? __uint_as_float(sv[cc][i]) * scale : 0.f;
            const float a1 = valid ? __uint_as_float(sv[cc][i + 1]) * scale : 0.f;
            const float d0 = kLn2 * a0 * (__uint_as_float(dv[cc][i]) - cs);
            const float d1 = kLn2 * a1 * (__uint_as_float(dv[cc][i + 1]) - cs);
            wa[ee] = pack_bf16x2(a0, a1);
            wd[ee] = valid ? pack_bf16x2(d0, d1) : 0u;
          }
          const int col = j0 + cc * 32 + u * 8;  // prototype of the unit's first element
          const uint32_t ua = sbase + Pl::kAS + (col >> 6) * Pl::kXBox + swz(row, (col & 63) >> 3);
          const uint32_t ud = ua + (KM / 64) * Pl::kXBox;
          st_shared_v4(ua, wa[0], wa[1], wa[2], wa[3]);
          st_shared_v4(ud, wd[0], wd[1], wd[2], wd[3]);
        }
      }
      if (!valid && (D / 64 > 1 || hf == 0)) {
        // Rows past the segment's end: cleared (0 * NaN is NaN in MMA4);
        // each half clears one 64-column box (d = 64: the first half).
        const int cb = D / 64 > 1 ? hf : 0;
        const uint32_t xrow = sbase + Pl::kX + (st * (D / 64) + cb) * Pl::kXBox + row * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i) st_shared_v4(xrow + i * 16, 0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      warp_arrive(p_full, lane);

      // The next tile (the next segment's first after a segment's last):
      // its logits and exponentials, while MMA3 and MMA4 of this tile run.
      int64_t nu = user, ns = s, ne = e, nlo = lo, nhi = hi, nr = r + kTileRows;
      bool has_next = true;
      if (last) {
        has_next = w.next(nu, ns, ne, nlo, nhi);
        nr = ns;
      }
      have_s = false;
      if (has_next) {
        if ((last && !warp_wait(gq_full, (seg + 1) & 1u, abort_flag, sticky)) ||
            !warp_wait(s_full, (t + 1) & 1u, abort_flag, sticky)) {
          ok = false;
          break;
        }
        tc_fence_after();
        load_exps();
        have_s = true;
      }

      // dX_t: TMEM row -> bf16 -> global; each half drains d / 2 columns
      // (all of its 32-column loads in flight before one wait).  With 128 prototypes the warp stages its 32 rows in
      // the part of the [A | dS'] tile that it alone writes (A's box hf,
      // rows 32 q ..), free once MMA3 has read it, then stores whole rows:
      // 128 (d = 64: 64) bytes of a row per 8 (4) lanes, instead of 16
      // bytes of 32 rows.  With 64 prototypes both halves write each A and
      // dS' box, so the rows go straight from registers.
      if (!warp_wait(dx_full, t & 1u, abort_flag, sticky)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        constexpr int XC = D / 64;  // 32-column chunks per half
        constexpr int U = D / 16;   // 16-byte units per half row
        const uint32_t box = sbase + Pl::kAS + hf * Pl::kXBox;
        uint32_t xall[XC][32];
#pragma unroll
        for (int cc = 0; cc < XC; ++cc)
          tmem_ld32(lane_addr + Pl::kColDX + hf * (D / 2) + cc * 32, xall[cc]);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < XC; ++cc) tmem_pin32(xall[cc]);
        tc_fence_before();
        warp_arrive(dx_empty, lane);
#pragma unroll
        for (int cc = 0; cc < XC; ++cc) {
          const uint32_t (&xv)[32] = xall[cc];
          if constexpr (KM == 64) {
            if (valid) {
              uint4* dst = reinterpret_cast<uint4*>(ba.dX + (r + row) * D + hf * (D / 2) + cc * 32);
#pragma unroll
              for (int u = 0; u < 4; ++u)
                dst[u] = make_uint4(pack_bf16x2(__uint_as_float(xv[8 * u]), __uint_as_float(xv[8 * u + 1])),
                                    pack_bf16x2(__uint_as_float(xv[8 * u + 2]), __uint_as_float(xv[8 * u + 3])),
                                    pack_bf16x2(__uint_as_float(xv[8 * u + 4]), __uint_as_float(xv[8 * u + 5])),
                                    pack_bf16x2(__uint_as_float(xv[8 * u + 6]), __uint_as_float(xv[8 * u + 7])));
            }
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              st_shared_v4(box + swz(row, cc * 4 + u),
                           pack_bf16x2(__uint_as_float(xv[8 * u]), __uint_as_float(xv[8 * u + 1])),
                           pack_bf16x2(__uint_as_float(xv[8 * u + 2]), __uint_as_float(xv[8 * u + 3])),
                           pack_bf16x2(__uint_as_float(xv[8 * u + 4]), __uint_as_float(xv[8 * u + 5])),
                           pack_bf16x2(__uint_as_float(xv[8 * u + 6]), __uint_as_float(xv[8 * u + 7])));
          }
        }
        if (kTmaDx && nrows == kTileRows) {
          // A whole tile: one TMA store of the warp's 32 staged rows.
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm_dx, box + q * 4096, hf * (D / 2), static_cast<int32_t>(r + q * 32));
            bulk_commit();
          }
        } else if constexpr (KM == 128) {
          __syncwarp();
          constexpr int RPI = 32 / U;  // rows per warp store
#pragma unroll
          for (int it = 0; it < U; ++it) {
            const int rr = q * 32 + it * RPI + lane / U;
            const int u = lane % U;
            if (rr < nrows) {
              const uint4 v = ld_shared_v4u(box + swz(rr, u));
              *reinterpret_cast<uint4*>(ba.dX + (r + rr) * D + hf * (D / 2) + u * 8) = v;
            }
          }
          __syncwarp();
        }
      }

      if (last) {
        // R_b (ln 2 dL/dQ') to the outputs or to this user's partial slot;
        // the mass outputs carry zeros.  Each half drains d / 2 columns.
        if (!warp_wait(&r_full[seg & 1u], (seg >> 1) & 1u, abort_flag, sticky)) { ok = false; break; }
        tc_fence_after();
        const int64_t slotp = segment_slot(c, lo, hi, R0, R1);
        float* dm = slotp < 0 ? a.out_m + user * a.k : a.part_m + slotp * a.k;
        float* dr = slotp < 0 ? a.out_x + user * a.k * D : a.part_x + slotp * a.k * D;
        const int j = (KM == 128 ? q * 32 : q * 16) + lane;
        const bool has = (KM == 128 || lane < 16) && j < k;
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc) {
          uint32_t v[32];
          tmem_ld32(lane_addr + Pl::kColR + hf * (D / 2) + cc * 32, v);
          tmem_wait_ld();
          tmem_pin32(v);
          if (has) {
            float4* dst = reinterpret_cast<float4*>(dr + static_cast<int64_t>(j) * D + hf * (D / 2) +
                                                    cc * 32);
#pragma unroll
            for (int w4 = 0; w4 < 8; ++w4)
              dst[w4] = make_float4(__uint_as_float(v[4 * w4]), __uint_as_float(v[4 * w4 + 1]),
                                    __uint_as_float(v[4 * w4 + 2]), __uint_as_float(v[4 * w4 + 3]));
          }
        }
        if (has && hf == 0) dm[j] = 0.f;
        tc_fence_before();
        warp_arrive(r_empty, lane);
      }
      if (!has_next) break;
      if (last) ++seg;
      user = nu;
      s = ns;
      e = ne;
      lo = nlo;
      hi = nhi;
      r = nr;
      ++t;
    }
    // This warp's last dX stores complete before the CTA exits.
    if (kTmaDx && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // A wait gave up: let issued copies and MMAs finish before the tensor
    // memory is released.
    if (warp == 0 && lane == 0) {
      const uint32_t t = tiles_issued;
      for (uint32_t u = (t > static_cast<uint32_t>(S) ? t - S : 0u); u < t; ++u)
        mbar_wait_bounded(&x_full[u % S], (u / S) & 1u);
      if (!a.user_queries) mbar_wait_bounded(q_full, 0);
    }
    if (warp == 2 && lane == 0 && g_loads > 0) mbar_wait_bounded(gq_full, (g_loads - 1) & 1u);
    if (warp == 1 && lane == 0) {
      mma_commit(drain);
      mbar_wait_bounded(drain, 0);
    }
    tc_fence_before();
    __syncthreads();
  }
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// G (batch x k x d fp32) -> bf16 rows of KM per user (rows >= k zero), and
// g (batch x k, or none) -> fp32 rows of KM (zeros past k).
__global__ void bwd_prep_kernel(const float* __restrict__ Gin, const float* __restrict__ gin,
                                int64_t batch, int k, int km, int d, uint16_t* __restrict__ Gb,
                                float* __restrict__ gp) {
  const int64_t n = batch * km * d;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = e / (static_cast<int64_t>(km) * d);
    const int j = static_cast<int>((e / d) % km);
    const int f = static_cast<int>(e % d);
    const float v = j < k ? Gin[(b * k + j) * d + f] : 0.f;
    Gb[e] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    if (f == 0) gp[b * km + j] = (gin != nullptr && j < k) ? gin[b * k + j] : 0.f;
  }
}

}  // namespace

// out = sum over b of R[b] (n entries each), fp64 accumulation in user order.
__global__ void sum_users_kernel(const float* __restrict__ R, int64_t batch, int64_t n,
                                 float* __restrict__ out) {
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    double s = 0.0;
    for (int64_t b = 0; b < batch; ++b) s += R[b * n + e];
    out[e] = static_cast<float>(s);
  }
}

cudaError_t launch_sum_users(const float* R, int64_t batch, int64_t n, float* out,
                             cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
  sum_users_kernel<<<grid, 256, 0, st>>>(R, batch, n, out);
  return cudaGetLastError();
}

// C[b] = alpha * op(A[b]) op(B[b]) (+ C[b] when accumulate), row-major, fp64
// accumulation; op transposes when the flag is set.  A[b] is m x l after
// op, B[b] is l x n after op; `batch` independent products (strides 0 for a
// shared operand).  Small products only (the parameter gradients).
// Tiles of 32 x 32 outputs per block of 16 x 16 threads (2 x 2 each), the
// shared dimension in steps of 32 through shared memory, loads coalesced
// along whichever index is contiguous in memory.
constexpr int kGemmTile = 32;

__global__ void __launch_bounds__(256)
    bwd_gemm_kernel(const float* __restrict__ A, int64_t sa, bool ta, const float* __restrict__ B,
                    int64_t sb, bool tb, float* __restrict__ C, int64_t sc, int m, int n, int l,
                    double alpha, bool accumulate) {
  __shared__ float As[kGemmTile][kGemmTile + 1];  // [i][p]
  __shared__ float Bs[kGemmTile][kGemmTile + 1];  // [p][j]
  const int64_t b = blockIdx.z;
  const float* Ab = A + b * sa;
  const float* Bb = B + b * sb;
  float* Cb = C + b * sc;
  const int i0 = blockIdx.y * kGemmTile, j0 = blockIdx.x * kGemmTile;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double acc[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
  for (int p0 = 0; p0 < l; p0 += kGemmTile) {
    for (int idx = threadIdx.x; idx < kGemmTile * kGemmTile; idx += 256) {
      const int x = idx % kGemmTile, y = idx / kGemmTile;  // x runs along contiguous memory
      {
        const int ii = ta ? x : y, pp = ta ? y : x;
        const int gi = i0 + ii, gp = p0 + pp;
        As[ii][pp] = (gi < m && gp < l)
                         ? (ta ? Ab[static_cast<int64_t>(gp) * m + gi] : Ab[static_cast<int64_t>(gi) * l + gp])
                         : 0.f;
      }
      {
        const int pp = tb ? x : y, jj = tb ? y : x;
        const int gp = p0 + pp, gj = j0 + jj;
        Bs[pp][jj] = (gp < l && gj < n)
                         ? (tb ? Bb[static_cast<int64_t>(gj) * l + gp] : Bb[static_cast<int64_t>(gp) * n + gj])
                         : 0.f;
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int pp = 0; pp < kGemmTile; ++pp) {
      const double a0 = As[2 * ty][pp], a1 = As[2 * ty + 1][pp];
      const double b0 = Bs[pp][2 * tx], b1 = Bs[pp][2 * tx + 1];
      acc[0][0] = fma(a0, b0, acc[0][0]);
      acc[0][1] = fma(a0, b1, acc[0][1]);
      acc[1][0] = fma(a1, b0, acc[1][0]);
      acc[1][1] = fma(a1, b1, acc[1][1]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int i = i0 + 2 * ty + u, j = j0 + 2 * tx + v;
      if (i < m && j < n) {
        const int64_t e = static_cast<int64_t>(i) * n + j;
        const double r = alpha * acc[u][v];
        Cb[e] = static_cast<float>(accumulate ? Cb[e] + r : r);
      }
    }
}

cudaError_t launch_bwd_gemm(const float* A, int64_t sa, bool ta, const float* B, int64_t sb,
                            bool tb, float* C, int64_t sc, int m, int n, int l, double alpha,
                            bool accumulate, int64_t batch, cudaStream_t st) {
  for (int64_t b0 = 0; b0 < batch; b0 += 65535) {  // grid z is at most 65535
    const int64_t nb = batch - b0 < 65535 ? batch - b0 : 65535;
    const dim3 grid(static_cast<unsigned>((n + kGemmTile - 1) / kGemmTile),
                    static_cast<unsigned>((m + kGemmTile - 1) / kGemmTile), static_cast<unsigned>(nb));
    bwd_gemm_kernel<<<grid, 256, 0, st>>>(A + b0 * sa, sa, ta, B + b0 * sb, sb, tb, C + b0 * sc, sc, m,
                                          n, l, alpha, accumulate);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

cudaError_t launch_bwd_prep(const float* G, const float* g, int64_t batch, int k, int km, int d,
                            uint16_t* Gb, float* gp, cudaStream_t st) {
  const int64_t n = batch * km * d;
  const unsigned grid = static_cast<unsigned>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  if (n == 0) return cudaSuccess;
  bwd_prep_kernel<<<grid, 256, 0, st>>>(G, g, batch, k, km, d, Gb, gp);
  return cudaGetLastError();
}

namespace {
template <int D, int KM>
cudaError_t launch_bwd_one(const CUtensorMap& tx, const CUtensorMap& tq, const CUtensorMap& tg,
                           const BwdArgs& ba, int grid, cudaStream_t st) {
  using Pl = BwdPlan<D, KM>;
  auto kern = ba.p.k == KM ? sa_backward_kernel<D, KM, true> : sa_backward_kernel<D, KM, false>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Pl::kSmem);
  if (err != cudaSuccess) return err;
  // dX as 32-row x 64-column boxes (one warp's rows of one half), 128-byte
  // swizzle: the layout the drain stages them in.
  CUtensorMap tdx;
  if (ba.p.total_rows > 0 &&
      !make_tmap_bf16_box(&tdx, ba.dX, static_cast<uint64_t>(ba.p.total_rows), static_cast<uint64_t>(D),
                          64, 32, 128))
    return cudaErrorInvalidValue;
  if (ba.p.total_rows == 0) tdx = tx;  // unused: no tile is drained
  kern<<<grid, kBwdThreads, Pl::kSmem, st>>>(tx, tq, tg, tdx, ba);
  return cudaGetLastError();
}
}  // namespace

bool backward_supported(int d, int k_pad) {
  return (d == 64 || d == 128) && (k_pad == 64 || k_pad == 128);
}

cudaError_t launch_backward(const CUtensorMap& tx, const CUtensorMap& tq, const CUtensorMap& tg,
                            int k_pad, const PassArgs& p, const float* g_pad, uint16_t* dX,
                            int grid, cudaStream_t st) {
  BwdArgs ba;
  ba.p = p;
  ba.g_pad = g_pad;
  ba.dX = dX;
  if (p.d == 64 && k_pad == 64) return launch_bwd_one<64, 64>(tx, tq, tg, ba, grid, st);
  if (p.d == 64 && k_pad == 128) return launch_bwd_one<64, 128>(tx, tq, tg, ba, grid, st);
  if (p.d == 128 && k_pad == 64) return launch_bwd_one<128, 64>(tx, tq, tg, ba, grid, st);
  if (p.d == 128 && k_pad == 128) return launch_bwd_one<128, 128>(tx, tq, tg, ba, grid, st);
  return cudaErrorInvalidValue;
}

}  // namespace sa
