// Fused SA pass for bf16 histories on sm_100a (tcgen05 + TMEM + TMA).
//
// One SA layer (section 2.1 "Sketch Attention" of the SequenceO1 reading
// notes, "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模"), computed the
// way section 2.4 describes FlashSA: affinity, stable softmax statistics and
// aggregation are tiled together so that the k x n score and assignment
// matrices never reach HBM, over batches of unequal lengths.
//
// Per 128-row tile X_t of one user (rows i, prototypes j):
//   MMA1  S^T_t = X_t Q'^T          M=128 rows, N=k_pad, K=d   (TMEM, fp32)
//   softmax over j, one thread per row i (the prototype axis lies along
//         the thread's own TMEM lane, so no cross-thread reduction):
//         a_ji = exp2(s_ji - max_j s_ji) / sum_j exp2(...)     (log2 e is in Q')
//         rounded to bf16 and stored to shared memory as the A operand of
//   MMA2  X~ += A_t X_t             M=k_pad, N=d, K=128        (TMEM, fp32)
//   MASS  m  += A_t 1               M=k_pad, N=16, K=128       (TMEM, fp32)
// The X tile in shared memory serves as the K-major A operand of MMA1 and
// as the MN-major B operand of MMA2; X is read from HBM once.
//
// Warp roles (384 threads):
//   warp 0      TMA producer (X ring of kStages tiles; Q' once)
//   warp 1      MMA issuer (one thread); MMA2 of tile t is issued after MMA1
//               of tile t+1 so that the softmax of t overlaps MMA1 of t+1
//   warp 2      TMEM allocation / release
//   warps 4-7   softmax group 0 (even tiles)
//   warps 8-11  softmax group 1 (odd tiles)
// The group that finishes a segment's last tile also drains the TMEM
// accumulator to the outputs (or to a partial slot for split users).
#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {
namespace {

constexpr int kThreads = 384;
constexpr int kRing = 16;  // issuer's ring of in-flight tile descriptors
constexpr int kMaxDynSmem = 232448;  // 227 KB per block on sm_100

template <int D, int KM>
struct Cfg {
  static constexpr int kQBytes = KM * D * 2;                // Q' (bf16), D/64 swizzled boxes
  static constexpr int kXBytes = kTileRows * D * 2;         // one X tile
  static constexpr int kPBytes = KM * kTileRows * 2;        // one probability tile
  static constexpr int kFixed = kQBytes + 2 * kPBytes + 1024 + 1024;  // + ones/barriers + align
  static constexpr int kStagesFit = (kMaxDynSmem - kFixed) / kXBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kSmem = kFixed + kStages * kXBytes;
  // TMEM columns (128 lanes x 512 columns of 32 bit are allocated)
  static constexpr uint32_t kColS = 0;              // two S^T buffers: [0,KM), [KM,2KM)
  static constexpr uint32_t kColAcc = 2 * KM;       // X~ accumulator, D columns
  static constexpr uint32_t kColMass = 2 * KM + D;  // mass accumulator, 16 columns
  static_assert(kColMass + 16 <= 512, "TMEM budget");
  static_assert(kStages >= 2, "shared memory budget");
  static_assert(kSmem <= kMaxDynSmem, "shared memory budget");
  static_assert(D % 64 == 0 && (KM == 64 || KM == 128), "shape");
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Warp-wide wait: every lane polls, and the warp leaves converged with one
// common verdict (tcgen05.ld that follows is .sync.aligned).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity,
                                          volatile uint32_t* abort_flag, uint32_t* sticky) {
  const bool ok = mbar_wait(bar, parity, abort_flag, sticky);
  return __all_sync(0xFFFFFFFFu, ok);
}

// FULL: k == KM, so no prototype column needs masking.
template <int D, int KM, bool FULL>
__global__ void __launch_bounds__(kThreads, 1)
    fused_sa_kernel(const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_q, const PassArgs a) {
  using C = Cfg<D, KM>;
  constexpr int S = C::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* q_s = smem;
  uint8_t* x_s = q_s + C::kQBytes;
  uint8_t* p_s = x_s + S * C::kXBytes;
  uint8_t* ones_s = p_s + 2 * C::kPBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ones_s + 512);
  uint64_t* x_full = bars;
  uint64_t* x_empty = bars + S;
  uint64_t* s_full = bars + 2 * S;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* p_empty = p_full + 2;
  // Two acc_full barriers, used by segment parity.  A softmax group that
  // waits for segment s cannot see a stale parity: segment s-2's
  // aggregation was issued before the MMA1 whose completion let the group
  // reach this tile, so that earlier phase of acc_full[s & 1] has completed.
  uint64_t* acc_full = p_empty + 2;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* q_full = acc_empty + 1;
  uint64_t* drain = q_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  int64_t* b0_slot = reinterpret_cast<int64_t*>(tmem_slot + 2);
  uint32_t* tile_ring = reinterpret_cast<uint32_t*>(b0_slot + 1);  // issuer's tile descriptors

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t c = blockIdx.x;
  const int64_t N = a.total_rows;
  const int64_t R0 = cta_row_begin(c, G, a.tiles, N);
  const int64_t R1 = cta_row_begin(c + 1, G, a.tiles, N);
  uint32_t* sticky = &a.header->timeout_flags;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&x_full[i], 1); mbar_init(&x_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_full[1], 1);
    mbar_init(acc_empty, 128);
    mbar_init(q_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    *b0_slot = (a.batch > 0 && R0 < R1) ? user_at_or_before(a.offsets, a.batch, R0) : a.batch;
    if (c == 0) { a.header->flags = 0u; a.header->timeout_flags = 0u; }
    fence_mbar_init();
  }
  if (threadIdx.x < 128) {  // 512 B of bf16 ones: B operand of the mass MMA
    reinterpret_cast<uint32_t*>(ones_s)[threadIdx.x] = 0x3F803F80u;
    fence_proxy_async_smem();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t b0 = *b0_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
      for (int cb = 0; cb < D / 64; ++cb)
        tma_load_2d(q_s + cb * KM * 128, &tm_q, q_full, cb * 64, 0);
      SegmentWalker w{a.offsets, a.batch, R0, R1, b0};
      int64_t user, s, e, lo, hi;
      uint32_t t = 0;
      bool ok = true;
      while (ok && w.next(user, s, e, lo, hi)) {
        for (int64_t r = s; r < e; r += kTileRows) {
          const int st = t % S;
          if (!mbar_wait(&x_empty[st], ((t / S) & 1u) ^ 1u, abort_flag, sticky)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&x_full[st], C::kXBytes);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_2d_hint(x_s + st * C::kXBytes + cb * 16384, &tm_x, &x_full[st], cb * 64,
                             static_cast<int32_t>(r), pol);
          ++t;
        }
      }
      if (!ok) {  // let the copies in flight land before the CTA exits
        for (uint32_t u = (t > static_cast<uint32_t>(S) ? t - S : 0u); u < t; ++u)
          mbar_wait_bounded(&x_full[u % S], (u / S) & 1u);
        mbar_wait_bounded(q_full, 0);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTileRows, KM, 0, 0);
      constexpr uint32_t idesc_x = idesc_bf16_f32(KM, D, 1, 1);
      constexpr uint32_t idesc_m = idesc_bf16_f32(KM, 16, 1, 0);
      const uint32_t q_a = smem_u32(q_s);
      const uint32_t x_a = smem_u32(x_s);
      const uint32_t p_a = smem_u32(p_s);
      const uint64_t ones_desc = smem_desc(smem_u32(ones_s), 128, 256, 0);
      // Base descriptors, built once.  A byte offset b within shared memory
      // is applied by adding b >> 4 to the start-address field (bits 0-13);
      // every address stays below 2^18 bytes, so the field never carries.
      // This keeps the issuing thread to one add per MMA: its own scalar
      // latency would otherwise pace the tensor pipe.
      const uint64_t xk_desc = smem_desc(x_a, 16, 1024, 2);      // X as K-major A
      const uint64_t q_desc = smem_desc(q_a, 16, 1024, 2);       // Q' as K-major B
      const uint64_t p_desc = smem_desc(p_a, 16384, 1024, 2);    // P as MN-major A
      const uint64_t xmn_desc = smem_desc(x_a, 16384, 1024, 2);  // X as MN-major B
      bool ok = mbar_wait(q_full, 0, abort_flag, sticky);
      tc_fence_after();

      // Non-blocking scheduler with two cursors over the CTA's tiles:
      //   t1: next tile whose affinity MMA (MMA1) is issued, as soon as its X
      //       stage has landed and its S^T buffer has been read out;
      //   t2: next tile whose aggregation (MMA2 + mass) is issued, as soon as
      //       its probabilities are in shared memory (and, for the first
      //       tile of a user segment, the accumulator has been drained).
      // MMA1 thus runs ahead of the softmax instead of waiting for the
      // previous tile's aggregation.  The tensor pipe executes the issued
      // MMAs in order.
      // Tile descriptors of issued-but-not-aggregated tiles, in shared memory:
      // bits 0-7 stage, bit 8 first of segment, bit 9 last, bits 10+ segment.
      static_assert(kRing >= S + 2, "tile ring");
      SegmentWalker w{a.offsets, a.batch, R0, R1, b0};
      int64_t user = 0, s = 0, e = 0, lo = 0, hi = 0, r = 0;
      bool have_seg = false, walker_done = false;
      uint32_t t1 = 0, t2 = 0, seg = 0;
      long long idle_since = cycles_now();
      while (ok) {
        bool progressed = false;
        // ---- MMA1 for tile t1
        if (!walker_done) {
          if (!have_seg) {
            have_seg = w.next(user, s, e, lo, hi);
            if (have_seg) r = s; else walker_done = true;
          }
          if (have_seg) {
            const int st = t1 % S;
            const int sb = t1 & 1;
            if (mbar_test_wait(&x_full[st], (t1 / S) & 1u) &&
                mbar_test_wait(&s_empty[sb], ((t1 >> 1) & 1u) ^ 1u)) {
              tc_fence_after();
              const uint64_t xd = xk_desc + ((st * C::kXBytes) >> 4);
              const uint32_t dcol = tmem + C::kColS + sb * KM;
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks) {
                mma_bf16_ss(dcol, xd + (((ks >> 2) * 16384 + (ks & 3) * 32) >> 4),
                            q_desc + (((ks >> 2) * (KM * 128) + (ks & 3) * 32) >> 4), idesc_s,
                            ks > 0 ? 1u : 0u);
              }
              mma_commit(&s_full[sb]);
              tile_ring[t1 % kRing] = static_cast<uint32_t>(st) | (r == s ? 0x100u : 0u) |
                                      (r + kTileRows >= e ? 0x200u : 0u) | (seg << 10);
              ++t1;
              r += kTileRows;
              if (r >= e) { have_seg = false; ++seg; }
              progressed = true;
            }
          }
        }
        // ---- MMA2 + mass for tile t2
        if (t2 < t1) {
          const uint32_t desc = tile_ring[t2 % kRing];
          const bool first = desc & 0x100u;
          const bool last = desc & 0x200u;
          const uint32_t sg = desc >> 10;
          const int pb = t2 & 1;
          if (mbar_test_wait(&p_full[pb], (t2 >> 1) & 1u) &&
              (!first || mbar_test_wait(acc_empty, (sg & 1u) ^ 1u))) {
            tc_fence_after();
            const int st = static_cast<int>(desc & 0xFFu);
            const uint64_t pd = p_desc + ((pb * C::kPBytes) >> 4);
            const uint64_t xd = xmn_desc + ((st * C::kXBytes) >> 4);
            const uint32_t acc0 = (!first) ? 1u : 0u;
#pragma unroll
            for (int ks = 0; ks < kTileRows / 16; ++ks)
              mma_bf16_ss(tmem + C::kColAcc, pd + ((ks * 2048) >> 4), xd + ((ks * 2048) >> 4),
                          idesc_x, ks > 0 ? 1u : acc0);
#pragma unroll
            for (int ks = 0; ks < kTileRows / 16; ++ks)
              mma_bf16_ss(tmem + C::kColMass, pd + ((ks * 2048) >> 4), ones_desc, idesc_m,
                          ks > 0 ? 1u : acc0);
            mma_commit(&x_empty[st]);
            mma_commit(&p_empty[pb]);
            if (last) mma_commit(&acc_full[sg & 1u]);
            ++t2;
            progressed = true;
          }
        }
        if (walker_done && t2 == t1) break;
        if (progressed) {
          idle_since = cycles_now();
        } else if (!*abort_flag && cycles_now() - idle_since <= kWaitTimeoutCycles) {
          // Nothing ready: back off briefly so that this polling thread does
          // not take issue slots from the softmax warps on its SM sub-partition.
          __nanosleep(64);
        } else if (*abort_flag) {
          ok = false;
        } else if (cycles_now() - idle_since > kWaitTimeoutCycles) {
          *abort_flag = 1u;
          atomicOr(sticky, DEVFLAG_TIMEOUT);
          ok = false;
        }
      }
      if (!ok) {  // make sure no MMA is still running when TMEM is released
        mma_commit(drain);
        mbar_wait_bounded(drain, 0);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int grp = (warp - 4) >> 2;       // 0: even tiles, 1: odd tiles
    const int q = warp & 3;                // TMEM lane quarter of this warp
    const int row = q * 32 + lane;         // tile row = TMEM lane of S^T
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int k = a.k;
    SegmentWalker w{a.offsets, a.batch, R0, R1, b0};
    int64_t user, s, e, lo, hi;
    uint32_t t = 0, seg = 0;
    bool ok = true;
    while (ok && w.next(user, s, e, lo, hi)) {
      for (int64_t r = s; r < e; r += kTileRows, ++t) {
        if (static_cast<int>(t & 1u) != grp) continue;
        const bool last = (r + kTileRows >= e);
        const int nrows = static_cast<int>((e - r) < kTileRows ? (e - r) : kTileRows);
        const bool valid = row < nrows;
        const int st = t % S;
        if (!warp_wait(&s_full[grp], (t >> 1) & 1u, abort_flag, sticky)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[KM / 32][32];
#pragma unroll
        for (int cc = 0; cc < KM / 32; ++cc)
          tmem_ld32(lane_addr + C::kColS + grp * KM + cc * 32, sr[cc]);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < KM / 32; ++cc) tmem_pin32(sr[cc]);
        tc_fence_before();
        mbar_arrive(&s_empty[grp]);

        // stable softmax over the prototype axis (thread-local); eight
        // independent max / sum chains keep the FP pipes busy
        float mx8[8], sm8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
        for (int j = 0; j < KM; ++j)
          if (FULL || j < k) mx8[j & 7] = fmaxf(mx8[j & 7], __uint_as_float(sr[j >> 5][j & 31]));
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
#pragma unroll
        for (int i = 0; i < 8; ++i) sm8[i] = 0.f;
        float pv[KM];
#pragma unroll
        for (int j = 0; j < KM; ++j) {
          const float ev = (FULL || j < k) ? ex2_approx(__uint_as_float(sr[j >> 5][j & 31]) - mx) : 0.f;
          pv[j] = ev;
          sm8[j & 7] += ev;
        }
        const float sum = ((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) + ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7]));
        const float inv = 1.0f / sum;

        if (!warp_wait(&p_empty[grp], ((t >> 1) & 1u) ^ 1u, abort_flag, sticky)) { ok = false; break; }
        // Row `row` of the probability tile, MN-major with 128-byte swizzle:
        // 64-prototype blocks 16 KB apart, 8-row groups 1 KB apart, the
        // 16-byte chunk index XOR-ed with (row mod 8).
        const uint32_t prow = smem_u32(p_s + grp * C::kPBytes) + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
        for (int mb = 0; mb < KM / 64; ++mb) {
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            const int j0 = mb * 64 + c8 * 8;
            uint32_t wv[4];
#pragma unroll
            for (int h = 0; h < 4; ++h)
              wv[h] = valid ? pack_bf16x2(pv[j0 + 2 * h] * inv, pv[j0 + 2 * h + 1] * inv) : 0u;
            st_shared_v4(prow + mb * 16384 + ((c8 ^ (row & 7)) << 4), wv[0], wv[1], wv[2], wv[3]);
          }
        }
        if (!valid) {
          // Rows past the segment's end hold another user's data (or TMA
          // zero fill).  Their weights are zero, but 0 * NaN is NaN, so the
          // rows themselves are cleared before the aggregation reads them.
          const uint32_t xrow = smem_u32(x_s + st * C::kXBytes) + row * 128;
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
#pragma unroll
            for (int i = 0; i < 8; ++i) st_shared_v4(xrow + cb * 16384 + i * 16, 0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        mbar_arrive(&p_full[grp]);

        if (last) {
          // ---------------------------------------------- drain X~ and m
          if (!warp_wait(&acc_full[seg & 1u], (seg >> 1) & 1u, abort_flag, sticky)) { ok = false; break; }
          tc_fence_after();
          const int64_t slot = segment_slot(c, lo, hi, R0, R1);
          float* dx = slot < 0 ? a.out_x + user * k * D : a.part_x + slot * k * D;
          float* dm = slot < 0 ? a.out_m + user * k : a.part_m + slot * k;
          // M=128: prototype j sits in TMEM lane j.  M=64: prototypes
          // 16q..16q+15 sit in lanes 32q..32q+15.
          const int j = (KM == 128) ? row : q * 16 + lane;
          const bool has = (KM == 128 ? true : lane < 16) && j < k;
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(lane_addr + C::kColAcc + cc * 32, v);
            tmem_wait_ld();
            tmem_pin32(v);
            if (has) {
              float4* dst = reinterpret_cast<float4*>(dx + static_cast<int64_t>(j) * D + cc * 32);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
          }
          uint32_t mv;
          tmem_ld1(lane_addr + C::kColMass, mv);
          tmem_wait_ld();
          tmem_pin1(mv);
          if (has) dm[j] = __uint_as_float(mv);
          tc_fence_before();
          mbar_arrive(acc_empty);
        }
      }
      ++seg;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int KM>
cudaError_t launch_one(const CUtensorMap& tx, const CUtensorMap& tq, const PassArgs& a,
                       int grid, cudaStream_t stream) {
  auto kern = a.k == KM ? fused_sa_kernel<D, KM, true> : fused_sa_kernel<D, KM, false>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D, KM>::kSmem);
  if (err != cudaSuccess) return err;
  kern<<<grid, kThreads, Cfg<D, KM>::kSmem, stream>>>(tx, tq, a);
  return cudaGetLastError();
}

}  // namespace

bool fused_bf16_supported(int d, int k_pad) {
  return (d == 64 && (k_pad == 64 || k_pad == 128)) ||
         (d == 128 && (k_pad == 64 || k_pad == 128)) || (d == 256 && k_pad == 64);
}

size_t fused_bf16_smem_bytes(int d, int k_pad) {
  if (d == 64) return k_pad == 64 ? Cfg<64, 64>::kSmem : Cfg<64, 128>::kSmem;
  if (d == 128) return k_pad == 64 ? Cfg<128, 64>::kSmem : Cfg<128, 128>::kSmem;
  return Cfg<256, 64>::kSmem;
}

cudaError_t launch_fused_bf16(const CUtensorMap& tx, const CUtensorMap& tq, int k_pad,
                              const PassArgs& a, int grid, cudaStream_t stream) {
  if (a.d == 64 && k_pad == 64) return launch_one<64, 64>(tx, tq, a, grid, stream);
  if (a.d == 64 && k_pad == 128) return launch_one<64, 128>(tx, tq, a, grid, stream);
  if (a.d == 128 && k_pad == 64) return launch_one<128, 64>(tx, tq, a, grid, stream);
  if (a.d == 128 && k_pad == 128) return launch_one<128, 128>(tx, tq, a, grid, stream);
  if (a.d == 256 && k_pad == 64) return launch_one<256, 64>(tx, tq, a, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sa
