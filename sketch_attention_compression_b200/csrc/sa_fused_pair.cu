// Fused SA pass for d = 256 and up to 256 prototypes: a cluster of two CTAs
// shares every X tile, each CTA owning half of the prototypes.
//
// Same layer and same per-tile steps as sa_fused.cu (section 2.1 "Sketch
// Attention" and the FlashSA paragraph of section 2.4 of the SequenceO1
// reading notes, "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模").
// With 256 prototypes and d = 256 the fp32 accumulator alone is 256 x 256,
// all 512 columns of one SM's tensor memory, so the prototypes are split:
// CTA h of the pair holds prototypes [128 h, 128 h + 128) and their slice
// of Q', and both CTAs read every X tile of their row range (the second read
// of a tile is served by L2).  The softmax over all 256 prototypes of a row
// combines the two halves: each CTA computes its half's maximum m_h and
// sum z_h = sum_j exp2(s_j - m_h) and sends (m_h, z_h) to the other CTA's
// shared memory (st.async, completing on that CTA's mbarrier); then
//   a_j = exp2(s_j - m_h) * exp2(m_h - M) / (z_0 exp2(m_0 - M) + z_1 exp2(m_1 - M)),
//   M = max(m_0, m_1).
// Per tile and CTA:
//   MMA1  S^T_t = X_t Q'_h^T                 M=128 rows, N=128, K=256   (TMEM, fp32)
//   MMA2  [X~_h | m_h] += A_t [X_t | 1]     M=128, N=128 + 144, K=128 (TMEM, fp32)
// Shared memory (16 KB blocks): Q'_h 0-3; the probability tile at 4, in two
// halves of 64 rows (the rows 64-127 are stored after MMA2 has read rows
// 0-63); X stages at (5, 6, 11, 12) and (8, 9, 7, 10); ones at 13.  The
// last two boxes of a stage and the ones lie at stride L = 1 and 3, read by
// MMA2's N = 144 half, as in sa_fused.cu.
// TMEM: S^T (one buffer, 128 columns) and the accumulator (272 columns).
// Warps: 0 TMA, 1 MMA1 issuer, 2 TMEM, 3 MMA2 issuer, 4-7 softmax (one row
// per thread).
#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace sa {
namespace {

constexpr int kPairThreads = 256;
constexpr int kB = 16384;  // block
constexpr int kPairStages = 2;
constexpr int kPairBars = 14 * kB;
constexpr int kPairSmem = kPairBars + 3072;
static_assert(kPairSmem <= 232448, "shared memory budget");
constexpr uint32_t kColS = 0;       // S^T, 128 columns
constexpr uint32_t kColAcc = 128;   // [X~ | m], 272 columns; m in column 256
constexpr int kOnesBlk = 13;
constexpr int kPBlk = 4;

__host__ __device__ constexpr int pair_box(int s, int b) {
  return s == 0 ? (b == 0 ? 5 : b == 1 ? 6 : b == 2 ? 11 : 12)
                : (b == 0 ? 8 : b == 1 ? 9 : b == 2 ? 7 : 10);
}
__host__ __device__ constexpr int pair_l(int s) { return s == 0 ? 1 : 3; }

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity,
                                          volatile uint32_t* abort_flag, uint32_t* sticky) {
  const bool ok = mbar_wait(bar, parity, abort_flag, sticky);
  return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ void warp_arrive(uint64_t* bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

template <bool FULL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    fused_sa_pair_kernel(const __grid_constant__ CUtensorMap tm_x,
                         const __grid_constant__ CUtensorMap tm_qh, const PassArgs a) {
  constexpr int D = 256;
  constexpr int S = kPairStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const bool aligned = (sbase & 1023u) == 0u;
  const uint32_t h = cluster_rank();   // prototype half of this CTA
  const uint32_t peer = h ^ 1u;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPairBars);
  uint64_t* x_full = bars;               // [S]
  uint64_t* x_empty = bars + S;          // [S]
  uint64_t* s_full = bars + 2 * S;
  uint64_t* s_empty = s_full + 1;
  uint64_t* plo_full = s_empty + 1;      // rows 0-63 of the probability tile stored
  uint64_t* plo_empty = plo_full + 1;    // ... and read by MMA2
  uint64_t* phi_full = plo_empty + 1;    // rows 64-127 stored
  uint64_t* phi_empty = phi_full + 1;    // ... and read by MMA2
  uint64_t* acc_full = phi_empty + 1;    // [2], by segment parity
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* q_full = acc_empty + 1;
  uint64_t* drain = q_full + 1;          // [2 issuers]
  uint64_t* xch = drain + 2;             // [2 tile parities]: the other half's (m, z) arrived
  uint64_t* q_empty = xch + 2;           // per-user queries: MMA1 is done with this segment's Q'
  float2* xslot = reinterpret_cast<float2*>(q_empty + 2);  // [2 tile parities][128 rows]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xslot + 256);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  int64_t* b0_slot = reinterpret_cast<int64_t*>(tmem_slot + 2);
  int64_t* range_slot = reinterpret_cast<int64_t*>(tmem_slot + 4);  // R0, R1
  // Published at exit for the abort drain: [0] abort flag, then per softmax
  // warp q the tiles it sent, saw complete and (q = 0) armed: [1 + 3q + i].
  uint32_t* pub = reinterpret_cast<uint32_t*>(range_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t G = gridDim.x / 2;             // row ranges (one per cluster)
  const int64_t c = blockIdx.x / 2;
  const int64_t N = a.total_rows;
  uint32_t* sticky = &a.header->timeout_flags;

  // The device flags of this call start clear (block 0's first global
  // access; another CTA can set a flag only after a bounded wait has run
  // out).  Every CTA has the same shared-memory layout, so on misalignment
  // all of them stop here and block 0 alone reports it.
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (!a.keep_flags) {
      a.header->flags = 0u;
      a.header->timeout_flags = aligned ? 0u : DEVFLAG_SMEM_ALIGN;
    } else if (!aligned) {
      atomicOr(&a.header->timeout_flags, DEVFLAG_SMEM_ALIGN);
    }
  }
  if (aligned && threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&x_full[i], 1); mbar_init(&x_empty[i], 1); }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 4);
    mbar_init(plo_full, 2);
    mbar_init(plo_empty, 1);
    mbar_init(phi_full, 2);
    mbar_init(phi_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&drain[i], 1);
      mbar_init(&xch[i], 1);
    }
    mbar_init(acc_empty, 4);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    *abort_flag = 0u;
    int64_t b0u;
    const int64_t r0 = range_begin(a.offsets, a.batch, N, c, G, &b0u);
    const int64_t r1 = range_begin(a.offsets, a.batch, N, c + 1, G);
    range_slot[0] = r0;
    range_slot[1] = r1;
    *b0_slot = r0 < r1 ? b0u : a.batch;
    fence_mbar_init();
  }
  if (aligned) {  // the block of bf16 ones read as MMA2's extra 16 columns
    const uint32_t ones = sbase + kOnesBlk * kB;
    for (int i = threadIdx.x; i < kB / 16; i += kPairThreads)
      st_shared_v4(ones + i * 16, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_proxy_async_smem();
  }
  if (aligned && warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  // The other CTA's barriers must be initialised before any st.async
  // reaches them.
  cluster_sync();
  tc_fence_after();

  uint32_t tiles_issued = 0;  // producer thread: X tiles whose TMA copy was issued
  uint32_t q_loads = 0;       // Q' loader thread (per-user queries): Q'_b copies issued
  // Per softmax thread: tiles whose (m, z) it sent, whose exchange phase it
  // saw complete, and (row 0, which arms the barrier) whose phase it armed.
  uint32_t xch_sent = 0, xch_waited = 0, xch_armed = 0;
  const bool user_q = a.user_queries != 0;
  if (aligned) {
    const uint32_t tmem = *tmem_slot;
    const int64_t b0 = *b0_slot;
    const int64_t R0 = range_slot[0], R1 = range_slot[1];
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        // Both CTAs of the pair read every tile; the default L2 policy keeps
        // a tile for the second reader.
        if (!user_q) {
          mbar_arrive_expect_tx(q_full, 128 * D * 2);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_2d(smem + cb * kB, &tm_qh, q_full, cb * 64, static_cast<int32_t>(128 * h));
        }
        TileCursor cur{SegmentWalker{a.offsets, a.batch, R0, R1, b0}};
        int64_t r;
        uint32_t t = 0;
        while (cur.next(r)) {
          const int st = t % S;
          if (!mbar_wait(&x_empty[st], ((t / S) & 1u) ^ 1u, abort_flag, sticky)) break;
          mbar_arrive_expect_tx(&x_full[st], kTileRows * D * 2);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_2d(smem + pair_box(st, cb) * kB, &tm_x, &x_full[st], cb * 64,
                        static_cast<int32_t>(r));
          ++t;
        }
        tiles_issued = t;
      }
    } else if (warp == 2) {
      // ---------------------------------------------------------- Q'_b loader
      // Per-user queries: segment g's half of Q'_b (rows (2 user + h) 128..
      // of the per-call array, 256 padded prototypes per user) once MMA1 has
      // finished segment g - 1 with the previous one.
      if (lane == 0 && user_q) {
        SegmentWalker w{a.offsets, a.batch, R0, R1, b0};
        int64_t user, s, e, lo, hi;
        uint32_t g = 0;
        while (w.next(user, s, e, lo, hi)) {
          if (g > 0 && !mbar_wait(q_empty, (g - 1) & 1u, abort_flag, sticky)) break;
          mbar_arrive_expect_tx(q_full, 128 * D * 2);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_2d(smem + cb * kB, &tm_qh, q_full, cb * 64,
                        static_cast<int32_t>((2 * user + h) * 128));
          ++g;
        }
        q_loads = g;
      }
    } else if (warp == 1 || warp == 3) {
      // ---------------------------------------------------------- MMA issuers
      if (lane == 0) {
        const int role = warp == 1 ? 0 : 1;
        const uint64_t base_k = smem_desc(sbase, 16, 1024, 2);            // K-major operands
        const uint64_t p_desc = smem_desc(sbase + kPBlk * kB, 8192, 1024, 2);  // P, MN-major A
        constexpr uint32_t idesc_s = idesc_bf16_f32(kTileRows, 128, 0, 0);
        constexpr uint32_t idesc_x0 = idesc_bf16_f32(128, 128, 1, 1);
        constexpr uint32_t idesc_x1 = idesc_bf16_f32(128, 144, 1, 1);
        bool ok = true;
        SegmentWalker w{a.offsets, a.batch, R0, R1, b0};
        int64_t user, s, e, lo, hi;
        uint32_t t = 0, seg = 0;
        while (ok && w.next(user, s, e, lo, hi)) {
          for (int64_t r = s; r < e; r += kTileRows, ++t) {
            const int st = t % S;
            if (role == 0) {
              // Q' of this segment: loaded once (phase 0) for shared
              // queries, phase seg of the per-user reloads otherwise.
              if ((r == s && !mbar_wait(q_full, user_q ? (seg & 1u) : 0u, abort_flag, sticky)) ||
                  !mbar_wait(&x_full[st], (t / S) & 1u, abort_flag, sticky) ||
                  !mbar_wait(s_empty, (t & 1u) ^ 1u, abort_flag, sticky)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks)
                mma_bf16_ss(tmem + kColS,
                            base_k + ((pair_box(st, ks >> 2) * kB + (ks & 3) * 32) >> 4),
                            base_k + (((ks >> 2) * kB + (ks & 3) * 32) >> 4), idesc_s,
                            ks > 0 ? 1u : 0u);
              mma_commit(s_full);
              if (user_q && r + kTileRows >= e) mma_commit(q_empty);
            } else {
              const bool first = (r == s);
              const bool last = (r + kTileRows >= e);
              const uint64_t bd0 = smem_desc(sbase + pair_box(st, 0) * kB, kB, 1024, 2);
              const uint64_t bd1 =
                  smem_desc(sbase + pair_box(st, 2) * kB, pair_l(st) * kB, 1024, 2);
              const uint32_t acc0 = first ? 0u : 1u;
              // rows 0-63
              if (!mbar_wait(plo_full, t & 1u, abort_flag, sticky) ||
                  (first && !mbar_wait(acc_empty, (seg & 1u) ^ 1u, abort_flag, sticky))) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                mma_bf16_ss(tmem + kColAcc, p_desc + ((ks * 2048) >> 4), bd0 + ((ks * 2048) >> 4),
                            idesc_x0, ks > 0 ? 1u : acc0);
                mma_bf16_ss(tmem + kColAcc + 128, p_desc + ((ks * 2048) >> 4),
                            bd1 + ((ks * 2048) >> 4), idesc_x1, ks > 0 ? 1u : acc0);
              }
              mma_commit(plo_empty);
              // rows 64-127 (stored in the same places once rows 0-63 were read)
              if (!mbar_wait(phi_full, t & 1u, abort_flag, sticky)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int ks = 4; ks < 8; ++ks) {
                mma_bf16_ss(tmem + kColAcc, p_desc + (((ks - 4) * 2048) >> 4),
                            bd0 + ((ks * 2048) >> 4), idesc_x0, 1u);
                mma_bf16_ss(tmem + kColAcc + 128, p_desc + (((ks - 4) * 2048) >> 4),
                            bd1 + ((ks * 2048) >> 4), idesc_x1, 1u);
              }
              mma_commit(phi_empty);
              mma_commit(&x_empty[st]);
              if (last) mma_commit(&acc_full[seg & 1u]);
            }
          }
          ++seg;
        }
      }
    } else if (warp >= 4) {
      // ---------------------------------------------------------- softmax
      const int q = warp & 3;
      const int row = q * 32 + lane;
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      const int k = a.k;
      const int jbase = 128 * static_cast<int>(h);  // first prototype of this half
      const uint32_t xslot_a = smem_u32(xslot);
      const uint32_t xch_a = smem_u32(xch);
      SegmentWalker w{a.offsets, a.batch, R0, R1, b0};
      int64_t user, s, e, lo, hi;
      uint32_t t = 0, seg = 0;
      bool ok = true;
      while (ok && w.next(user, s, e, lo, hi)) {
        for (int64_t r = s; r < e; r += kTileRows, ++t) {
          const bool last = (r + kTileRows >= e);
          const int nrows = static_cast<int>((e - r) < kTileRows ? (e - r) : kTileRows);
          const bool valid = row < nrows;
          const int st = t % S;
          const uint32_t par = t & 1u;
          if (!warp_wait(s_full, t & 1u, abort_flag, sticky)) { ok = false; break; }
          tc_fence_after();
          uint32_t sr[4][32];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) tmem_ld32(lane_addr + kColS + cc * 32, sr[cc]);
          tmem_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) tmem_pin32(sr[cc]);
          tc_fence_before();
          warp_arrive(s_empty, lane);

          // this half's maximum and sum
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int j = 0; j < 128; j += 8) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int ja = j + 2 * u, jb = ja + 1;
              const float va = (FULL || jbase + ja < k) ? __uint_as_float(sr[ja >> 5][ja & 31]) : -INFINITY;
              const float vb = (FULL || jbase + jb < k) ? __uint_as_float(sr[jb >> 5][jb & 31]) : -INFINITY;
              mx4[u] = max3f(mx4[u], va, vb);
            }
          }
          const float m_h = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
          const uint64_t neg_m = f2_pack(-m_h, -m_h);
          uint64_t z2[4] = {0, 0, 0, 0};
#pragma unroll
          for (int j = 0; j < 128; j += 2) {
            float x0, x1;
            f2_unpack(f2_add(f2_pack(__uint_as_float(sr[j >> 5][j & 31]),
                                     __uint_as_float(sr[(j + 1) >> 5][(j + 1) & 31])),
                             neg_m),
                      x0, x1);
            const float e0 = (FULL || jbase + j < k) ? ex2_approx(x0) : 0.f;
            const float e1 = (FULL || jbase + j + 1 < k) ? ex2_approx(x1) : 0.f;
            sr[j >> 5][j & 31] = __float_as_uint(e0);
            sr[(j + 1) >> 5][(j + 1) & 31] = __float_as_uint(e1);
            z2[(j >> 1) & 3] = f2_add(z2[(j >> 1) & 3], f2_pack(e0, e1));
          }
          float za, zb, zc, zd;
          f2_unpack(f2_add(z2[0], z2[1]), za, zb);
          f2_unpack(f2_add(z2[2], z2[3]), zc, zd);
          const float z_h = (za + zb) + (zc + zd);

          // Exchange (m, z) with the other CTA.  Slots and barriers are
          // double-buffered by tile parity: the other CTA sends tile t + 2's
          // values only after it received this CTA's tile t + 1 values,
          // which are sent after this CTA read tile t's slot, so neither a
          // slot nor a barrier phase is reused early.
          if (row == 0) mbar_arrive_expect_tx(&xch[par], 128 * 8);
          xch_armed = t + 1;
          st_async_v2f(map_to_cta(xslot_a + (par * 128 + row) * 8, peer), m_h, z_h,
                       map_to_cta(xch_a + par * 8, peer));
          xch_sent = t + 1;
          if (!mbar_wait_cluster(&xch[par], (t >> 1) & 1u, abort_flag, sticky)) { ok = false; break; }
          xch_waited = t + 1;
          const float2 other = xslot[par * 128 + row];
          const float m_row = fmaxf(m_h, other.x);
          const float f_h = ex2_approx(m_h - m_row);  // 0 when this half is fully masked
          const float f_o = ex2_approx(other.x - m_row);
          const float scale = valid ? f_h / (z_h * f_h + other.y * f_o) : 0.f;
          const uint64_t scale2 = f2_pack(scale, scale);

          // Rows 0-63 wait until the previous tile's MMA2 has read rows
          // 64-127 (the buffer is free); rows 64-127 wait until this tile's
          // MMA2 has read rows 0-63.
          const bool lower = row < 64;
          if (lower ? (t > 0 && !warp_wait(phi_empty, (t - 1) & 1u, abort_flag, sticky))
                    : !warp_wait(plo_empty, t & 1u, abort_flag, sticky)) {
            ok = false;
            break;
          }
          // Row (row mod 64) of a 64-row half tile, MN-major, 128-byte
          // swizzle: the two 64-prototype chunks 8 KB apart.
          const int rr = row & 63;
          const uint32_t prow = sbase + kPBlk * kB + (rr >> 3) * 1024 + (rr & 7) * 128;
#pragma unroll
          for (int c8 = 0; c8 < 16; ++c8) {
            uint32_t pw[4];
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
              const int j = c8 * 8 + 2 * hh;
              float p0, p1;
              f2_unpack(f2_mul(f2_pack(__uint_as_float(sr[j >> 5][j & 31]),
                                       __uint_as_float(sr[(j + 1) >> 5][(j + 1) & 31])),
                               scale2),
                        p0, p1);
              pw[hh] = valid ? pack_bf16x2(p0, p1) : 0u;
            }
            st_shared_v4(prow + (c8 >> 3) * 8192 + (((c8 & 7) ^ (rr & 7)) << 4), pw[0], pw[1],
                         pw[2], pw[3]);
          }
          if (!valid) {  // 0 * NaN is NaN: clear rows past the segment's end
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb) {
              const uint32_t xrow = sbase + pair_box(st, cb) * kB + row * 128;
#pragma unroll
              for (int i = 0; i < 8; ++i) st_shared_v4(xrow + i * 16, 0u, 0u, 0u, 0u);
            }
          }
          fence_proxy_async_smem();
          warp_arrive(lower ? plo_full : phi_full, lane);

          if (last) {
            if (!warp_wait(&acc_full[seg & 1u], (seg >> 1) & 1u, abort_flag, sticky)) { ok = false; break; }
            tc_fence_after();
            const int64_t slotp = segment_slot(c, lo, hi, R0, R1);
            float* dx = slotp < 0 ? a.out_x + user * k * D : a.part_x + slotp * k * D;
            float* dm = slotp < 0 ? a.out_m + user * k : a.part_m + slotp * k;
            const int j = jbase + row;  // prototype j sits in TMEM lane row
            const bool has = j < k;
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t v[32];
              tmem_ld32(lane_addr + kColAcc + cc * 32, v);
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
            tmem_ld1(lane_addr + kColAcc + D, mv);
            tmem_wait_ld();
            tmem_pin1(mv);
            if (has) dm[j] = __uint_as_float(mv);
            tc_fence_before();
            warp_arrive(acc_empty, lane);
          }
        }
        ++seg;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (aligned && *abort_flag) {
    // A role gave up (a bounded wait ran out): let the copies and MMAs that
    // other roles issued finish before the tensor memory is released.
    if (warp == 0 && lane == 0) {
      const uint32_t t = tiles_issued;
      for (uint32_t u = (t > static_cast<uint32_t>(S) ? t - S : 0u); u < t; ++u)
        mbar_wait_bounded(&x_full[u % S], (u / S) & 1u);
      if (!user_q) mbar_wait_bounded(q_full, 0);
    }
    if (warp == 2 && lane == 0 && q_loads > 0) mbar_wait_bounded(q_full, (q_loads - 1) & 1u);
    if ((warp == 1 || warp == 3) && lane == 0) {
      const int role = warp == 1 ? 0 : 1;
      mma_commit(&drain[role]);
      mbar_wait_bounded(&drain[role], 0);
    }
    tc_fence_before();
    __syncthreads();
  }
  if (aligned && warp == 2) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, 512);
  }
  // The (m, z) values travel with st.async, which the cluster barrier does
  // not order.  On the normal path every value a CTA was sent has been
  // waited for.  If either CTA gave up, a value may still be in flight to a
  // CTA that stopped waiting, so before the final barrier each CTA waits
  // until everything sent to it has landed: both publish their abort flag
  // and exchange counts and pass a cluster barrier (on every path); then, if
  // either aborted, thread 0 of the softmax warps arms the at most one phase
  // the peer sent to but this CTA did not arm, settles with complete_tx the
  // shares the peer's stopped warps never sent, and waits (bounded) for
  // those phases.  The peer sends tile t + 1 only after receiving this CTA's
  // tile t, which row 0 sends after arming it, and row 0 arms tile t + 1
  // only after tile t completed; so only tiles `waited` and `waited` + 1
  // can be open, one on each barrier of the double buffer.  (The row-0
  // thread's counts stand for its warp; another lane's later success only
  // means a phase is complete, which the drain then finds at once.)
  if (aligned) {
    if (warp >= 4 && lane == 0) {
      const int q = warp & 3;
      pub[1 + 3 * q] = xch_sent;
      pub[2 + 3 * q] = xch_waited;
      pub[3 + 3 * q] = xch_armed;
    }
    if (threadIdx.x == 0) pub[0] = *abort_flag;
  }
  cluster_sync();
  if (aligned && warp == 4 && lane == 0) {
    const uint32_t peer_pub = map_to_cta(smem_u32(pub), peer);
    if (pub[0] | ld_shared_cluster_u32(peer_pub)) {
      uint32_t waited = 0;
      for (int q = 0; q < 4; ++q) waited = max(waited, pub[2 + 3 * q]);
      const uint32_t armed = pub[3];
      uint32_t sent[4];
      uint32_t top = armed;
      for (int q = 0; q < 4; ++q) {
        sent[q] = ld_shared_cluster_u32(peer_pub + 4 * (1 + 3 * q));
        top = max(top, sent[q]);
      }
      for (uint32_t v = waited; v < top && v < waited + 2; ++v) {
        if (v >= armed) mbar_arrive_expect_tx(&xch[v & 1u], 128 * 8);
        for (int q = 0; q < 4; ++q)
          if (sent[q] <= v) mbar_complete_tx(&xch[v & 1u], 32 * 8);
      }
      for (uint32_t v = waited; v < top && v < waited + 2; ++v)
        mbar_wait_bounded(&xch[v & 1u], (v >> 1) & 1u);
    }
  }
  // No CTA leaves while the other may still read its published counts or
  // store into its shared memory.
  cluster_sync();
}

}  // namespace

int fused_bf16_pair_max_clusters() {
  if (cudaFuncSetAttribute(fused_sa_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kPairSmem) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = kPairSmem;
  int n = 0;  // the kernel's own cluster size (2) applies
  if (cudaOccupancyMaxActiveClusters(&n, fused_sa_pair_kernel<true>, &cfg) != cudaSuccess) return 0;
  return n;
}

cudaError_t launch_fused_bf16_pair(const CUtensorMap& tx, const CUtensorMap& tq_half,
                                   const PassArgs& a, int ranges, cudaStream_t stream) {
  if (a.d != 256) return cudaErrorInvalidValue;
  auto kern = a.k == 256 ? fused_sa_pair_kernel<true> : fused_sa_pair_kernel<false>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmem);
  if (err != cudaSuccess) return err;
  kern<<<2 * ranges, kPairThreads, kPairSmem, stream>>>(tx, tq_half, a);
  return cudaGetLastError();
}

}  // namespace sa
