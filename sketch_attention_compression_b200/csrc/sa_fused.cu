// Fused SA pass for bf16 histories on sm_100a (tcgen05 + TMEM + TMA).
//
// One SA layer (section 2.1 "Sketch Attention" of the SequenceO1 reading
// notes, "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模"), computed the
// way section 2.4 describes FlashSA: affinity, stable softmax statistics and
// aggregation are tiled together so that the k x n score and assignment
// matrices never reach HBM, over batches of unequal lengths.
//
// Per 128-row tile X_t of one user (rows i, prototypes j):
//   MMA1  S^T_t = X_t Q'^T            M=128 rows, N=k_pad, K=d     (TMEM, fp32)
//   softmax over j for every row i (log2 e is folded into Q'):
//         a_ji = exp2(s_ji - max_j s_ji) / sum_j exp2(...)
//         rounded to bf16 and stored to shared memory as the A operand of
//   MMA2  [X~ | m] += A_t [X_t | 1]   M=k_pad, N=d+16, K=128       (TMEM, fp32)
// The X tile in shared memory serves as the K-major A operand of MMA1 and
// as the MN-major B operand of MMA2; X is read from HBM once.
//
// The masses m_j = sum_i a_ji come out of MMA2 itself: its B operand has 16
// columns more than X, read from a block of bf16 ones, so accumulator
// column d holds the masses, computed from the same rounded weights as X~.
// An MN-major operand with 128-byte swizzle is read in 64-column chunks at
// a fixed stride (the descriptor's leading byte offset), so every X stage
// is placed such that its last two boxes and the one shared block of ones
// lie at that stride (see Plan).  This costs MMA2 one eighth more tensor
// time and nothing else; summing the weights over rows with the CUDA cores
// instead (shuffles, or row-sums kept in TMEM) loads the same shared-memory
// and tensor-memory path that the probability stores and the MMA issue
// already saturate.
//
// Warp roles (384 threads):
//   warp 0      TMA producer (X ring of Plan::S tiles; Q' once)
//   warp 1      MMA1 issuer (one thread): as soon as an X stage has landed
//               and its group's S^T buffer has been read out
//   warp 2      TMEM allocation / release; with per-user queries, one
//               thread loads each segment's Q'_b once MMA1 has finished
//               with the previous user's
//   warp 3      MMA2 issuer (one thread): as soon as the probabilities are
//               stored (and, for a segment's first tile, X~ was drained)
//   warps 4-7   softmax group 0 (even tiles), one thread per row
//   warps 8-11  softmax group 1 (odd tiles)
// Issuing one tcgen05.mma takes a thread tens of cycles, about as long as
// an N = 128 MMA runs, so the two kinds of MMA get a thread each, and each
// thread waits on its own barriers only.  The two softmax groups overlap
// one tile's exponentials with the other tile's stores; they share the one
// probability buffer.  The group that finishes a segment's last tile drains
// X~ and m to the outputs (or to a partial slot for a user that crosses CTA
// ranges).
//
// More than 128 prototypes (CLU): a cluster of C = k_pad / 128 CTAs (up to
// 8, so k <= 1024; section 2.2 of the notes puts the final layers at about
// a thousand prototypes) shares each row range.  CTA h holds prototypes
// [128 h, 128 h + 128): its slice of Q', its S^T columns, its rows of the
// accumulator; every CTA reads every X tile of the range (HBM once, L2 for
// the others).  The softmax over all k prototypes of a row combines the
// slices: each CTA computes its slice's maximum m_h and sum
// z_h = sum_j exp2(s_j - m_h), i.e. the slice's total in log2 form
// L_h = m_h + log2 z_h, and sends L_h of every row to the other CTAs: each
// softmax warp's 32 values go to each other CTA as one 128-byte bulk copy
// that lands in the receiver's slots and counts as arrived bytes on its
// barrier.  Each CTA then takes M = max_h L_h and Z = sum_h exp2(L_h - M) over
// all C values (in rank order, so every CTA gets the same M and Z bit for
// bit) and scales its exponentials by exp2(m_h - M) / Z.  The values land
// in slots that take the place of the drain staging (cluster CTAs drain
// straight from registers: they hold few segments), double-buffered by
// tile: a CTA sends tile u + 2 of a softmax group only after it has
// received every CTA's tile u + 1, which each CTA sends only after it has
// read its tile u slots, so no slot or barrier phase is overwritten early
// and no acknowledgement has to travel back.  The same order covers the
// copies' sources: a CTA rewrites its own tile u slot (tile u + 2) only
// after every CTA's tile u + 1 arrived, and each sent that only after this
// CTA's tile u copy to it had landed.
//
// Per-user queries (the SA step of a refinement layer, section 2.2 "Stacked
// Refinement" of the notes): the one Q' buffer is reloaded per segment.
// MMA1 waits for Q'_b before a segment's first tile and commits q_empty
// after its last, which lets warp 2 fetch the next user's Q' (from L2: the
// per-call Q' array was just written).  The reload costs one TMA round trip
// per segment boundary, partly hidden behind the two S^T buffers.
#include "sa_internal.h"
#include "sa_plan.h"
#include "sa_ptx.cuh"

#ifdef SA_FAULT_INJECT
// Fault-injection build only (libsa_inject.so, for the tests): when
// sa_debug_inject_stall(t) has set a tile index >= 0, CTA 0's producer never
// issues the copy of its tile t, so MMA1 waits on a barrier that nothing
// completes until the (shortened) wait limit runs out, and the pass must
// report DEVFLAG_TIMEOUT and leave the context usable.
__device__ int g_inject_stall_tile = -1;
extern "C" int sa_debug_inject_stall(int tile) {
  return static_cast<int>(cudaMemcpyToSymbol(g_inject_stall_tile, &tile, sizeof(int)));
}
#endif

namespace sa {
namespace {

constexpr int kThreads = 384;
constexpr int kBlock = kPlanBlock;

// Warp-wide wait: every lane polls, and the warp leaves converged with one
// common verdict (tcgen05.ld that follows is .sync.aligned).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity,
                                          volatile uint32_t* abort_flag, uint32_t* sticky) {
  const bool ok = mbar_wait(bar, parity, abort_flag, sticky);
  return __all_sync(0xFFFFFFFFu, ok);
}

// One arrival per warp, after every lane's prior work (callers fence first).
__device__ __forceinline__ void warp_arrive(uint64_t* bar, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// MMA1 of tile t is issued only after MMA2 of tile t - kMma1Lead has been
// issued.  The tensor pipe runs MMAs in issue order; MMA2 frees the X stage
// and the probability buffer, so it must not queue behind affinities that no
// softmax group needs yet.  The lead still leaves MMA1 of tile t about one
// tile period ahead of the group that consumes it (that group is busy with
// tile t - 2 until MMA2 of t - 2 can be issued).
#ifndef SA_MMA1_LEAD
#define SA_MMA1_LEAD 4
#endif
constexpr uint32_t kMma1Lead = SA_MMA1_LEAD;

#ifndef SA_EARLY_TRIGGER
#define SA_EARLY_TRIGGER 1
#endif


// Bounded wait until the counter `cnt` (a shared-memory word that only
// grows) reaches `target`; same abort and timeout contract as mbar_wait.
__device__ __forceinline__ bool wait_count(volatile uint32_t* cnt, uint32_t target,
                                           volatile uint32_t* abort_flag, uint32_t* sticky_flag) {
  if (*cnt >= target) return true;
  const long long t0 = cycles_now();
  while (*cnt < target) {
    if (*abort_flag) return false;
    if (cycles_now() - t0 > kWaitTimeoutCycles) {
      *abort_flag = 1u;
      atomicOr(sticky_flag, DEVFLAG_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Warp-wide wait with cluster-scope acquire (data published by other CTAs).
__device__ __forceinline__ bool warp_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  volatile uint32_t* abort_flag, uint32_t* sticky) {
  const bool ok = mbar_wait_cluster(bar, parity, abort_flag, sticky);
  return __all_sync(0xFFFFFFFFu, ok);
}

constexpr int kMaxCluster = 8;

// FULL: no prototype column needs masking (k == KM, or k == KM * C for a
// cluster).  CLU: prototype-split cluster of C CTAs (KM == 128 each); 0 none,
// 1 for C <= 4, 2 for C > 4 (how many exchange sources the softmax reads;
// a template choice, because reading all eight slots behind a runtime
// bound cost the small clusters in code generation).
template <int D, int KM, bool FULL, int CLU>
__global__ void __launch_bounds__(kThreads, 1)
    fused_sa_kernel(const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_q, const PassArgs a) {
  using Pl = Plan<D, KM>;
  constexpr int S = Pl::S;
  static_assert(CLU == 0 || KM == 128, "clusters split the prototypes in slices of 128");
  constexpr bool kClu = CLU != 0;

  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0u) {  // the 128-byte swizzle needs 1024-byte alignment
    grid_dependency_wait();
    // Every CTA of the launch has the same layout and takes this path, so
    // block 0 alone reports it (clearing the previous call's offset bits).
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      if (a.keep_flags) {
        atomicOr(&a.header->timeout_flags, DEVFLAG_SMEM_ALIGN);
      } else {
        a.header->flags = 0u;
        a.header->timeout_flags = DEVFLAG_SMEM_ALIGN;
      }
    }
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  uint8_t* q_s = smem;                               // Q', block 0
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Pl::kBars);
  uint64_t* x_full = bars;
  uint64_t* x_empty = bars + S;
  uint64_t* s_full = bars + 2 * S;  // [group]
  uint64_t* s_empty = s_full + 2;   // [group]
  // The probability buffer is handed over in four slices: slice q holds the
  // tile rows 32q..32q+31 that softmax warp q computes, which are K-steps
  // 2q and 2q+1 of MMA2.
  uint64_t* p_full = s_empty + 2;   // [group][slice]: the warp's probabilities are stored
  uint64_t* p_empty = p_full + 8;   // [tile parity][slice]: that tile's MMA2 has read the slice
  // Two acc_full barriers, used by segment parity, so that no wait can
  // confuse the phase of segment s with that of segment s - 2.
  uint64_t* acc_full = p_empty + 8;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* q_full = acc_empty + 1;
  uint64_t* drain = q_full + 1;     // [issuer]: abort path, all of its MMAs done
  // [lane quarter]: the drain of segment s has finished reading its staging
  // buffers (phase s), so the drain of segment s + 1 may refill them.
  uint64_t* stage_free = drain + 2;
  uint64_t* q_empty = stage_free + 4;  // per-user queries: MMA1 is done with this segment's Q'
  // Clusters: [group][tile parity] the other CTAs' row statistics of the
  // tile have arrived.
  uint64_t* stats_full = q_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stats_full + 4);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  int64_t* b0_slot = reinterpret_cast<int64_t*>(tmem_slot + 2);
  volatile uint32_t* mma2_issued = tmem_slot + 4;  // tiles whose MMA2 has been issued
  int64_t* range_slot = reinterpret_cast<int64_t*>(tmem_slot + 6);  // R0, R1

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Row ranges: one per CTA, or one per cluster (whose CTAs are
  // consecutive blocks; CTA h = rank h holds prototype slice h).
  const uint32_t ncl = kClu ? cluster_size() : 1u;
  const uint32_t h = kClu ? cluster_rank() : 0u;
  const int64_t G = gridDim.x / ncl;
  const int64_t c = blockIdx.x / ncl;
  const int64_t N = a.total_rows;
  const int k_loc = kClu ? min(KM, a.k - static_cast<int>(h) * KM) : a.k;  // this CTA's prototypes
  uint32_t* sticky = &a.header->timeout_flags;

  int64_t* off_cache = reinterpret_cast<int64_t*>(smem + Pl::kOffs);
  // Set-up in two parts.  The launch may overlap the end of the preceding
  // kernel in the stream (programmatic dependent launch), so the first part
  // touches shared and tensor memory only; grid_dependency_wait then makes
  // everything that kernel wrote visible before any global access.
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&x_full[i], 1); mbar_init(&x_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
      for (int sq = 0; sq < 4; ++sq) {
        mbar_init(&p_full[i * 4 + sq], 1);
        mbar_init(&p_empty[i * 4 + sq], 1);
      }
      mbar_init(&acc_full[i], 1);
      mbar_init(&drain[i], 1);
    }
    mbar_init(acc_empty, 4);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&stage_free[i], 1);
    if (kClu)
      for (int i = 0; i < 4; ++i) mbar_init(&stats_full[i], 1);
    *abort_flag = 0u;
    *mma2_issued = 0u;
    fence_mbar_init();
  }
  {  // the block of bf16 ones read as MMA2's extra 16 columns
    const uint32_t ones = sbase + Pl::kOnes * kBlock;
    for (int i = threadIdx.x; i < kBlock / 16; i += kThreads)
      st_shared_v4(ones + i * 16, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_proxy_async_smem();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  grid_dependency_wait();
#if SA_EARLY_TRIGGER
  // The next kernel in the stream (the finalize pass) may be scheduled as
  // SMs free up; its own grid_dependency_wait still waits for this pass to
  // complete, so only its launch overlaps this pass's tail.
  grid_dependency_launch();
#endif
  // The device flags of this call start clear.  This is block 0's first
  // global access: the preceding kernel's writes are visible, and any other
  // CTA can set a flag only after a bounded wait has run out (seconds).
  if (blockIdx.x == 0 && threadIdx.x == 0 && !a.keep_flags) {
    a.header->flags = 0u;
    a.header->timeout_flags = 0u;
  }
  if (warp == 0) {
    // This CTA's row range and its first user (the work split of
    // sa_internal.h, searched by the whole warp).
    int64_t b0v, b1v;
    const int64_t r0 = warp_range_begin(a.offsets, a.batch, N, c, G, lane, &b0v);
    const int64_t r1 = warp_range_begin(a.offsets, a.batch, N, c + 1, G, lane, &b1v);
    if (!(r0 < r1)) b0v = a.batch;
    if (lane == 0) {
      range_slot[0] = r0;
      range_slot[1] = r1;
      *b0_slot = b0v;
    }
    // Offsets from the CTA's first user on, in shared memory: every role
    // walks them at each segment change, and a global load there (a
    // round trip through a loaded memory system) would stall the role.
    for (int i = lane; i < Pl::kOffCache && b0v + i <= a.batch; i += 32)
      off_cache[i] = a.offsets[b0v + i];
  }
  tc_fence_before();
  // With a cluster, the other CTAs' barriers must be initialised before
  // this CTA signals them: the cluster barrier also covers the CTA's own.
  if (kClu) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t b0 = *b0_slot;
  const int64_t R0 = range_slot[0], R1 = range_slot[1];
  const int64_t n_cached =
      (a.batch + 1 - b0) < Pl::kOffCache ? (a.batch + 1 - b0) : Pl::kOffCache;

  const bool user_q = a.user_queries != 0;
  uint32_t tiles_issued = 0;  // producer thread: X tiles whose TMA copy was issued
  uint32_t q_loads = 0;       // Q' loader thread (per-user queries): Q'_b copies issued
  // Clusters, per softmax warp: the group's tiles (local index u) whose row
  // totals this warp sent, whose exchange phase it saw complete, and (warp
  // q = 0, which arms the group's barrier) whose phase it armed.  The abort
  // drain at exit reads them.
  uint32_t xch_sent = 0, xch_waited = 0, xch_armed = 0;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      if (!user_q) {
        mbar_arrive_expect_tx(q_full, KM * D * 2);
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_2d(q_s + cb * KM * 128, &tm_q, q_full, cb * 64, static_cast<int32_t>(h * KM));
      }
      TileCursor cur{SegmentWalker{a.offsets, a.batch, R0, R1, b0, off_cache, b0, n_cached}};
      int64_t r;
      uint32_t t = 0;
      while (cur.next(r)) {
        const int st = t % S;
#ifdef SA_FAULT_INJECT
        if (c == 0 && static_cast<int>(t) == g_inject_stall_tile) {
          ++t;
          continue;
        }
#endif
        if (!mbar_wait(&x_empty[st], ((t / S) & 1u) ^ 1u, abort_flag, sticky)) break;
        mbar_arrive_expect_tx(&x_full[st], kTileRows * D * 2);
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_2d_hint(smem + Pl::box(st, cb) * kBlock, &tm_x, &x_full[st], cb * 64,
                           static_cast<int32_t>(r), pol);
        ++t;
      }
      tiles_issued = t;
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ Q'_b loader
    // Segment g's Q' (phase g of q_full) is copied once MMA1 has finished
    // segment g - 1 (phase g - 1 of q_empty): rows user * k_pad + h * KM..
    // of the per-call array (k_pad = KM * C).
    if (lane == 0 && user_q) {
      SegmentWalker w{a.offsets, a.batch, R0, R1, b0, off_cache, b0, n_cached};
      int64_t user, s, e, lo, hi;
      uint32_t g = 0;
      while (w.next(user, s, e, lo, hi)) {
        if (g > 0 && !mbar_wait(q_empty, (g - 1) & 1u, abort_flag, sticky)) break;
        mbar_arrive_expect_tx(q_full, KM * D * 2);
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb)
          tma_load_2d(q_s + cb * KM * 128, &tm_q, q_full, cb * 64,
                      static_cast<int32_t>((user * ncl + h) * KM));
        ++g;
      }
      q_loads = g;
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // A commit covers the MMAs of its own thread only: MMA1's commits
    // release S^T buffers; MMA2's release X stages (MMA2 of a tile starts
    // after that tile's MMA1 has completed, because its probabilities were
    // computed from the MMA1 result), the probability buffer and the
    // accumulator.
    if (lane == 0) {
      const int role = warp == 1 ? 0 : 1;
      // Descriptors.  A byte offset b within shared memory is applied by
      // adding b >> 4 to the start-address field (bits 0-13); every address
      // stays below 2^18 bytes, so the field never carries.
      const uint64_t xk_desc = smem_desc(sbase, 16, 1024, 2);                // X as K-major A
      const uint64_t q_desc = smem_desc(sbase, 16, 1024, 2);                 // Q' as K-major B
      const uint64_t p_desc =
          smem_desc(sbase + Pl::kP0 * kBlock, Pl::kPStride * kBlock, 1024, 2);  // P, MN-major A
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTileRows, KM, 0, 0);
      constexpr uint32_t idesc_x0 = idesc_bf16_f32(KM, Pl::kPartN0, 1, 1);
      constexpr uint32_t idesc_x1 = idesc_bf16_f32(KM, 144, 1, 1);
      bool ok = true;
      SegmentWalker w{a.offsets, a.batch, R0, R1, b0, off_cache, b0, n_cached};
      int64_t user, s, e, lo, hi;
      uint32_t t = 0, seg = 0;
      while (ok && w.next(user, s, e, lo, hi)) {
        for (int64_t r = s; r < e; r += kTileRows, ++t) {
          const int st = t % S;
          if (role == 0) {
            // ---- MMA1: S^T_t = X_t Q'^T into the S^T buffer of tile t's group
            const int sb = t & 1;
            // Q' for this segment: loaded once (phase 0) for shared
            // queries, phase seg of the per-user reloads otherwise.
            if ((r == s && !mbar_wait(q_full, user_q ? (seg & 1u) : 0u, abort_flag, sticky)) ||
                (t >= kMma1Lead && !wait_count(mma2_issued, t + 1 - kMma1Lead, abort_flag, sticky)) ||
                !mbar_wait(&x_full[st], (t / S) & 1u, abort_flag, sticky) ||
                !mbar_wait(&s_empty[sb], ((t >> 1) & 1u) ^ 1u, abort_flag, sticky)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t dcol = tmem + Pl::kColS + sb * KM;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
              mma_bf16_ss(dcol, xk_desc + ((Pl::box(st, ks >> 2) * kBlock + (ks & 3) * 32) >> 4),
                          q_desc + (((ks >> 2) * (KM * 128) + (ks & 3) * 32) >> 4), idesc_s,
                          ks > 0 ? 1u : 0u);
            mma_commit(&s_full[sb]);
            if (user_q && r + kTileRows >= e) mma_commit(q_empty);
          } else {
            // ---- MMA2: [X~ | m] += A_t [X_t | 1]  (a segment's first tile overwrites)
            const bool first = (r == s);
            const bool last = (r + kTileRows >= e);
            if (first && !mbar_wait(acc_empty, (seg & 1u) ^ 1u, abort_flag, sticky)) {
              ok = false;
              break;
            }
            const uint32_t acc0 = first ? 0u : 1u;
            const uint64_t bd0 = smem_desc(sbase + Pl::b_start(st, 0) * kBlock,
                                           Pl::b_stride(st, 0) * kBlock, 1024, 2);
            const uint64_t bd1 = smem_desc(sbase + Pl::b_start(st, 1) * kBlock,
                                           Pl::b_stride(st, 1) * kBlock, 1024, 2);
            // Slice by slice: K-steps 2q and 2q+1 as soon as warp q's rows
            // are stored, then a commit that frees that slice for the next
            // tile.
#pragma unroll
            for (int sq = 0; sq < 4; ++sq) {
              if (!mbar_wait(&p_full[(t & 1u) * 4 + sq], (t >> 1) & 1u, abort_flag, sticky)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) {
                const int ks = 2 * sq + kk;
                mma_bf16_ss(tmem + Pl::kColAcc, p_desc + ((ks * 2048) >> 4),
                            bd0 + ((ks * 2048) >> 4), idesc_x0, ks > 0 ? 1u : acc0);
                if (Pl::kParts == 2)
                  mma_bf16_ss(tmem + Pl::kColAcc + 128, p_desc + ((ks * 2048) >> 4),
                              bd1 + ((ks * 2048) >> 4), idesc_x1, ks > 0 ? 1u : acc0);
              }
              mma_commit(&p_empty[(t & 1u) * 4 + sq]);
            }
            if (!ok) break;
            mma_commit(&x_empty[st]);
            if (last) mma_commit(&acc_full[seg & 1u]);
            *mma2_issued = t + 1;
          }
        }
        ++seg;
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int grp = (warp - 4) >> 2;       // 0: even tiles, 1: odd tiles
    const int q = warp & 3;                // TMEM lane quarter of this warp
    const int row = q * 32 + lane;         // tile row = TMEM lane of S^T
    const uint32_t xch_a = sbase + Pl::kXch;  // clusters: [group][parity] 4 KB of row totals
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int k = k_loc;
    SegmentWalker w{a.offsets, a.batch, R0, R1, b0, off_cache, b0, n_cached};
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
          tmem_ld32(lane_addr + Pl::kColS + grp * KM + cc * 32, sr[cc]);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < KM / 32; ++cc) tmem_pin32(sr[cc]);
        tc_fence_before();
        warp_arrive(&s_empty[grp], lane);

        // Padded prototypes (j >= k) get logit -inf, so they add nothing
        // to the maximum and exp2 gives them exactly 0.  Only 32-column
        // chunks that reach past k are touched (the test is uniform).
        if constexpr (!FULL) {
#pragma unroll
          for (int cc = 0; cc < KM / 32; ++cc) {
            if (cc * 32 + 32 > k) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (cc * 32 + i >= k) sr[cc][i] = __float_as_uint(-INFINITY);
            }
          }
        }
        // Stable softmax over the prototype axis (thread-local): four
        // independent max chains (three-input max) and four packed sums.
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < KM; j += 8) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int ja = j + 2 * u, jb = ja + 1;
            mx4[u] = max3f(mx4[u], __uint_as_float(sr[ja >> 5][ja & 31]),
                           __uint_as_float(sr[jb >> 5][jb & 31]));
          }
        }
        const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        const uint64_t neg_m = f2_pack(-mx, -mx);
        uint64_t z2[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < KM; j += 2) {
          float x0, x1;
          f2_unpack(f2_add(f2_pack(__uint_as_float(sr[j >> 5][j & 31]),
                                   __uint_as_float(sr[(j + 1) >> 5][(j + 1) & 31])),
                           neg_m),
                    x0, x1);
          const float e0 = ex2_approx(x0);
          const float e1 = ex2_approx(x1);
          sr[j >> 5][j & 31] = __float_as_uint(e0);
          sr[(j + 1) >> 5][(j + 1) & 31] = __float_as_uint(e1);
          z2[(j >> 1) & 3] = f2_add(z2[(j >> 1) & 3], f2_pack(e0, e1));
        }
        float za, zb, zc, zd;
        f2_unpack(f2_add(z2[0], z2[1]), za, zb);
        f2_unpack(f2_add(z2[2], z2[3]), zc, zd);
        const float zl = (za + zb) + (zc + zd);
        float inv;
        if constexpr (kClu) {
          // Send L_h of this row to every other CTA and wait for theirs.
          // Each [group][parity] region holds 8 sources x 128 rows,
          // source-major: a warp's 32 values are 128 contiguous bytes,
          // which lane p sends to CTA p with one bulk copy (a message per
          // row and CTA cost more than the rest of the exchange).  The
          // slot is rewritten two tiles of the group later, after every
          // CTA's next tile has arrived here, which each CTA sends only
          // once this tile's copies to it have landed.
          const uint32_t u = t >> 1, par = u & 1u;
          uint64_t* sfull = &stats_full[grp * 2 + par];
          if (q == 0 && lane == 0) mbar_arrive_expect_tx(sfull, (ncl - 1) * 128 * 4);
          if (q == 0) xch_armed = u + 1;
          const float Lh = mx + lg2_approx(zl);
          const uint32_t sfull_a = smem_u32(sfull);
          constexpr int kSrc = CLU == 2 ? kMaxCluster : 4;  // sources the reads cover
          const uint32_t region = xch_a + (grp * 2 + par) * 4096;
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(region + h * 512 + row * 4), "f"(Lh)
                       : "memory");
          fence_proxy_async_smem();
          __syncwarp();
          const uint32_t wslot = region + h * 512 + q * 128;
          if (static_cast<uint32_t>(lane) < ncl && static_cast<uint32_t>(lane) != h)
            bulk_copy_to_cta(map_to_cta(wslot, lane), wslot, 128, map_to_cta(sfull_a, lane));
          xch_sent = u + 1;
          if (!warp_wait_cluster(sfull, (u >> 1) & 1u, abort_flag, sticky)) {
            ok = false;
            break;
          }
          xch_waited = u + 1;
          float Lv[kSrc];
#pragma unroll
          for (int p = 0; p < kSrc; ++p)
            Lv[p] = p < static_cast<int>(ncl) ? ld_shared_f32(region + p * 512 + row * 4)
                                              : -INFINITY;
          float Mx = Lv[0];
#pragma unroll
          for (int p = 1; p < kSrc; ++p) Mx = fmaxf(Mx, Lv[p]);
          float Z = 0.f;
#pragma unroll
          for (int p = 0; p < kSrc; ++p)
            if (p < static_cast<int>(ncl)) Z += ex2_approx(Lv[p] - Mx);
          inv = valid ? ex2_approx(mx - Mx) / Z : 0.f;
        } else {
          inv = valid ? 1.0f / zl : 0.f;
        }
        const uint64_t inv2 = f2_pack(inv, inv);

        // This warp's slice of the probability buffer is free once the
        // previous tile's MMA2 (of the other group) has read it.
        if (t > 0 &&
            !warp_wait(&p_empty[((t - 1) & 1u) * 4 + q], ((t - 1) >> 1) & 1u, abort_flag, sticky)) {
          ok = false;
          break;
        }
        // Row `row` of the probability tile, MN-major with 128-byte swizzle:
        // 64-prototype chunks kPStride blocks apart, 8-row groups 1 KB apart,
        // the 16-byte unit index XOR-ed with (row mod 8).  Rows past the
        // segment's end may hold NaN (another user's data): their weights
        // are forced to zero, not scaled by zero.
        const uint32_t prow = sbase + Pl::kP0 * kBlock + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
        for (int c8 = 0; c8 < KM / 8; ++c8) {
          uint32_t pw[4];
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            const int j = c8 * 8 + 2 * hh;
            float p0, p1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(sr[j >> 5][j & 31]),
                                     __uint_as_float(sr[(j + 1) >> 5][(j + 1) & 31])),
                             inv2),
                      p0, p1);
            pw[hh] = valid ? pack_bf16x2(p0, p1) : 0u;
          }
          st_shared_v4(prow + (c8 >> 3) * (Pl::kPStride * kBlock) + (((c8 & 7) ^ (row & 7)) << 4),
                       pw[0], pw[1], pw[2], pw[3]);
        }
        if (!valid) {
          // The rows themselves are cleared too, because 0 * NaN is NaN in
          // the aggregation (the block of ones is never touched).
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            const uint32_t xrow = sbase + Pl::box(st, cb) * kBlock + row * 128;
#pragma unroll
            for (int i = 0; i < 8; ++i) st_shared_v4(xrow + i * 16, 0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
        warp_arrive(&p_full[grp * 4 + q], lane);

        if (last) {
          // ---------------------------------------------- drain X~ and m
          if (!warp_wait(&acc_full[seg & 1u], (seg >> 1) & 1u, abort_flag, sticky)) { ok = false; break; }
          tc_fence_after();
          const int64_t slotp = segment_slot(c, lo, hi, R0, R1);
          // This CTA's prototype rows start at h * KM of the user's k.
          const int64_t krow = static_cast<int64_t>(h) * KM;
          float* dm = (slotp < 0 ? a.out_m + user * a.k : a.part_m + slotp * a.k) + krow;
          float* dxo = (slotp < 0 ? a.out_x + user * a.k * D : a.part_x + slotp * a.k * D) + krow * D;
          // M=128: prototype j sits in TMEM lane j.  M=64: prototypes
          // 16q..16q+15 sit in lanes 32q..32q+15.
          const int j0 = KM == 128 ? q * 32 : q * 16;
          const int j = j0 + lane;
          const bool has = (KM == 128 ? true : lane < 16) && j < k;
          if (!kClu && seg > 0 && !warp_wait(&stage_free[q], (seg - 1) & 1u, abort_flag, sticky)) {
            ok = false;
            break;
          }
          // The accumulator is copied to registers in batches of up to 128
          // columns; the last batch's loads release it (acc_empty), so the
          // next segment's first MMA2 waits for TMEM reads only.  Each
          // 32-column chunk is then staged in shared memory (one row per
          // lane) and read back so that every warp store writes four whole
          // 128-byte rows of X~, instead of a 16-byte piece of 32 different
          // rows, which would hold up the other group's shared-memory
          // stores behind it.
          const uint32_t stage = sbase + Pl::kDrain + q * Pl::kDrainBuf;
          constexpr int kDrainCols = D < 128 ? D : 128;
          uint32_t mv = 0;
          uint32_t chunk = 0;
#pragma unroll 1
          for (int bt = 0; bt < D / kDrainCols; ++bt) {
            const bool final_batch = bt == D / kDrainCols - 1;
            uint32_t v[kDrainCols / 32][32];
#pragma unroll
            for (int cc = 0; cc < kDrainCols / 32; ++cc)
              tmem_ld32(lane_addr + Pl::kColAcc + bt * kDrainCols + cc * 32, v[cc]);
            if (final_batch) tmem_ld1(lane_addr + Pl::kColAcc + D, mv);
            tmem_wait_ld();
#pragma unroll
            for (int cc = 0; cc < kDrainCols / 32; ++cc) tmem_pin32(v[cc]);
            tmem_pin1(mv);
            if (final_batch) {
              tc_fence_before();
              warp_arrive(acc_empty, lane);
            }
            if constexpr (kClu) {
              // Straight from registers: lane j writes its row's columns.
              if (has) {
#pragma unroll
                for (int cc = 0; cc < kDrainCols / 32; ++cc) {
                  float4* dst = reinterpret_cast<float4*>(dxo + static_cast<int64_t>(j) * D +
                                                          bt * kDrainCols + cc * 32);
#pragma unroll
                  for (int w4 = 0; w4 < 8; ++w4)
                    dst[w4] = make_float4(__uint_as_float(v[cc][4 * w4]),
                                          __uint_as_float(v[cc][4 * w4 + 1]),
                                          __uint_as_float(v[cc][4 * w4 + 2]),
                                          __uint_as_float(v[cc][4 * w4 + 3]));
                }
              }
            } else {
              // 32-column chunks: each lane stages its row (128 bytes, the
              // 16-byte unit index XOR-ed with row mod 8), then the warp
              // writes four whole rows per store.
#pragma unroll
              for (int cc = 0; cc < kDrainCols / 32; ++cc, ++chunk) {
                if (chunk > 0) __syncwarp();  // the previous chunk's reads are done
                if (lane < Pl::kDrainRows) {
#pragma unroll
                  for (int u = 0; u < 8; ++u)
                    st_shared_v4(stage + lane * 128 + ((u ^ (lane & 7)) << 4), v[cc][4 * u],
                                 v[cc][4 * u + 1], v[cc][4 * u + 2], v[cc][4 * u + 3]);
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < Pl::kDrainRows / 4; ++i) {
                  const int rr = 4 * i + (lane >> 3), uu = lane & 7;
                  const float4 w = ld_shared_v4f(stage + rr * 128 + ((uu ^ (rr & 7)) << 4));
                  if (j0 + rr < k)
                    *reinterpret_cast<float4*>(dxo + static_cast<int64_t>(j0 + rr) * D +
                                               bt * kDrainCols + cc * 32 + uu * 4) = w;
                }
              }
            }
          }
          __syncwarp();
          if (!kClu && lane == 0) mbar_arrive(&stage_free[q]);
          if (has) dm[j] = __uint_as_float(mv);
        }
      }
      ++seg;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // A role gave up (a bounded wait ran out): every role has now stopped,
    // but copies and MMAs that the others issued may still be in flight.
    // They must finish before the tensor memory is released and the CTA's
    // shared memory is handed to the next CTA.
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
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if constexpr (kClu) {
    // Row totals travel between the CTAs as bulk copies, which the cluster
    // barrier does not order (and which read the sender's shared memory
    // until they land).  On the normal path every value a CTA was sent has
    // been waited for.  If any CTA of the cluster gave up, a copy may still
    // be in flight to a CTA that stopped waiting, so before the
    // final barrier each CTA waits until everything sent to it has landed:
    //   1. every CTA publishes its abort flag and, per softmax warp, its
    //      exchange counts (in the offset cache, unused from here on), then
    //      all pass one cluster barrier, on every path;
    //   2. if any CTA aborted, one thread per group re-arms the at most one
    //      phase that was sent to but not armed, settles with complete_tx
    //      the shares of every phase that a stopped warp never sent, and
    //      waits (bounded) until those phases complete, i.e. until the
    //      values in flight have landed.
    // A sender can only send tile u + 1 of a group after it received the
    // receiver's tile u, which the receiver sends after arming it, and a
    // warp arms tile u + 1 only after it saw tile u complete; so the
    // phases left open are the group's tiles waited and waited + 1, on the
    // two different barriers of its double buffer.
    uint32_t* pub = reinterpret_cast<uint32_t*>(off_cache);  // [0] abort, [1 + 12 g + 3 q + i]
    if (warp >= 4 && lane == 0) {
      const int g = (warp - 4) >> 2, q = warp & 3;
      pub[1 + 12 * g + 3 * q + 0] = xch_sent;
      pub[1 + 12 * g + 3 * q + 1] = xch_waited;
      pub[1 + 12 * g + 3 * q + 2] = xch_armed;
    }
    if (threadIdx.x == 0) pub[0] = *abort_flag;
    cluster_sync();
    if ((warp == 4 || warp == 8) && lane == 0) {
      const int g = (warp - 4) >> 2;
      const uint32_t pub_a = smem_u32(pub);
      uint32_t any = 0;
      for (uint32_t p = 0; p < ncl; ++p) any |= ld_shared_cluster_u32(map_to_cta(pub_a, p));
      if (any) {
        uint32_t waited = 0;
        for (int q = 0; q < 4; ++q) waited = max(waited, pub[1 + 12 * g + 3 * q + 1]);
        const uint32_t armed = pub[1 + 12 * g + 2];
        uint32_t sent[kMaxCluster][4];
        uint32_t top = armed;
        for (uint32_t p = 0; p < ncl; ++p)
          for (int q = 0; q < 4; ++q) {
            sent[p][q] = p == h ? 0u : ld_shared_cluster_u32(map_to_cta(pub_a + 4 * (1 + 12 * g + 3 * q), p));
            top = max(top, sent[p][q]);
          }
        for (uint32_t v = waited; v < top && v < waited + 2; ++v) {
          uint64_t* bar = &stats_full[g * 2 + (v & 1u)];
          if (v >= armed) mbar_arrive_expect_tx(bar, (ncl - 1) * 128 * 4);
          for (uint32_t p = 0; p < ncl; ++p)
            for (int q = 0; q < 4; ++q)
              if (p != h && sent[p][q] <= v) mbar_complete_tx(bar, 32 * 4);
        }
        for (uint32_t v = waited; v < top && v < waited + 2; ++v)
          mbar_wait_bounded(&stats_full[g * 2 + (v & 1u)], (v >> 1) & 1u);
      }
    }
    // No CTA of a cluster leaves while another may still read its published
    // counts or signal its barriers.
    cluster_sync();
  }
}

template <int D, int KM>
cudaError_t launch_one(const CUtensorMap& tx, const CUtensorMap& tq, const PassArgs& a,
                       int grid, cudaStream_t stream) {
  auto kern = a.k == KM ? fused_sa_kernel<D, KM, true, 0> : fused_sa_kernel<D, KM, false, 0>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Plan<D, KM>::kSmem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Plan<D, KM>::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tx, tq, a);
}

// Prototype-split clusters: `ranges` clusters of `ncl` CTAs (k_pad = 128 ncl).
template <int D>
cudaLaunchConfig_t cluster_config(int ranges, int ncl, cudaStream_t stream,
                                  cudaLaunchAttribute (&attr)[2]) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ranges * ncl));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Plan<D, 128>::kSmem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(ncl);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cfg;
}

template <int D>
cudaError_t launch_cluster(const CUtensorMap& tx, const CUtensorMap& tq, const PassArgs& a,
                           int ranges, int ncl, cudaStream_t stream) {
  const bool full = a.k == 128 * ncl;
  auto kern = ncl > 4 ? (full ? fused_sa_kernel<D, 128, true, 2> : fused_sa_kernel<D, 128, false, 2>)
                      : (full ? fused_sa_kernel<D, 128, true, 1> : fused_sa_kernel<D, 128, false, 1>);
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Plan<D, 128>::kSmem);
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = cluster_config<D>(ranges, ncl, stream, attr);
  return cudaLaunchKernelEx(&cfg, kern, tx, tq, a);
}

template <int D>
int cluster_capacity(int ncl) {
  auto kern = ncl > 4 ? fused_sa_kernel<D, 128, false, 2> : fused_sa_kernel<D, 128, false, 1>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Plan<D, 128>::kSmem) != cudaSuccess)
    return 0;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = cluster_config<D>(1, ncl, nullptr, attr);
  cfg.numAttrs = 1;  // the cluster shape alone
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) return 0;
  return n;
}

}  // namespace

int fused_bf16_cluster_max_clusters(int d, int ncl) {
  if (ncl < 2 || ncl > kMaxCluster) return 0;
  if (d == 64) return cluster_capacity<64>(ncl);
  if (d == 128) return cluster_capacity<128>(ncl);
  return 0;
}

cudaError_t launch_fused_bf16_cluster(const CUtensorMap& tx, const CUtensorMap& tq,
                                      const PassArgs& a, int ranges, int ncl,
                                      cudaStream_t stream) {
  if (ncl < 2 || ncl > kMaxCluster || a.k > 128 * ncl || a.k <= 128 * (ncl - 1))
    return cudaErrorInvalidValue;
  if (a.d == 64) return launch_cluster<64>(tx, tq, a, ranges, ncl, stream);
  if (a.d == 128) return launch_cluster<128>(tx, tq, a, ranges, ncl, stream);
  return cudaErrorInvalidValue;
}

bool fused_bf16_supported(int d, int k_pad) {
  return (d == 64 && (k_pad == 64 || k_pad == 128)) ||
         (d == 128 && (k_pad == 64 || k_pad == 128)) ||
         (d == 256 && (k_pad == 64 || k_pad == 256));  // 256: the two-CTA pass
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
