// Sketch cache and width adapter (sections 2.3 and 2.4 of the SequenceO1
// reading notes, "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模").
//
// Cache.  Section 2.4 keeps only the narrow user-side sketch, keyed by the
// user, the model version, the history timestamp and the sketch
// configuration, for a time-to-live, with capacity eviction; a miss runs the
// compression once and serves every target of the group.  The sketches live
// in a device pool of `capacity` slots (k x d fp32 plus k masses each); the
// index (key -> slot, insertion and last-use times) is host code, because the
// keys arrive with the host's request and every decision is a few map
// operations.  Decisions: an entry is fresh while now - t_insert < ttl; a hit
// refreshes its last use; eviction takes the smallest free slot, else the
// expired entry inserted earliest, else the least recently used (ties: the
// smaller slot); inserting a present key replaces it, and within a batch the
// later of two equal keys wins.  Data moves only on the device: a gather of
// hit slots into the caller's outputs, a scatter of new sketches into slots.
// sa_cache_forward runs the whole section 2.4 flow for a batch: look up,
// gather the hits, run the SA layer in place on each run of consecutive
// missed users (their rows and outputs are contiguous) and insert those
// sketches.
//
// Width adapter.  Section 2.3 widens the sketch for the ranking model with a
// linear W_A in R^{d x D} (D = 1024 in the final configuration); the adapted
// sketch keeps its k rows and is not cached (section 2.4).  Y = X~ W_A runs on
// the tensor cores: per CTA a tile of 128 sketch rows x 256 output columns,
// X~ rounded to bf16 by the threads into a K-major, 128-byte-swizzled A
// operand, W_A^T (bf16, made once) by TMA as the K-major B operand, the
// product in TMEM (256 fp32 columns), written back as bf16.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <map>
#include <mutex>
#include <new>
#include <set>
#include <utility>
#include <vector>

#include "sa.h"
#include "sa_internal.h"
#include "sa_ptx.cuh"

namespace {

struct KeyLess {
  bool operator()(const sa_cache_key& a, const sa_cache_key& b) const {
    if (a.user != b.user) return a.user < b.user;
    if (a.model_version != b.model_version) return a.model_version < b.model_version;
    if (a.history_ts != b.history_ts) return a.history_ts < b.history_ts;
    return a.config < b.config;
  }
};

}  // namespace

// Pinned host staging for the slot and offset lists a call copies to the
// device.  Calls alternate between two halves; a call waits (on its half's
// event) only for the copies of the call two before it, so the host runs
// ahead of the device instead of waiting for each copy as a copy from
// pageable memory would.
struct SaStaging {
  int64_t* host = nullptr;
  size_t cap = 0;
  size_t used = 0;
  cudaEvent_t ev = nullptr;
  bool recorded = false;
};

struct sa_cache_s {
  int device;
  int k;
  int d;
  int64_t capacity;
  double ttl;
  float* pool_x;   // [capacity][k][d]
  float* pool_m;   // [capacity][k]
  int64_t* d_slots = nullptr;  // per-call slot list on the device
  int64_t d_slots_cap = 0;
  SaStaging stg[2];
  uint64_t calls = 0;
  std::map<sa_cache_key, int64_t, KeyLess> index;
  std::vector<sa_cache_key> slot_key;
  std::vector<bool> used;
  std::vector<double> t_insert, t_use;
  std::set<int64_t> free_slots;
  std::set<std::pair<double, int64_t>> by_insert, by_use;
  int64_t hits = 0, misses = 0, evictions = 0;
  std::mutex mu;
};

struct sa_adapter_s {
  int device;
  int d;
  int D;
  uint16_t* wt;  // W_A^T: D x d bf16
  CUtensorMap tm_w;
};

namespace sa {
namespace {

// ------------------------------------------------------------------ index

bool fresh(const sa_cache_s* c, int64_t s, double now) { return now - c->t_insert[s] < c->ttl; }

void drop(sa_cache_s* c, int64_t s) {
  c->index.erase(c->slot_key[s]);
  c->by_insert.erase({c->t_insert[s], s});
  c->by_use.erase({c->t_use[s], s});
  c->used[s] = false;
  c->free_slots.insert(s);
}

void touch(sa_cache_s* c, int64_t s, double now) {
  c->by_use.erase({c->t_use[s], s});
  c->t_use[s] = now;
  c->by_use.insert({now, s});
}

int64_t lookup_one(sa_cache_s* c, const sa_cache_key& key, double now) {
  auto it = c->index.find(key);
  int64_t s = it == c->index.end() ? -1 : it->second;
  if (s >= 0 && !fresh(c, s, now)) {
    drop(c, s);
    s = -1;
  }
  if (s >= 0) {
    touch(c, s, now);
    ++c->hits;
  } else {
    ++c->misses;
  }
  return s;
}

int64_t victim(sa_cache_s* c, double now) {
  if (!c->free_slots.empty()) {
    const int64_t s = *c->free_slots.begin();
    c->free_slots.erase(c->free_slots.begin());
    return s;
  }
  int64_t s = c->by_insert.begin()->second;  // earliest inserted
  if (fresh(c, s, now)) s = c->by_use.begin()->second;  // none expired: least recently used
  drop(c, s);
  c->free_slots.erase(s);
  ++c->evictions;
  return s;
}

int64_t insert_one(sa_cache_s* c, const sa_cache_key& key, double now) {
  auto it = c->index.find(key);
  int64_t s;
  if (it != c->index.end()) {
    s = it->second;
    c->by_insert.erase({c->t_insert[s], s});
    c->by_use.erase({c->t_use[s], s});
  } else {
    s = victim(c, now);
    c->index[key] = s;
    c->slot_key[s] = key;
    c->used[s] = true;
  }
  c->t_insert[s] = now;
  c->t_use[s] = now;
  c->by_insert.insert({now, s});
  c->by_use.insert({now, s});
  return s;
}

// ------------------------------------------------------------------ device data movement

// out[b] = pool[slot[b]] for slot[b] >= 0 (k*d floats and k masses per entry).
__global__ void cache_gather_kernel(const float4* __restrict__ pool_x, const float* __restrict__ pool_m,
                                    const int64_t* __restrict__ slot, int64_t batch, int kd4, int k,
                                    float4* __restrict__ out_x, float* __restrict__ out_m) {
  const int64_t n = batch * kd4;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = e / kd4;
    const int64_t s = slot[b];
    if (s < 0) continue;
    const int64_t i = e % kd4;
    out_x[e] = pool_x[s * kd4 + i];
    if (i < k) out_m[b * k + i] = pool_m[s * k + i];
  }
}

// pool[slot[b]] = in[b] for slot[b] >= 0; or, with `to_pool` false,
// out[slot[b]] = in[b] (the compacted results back to the batch's positions).
__global__ void cache_scatter_kernel(const float4* __restrict__ in_x, const float* __restrict__ in_m,
                                     const int64_t* __restrict__ slot, int64_t batch, int kd4, int k,
                                     float4* __restrict__ dst_x, float* __restrict__ dst_m) {
  const int64_t n = batch * kd4;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = e / kd4;
    const int64_t s = slot[b];
    if (s < 0) continue;
    const int64_t i = e % kd4;
    dst_x[s * kd4 + i] = in_x[e];
    if (i < k) dst_m[s * k + i] = in_m[b * k + i];
  }
}

unsigned grid_for_elems(int64_t n) {
  const int64_t g = (n + 255) / 256;
  return static_cast<unsigned>(g < 8192 ? (g > 0 ? g : 1) : 8192);
}

bool ensure_slots(sa_cache_s* c, int64_t n, cudaStream_t st) {
  if (n <= c->d_slots_cap) return true;
  // The old list may still be read by a kernel enqueued earlier.
  if (c->d_slots != nullptr && (cudaStreamSynchronize(st) != cudaSuccess || cudaFree(c->d_slots) != cudaSuccess))
    return false;
  c->d_slots = nullptr;
  c->d_slots_cap = 0;
  const int64_t cap = std::max<int64_t>(n, 256);
  if (cudaMalloc(&c->d_slots, cap * sizeof(int64_t)) != cudaSuccess) return false;
  c->d_slots_cap = cap;
  return true;
}

// The staging half of a call that copies at most n values: its copies of
// two calls ago are waited for, then it is reset (and grown if needed).
SaStaging* begin_call(sa_cache_s* c, size_t n) {
  SaStaging* s = &c->stg[c->calls & 1];
  if (s->recorded && cudaEventSynchronize(s->ev) != cudaSuccess) return nullptr;
  s->recorded = false;
  if (s->ev == nullptr && cudaEventCreateWithFlags(&s->ev, cudaEventDisableTiming) != cudaSuccess)
    return nullptr;
  if (n > s->cap) {
    cudaFreeHost(s->host);
    s->host = nullptr;
    s->cap = 0;
    const size_t cap = std::max<size_t>(n, 1024);
    if (cudaMallocHost(&s->host, cap * sizeof(int64_t)) != cudaSuccess) return nullptr;
    s->cap = cap;
  }
  s->used = 0;
  return s;
}

// Marks the end of a call's copies on the stream.
bool end_call(sa_cache_s* c, SaStaging* s, cudaStream_t st) {
  ++c->calls;
  s->recorded = cudaEventRecord(s->ev, st) == cudaSuccess;
  return s->recorded;
}

// Copies a host vector to the device through the call's pinned staging.
bool upload(SaStaging* s, int64_t* dst, const std::vector<int64_t>& v, cudaStream_t st) {
  if (v.empty()) return true;
  if (s->used + v.size() > s->cap) return false;
  int64_t* h = s->host + s->used;
  std::copy(v.begin(), v.end(), h);
  s->used += v.size();
  return cudaMemcpyAsync(dst, h, v.size() * sizeof(int64_t), cudaMemcpyHostToDevice, st) ==
         cudaSuccess;
}

sa_status lookup_impl(sa_cache_s* c, SaStaging* sg, const sa_cache_key* keys, int64_t batch,
                      double now, uint8_t* hit, float* X_tilde, float* mass, cudaStream_t st) {
  std::vector<int64_t> slots(batch);
  for (int64_t b = 0; b < batch; ++b) {
    slots[b] = lookup_one(c, keys[b], now);
    hit[b] = slots[b] >= 0 ? 1 : 0;
  }
  if (!ensure_slots(c, batch, st) || !upload(sg, c->d_slots, slots, st)) return SA_ERR_CUDA;
  const int kd4 = c->k * c->d / 4;
  cache_gather_kernel<<<grid_for_elems(batch * kd4), 256, 0, st>>>(
      reinterpret_cast<const float4*>(c->pool_x), c->pool_m, c->d_slots, batch, kd4, c->k,
      reinterpret_cast<float4*>(X_tilde), mass);
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status insert_impl(sa_cache_s* c, SaStaging* sg, const sa_cache_key* keys, int64_t batch,
                      double now, const float* X_tilde, const float* mass, cudaStream_t st) {
  std::vector<int64_t> slots(batch);
  for (int64_t b = 0; b < batch; ++b) slots[b] = insert_one(c, keys[b], now);
  // Two equal keys in one batch share a slot: only the later one is copied.
  std::map<int64_t, int64_t> last;
  for (int64_t b = 0; b < batch; ++b) last[slots[b]] = b;
  for (int64_t b = 0; b < batch; ++b)
    if (last[slots[b]] != b) slots[b] = -1;
  if (!ensure_slots(c, batch, st) || !upload(sg, c->d_slots, slots, st)) return SA_ERR_CUDA;
  const int kd4 = c->k * c->d / 4;
  cache_scatter_kernel<<<grid_for_elems(batch * kd4), 256, 0, st>>>(
      reinterpret_cast<const float4*>(X_tilde), mass, c->d_slots, batch, kd4, c->k,
      reinterpret_cast<float4*>(c->pool_x), c->pool_m);
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

// ------------------------------------------------------------------ width adapter

constexpr int kAdThreads = 128;
constexpr int kAdN = 256;  // output columns per CTA

template <int KD>
struct AdPlan {
  static constexpr int kABox = 128 * 128;      // 128 rows x 64 bf16
  static constexpr int kBBox = kAdN * 128;     // 256 rows x 64 bf16
  static constexpr int kA = 0;
  static constexpr int kB = (KD / 64) * kABox;
  static constexpr int kBars = kB + (KD / 64) * kBBox;
  static constexpr int kSmem = kBars + 64;
};

__device__ __forceinline__ uint32_t swz(int r, int u) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((u ^ (r & 7)) << 4);
}

template <int KD>
__global__ void __launch_bounds__(kAdThreads, 1)
    adapter_kernel(const __grid_constant__ CUtensorMap tm_w, const float* __restrict__ X,
                   int64_t rows, int Dout, uint16_t* __restrict__ Y, uint32_t* flags) {
  using Pl = AdPlan<KD>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5;
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (tid == 0 && flags != nullptr) atomicOr(flags, DEVFLAG_SMEM_ALIGN);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Pl::kBars);
  uint64_t* w_full = bars;
  uint64_t* mma_done = bars + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  uint32_t* local_flags = tmem_slot + 2;
  if (tid == 0) {
    mbar_init(w_full, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0u;
    *local_flags = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  uint32_t* sticky = flags != nullptr ? flags : local_flags;
  const uint32_t tmem = *tmem_slot;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 128;
  const int n0 = blockIdx.y * kAdN;
  if (tid == 0) {
    mbar_arrive_expect_tx(w_full, kAdN * KD * 2);
#pragma unroll
    for (int b = 0; b < KD / 64; ++b)
      tma_load_2d(smem + Pl::kB + b * Pl::kBBox, &tm_w, w_full, b * 64, n0);
  }
  // This thread's sketch row, rounded to bf16, into the A operand.
  const int64_t r = r0 + tid;
  const bool valid = r < rows;
#pragma unroll
  for (int b = 0; b < KD / 64; ++b)
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo;
      if (valid) {
        const float4* src = reinterpret_cast<const float4*>(X + r * KD + b * 64 + u * 8);
        lo = src[0];
        hi = src[1];
      }
      st_shared_v4(sbase + Pl::kA + b * Pl::kABox + swz(tid, u), pack_bf16x2(lo.x, lo.y),
                   pack_bf16x2(lo.z, lo.w), pack_bf16x2(hi.x, hi.y), pack_bf16x2(hi.z, hi.w));
    }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  bool issued = false;
  if (tid == 0 && mbar_wait(w_full, 0, abort_flag, sticky)) {
    issued = true;
    tc_fence_after();
    const uint64_t da = smem_desc(sbase + Pl::kA, 16, 1024, 2);
    const uint64_t db = smem_desc(sbase + Pl::kB, 16, 1024, 2);
    constexpr uint32_t idesc = idesc_bf16_f32(128, kAdN, 0, 0);
#pragma unroll
    for (int ks = 0; ks < KD / 16; ++ks)
      mma_bf16_ss(tmem, da + (((ks >> 2) * Pl::kABox + (ks & 3) * 32) >> 4),
                  db + (((ks >> 2) * Pl::kBBox + (ks & 3) * 32) >> 4), idesc, ks > 0 ? 1u : 0u);
    mma_commit(mma_done);
  }
  if (!*abort_flag && mbar_wait(mma_done, 0, abort_flag, sticky)) {
    tc_fence_after();
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
    for (int cc = 0; cc < kAdN / 32; ++cc) {
      uint32_t v[32];
      tmem_ld32(lane_addr + cc * 32, v);
      tmem_wait_ld();
      tmem_pin32(v);
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(Y + r * Dout + n0 + cc * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          dst[u] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * u]), __uint_as_float(v[8 * u + 1])),
                              pack_bf16x2(__uint_as_float(v[8 * u + 2]), __uint_as_float(v[8 * u + 3])),
                              pack_bf16x2(__uint_as_float(v[8 * u + 4]), __uint_as_float(v[8 * u + 5])),
                              pack_bf16x2(__uint_as_float(v[8 * u + 6]), __uint_as_float(v[8 * u + 7])));
      }
    }
  }
  if (*abort_flag && tid == 0) {
    // A wait gave up: let the copy and any issued MMAs finish before the
    // shared memory and TMEM are released.
    mbar_wait_bounded(w_full, 0);
    if (issued) mbar_wait_bounded(mma_done, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

__global__ void transpose_w_kernel(const float* __restrict__ W, int d, int D, uint16_t* __restrict__ out) {
  const int64_t n = static_cast<int64_t>(d) * D;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t c = e / d, i = e % d;  // out[c][i] = W[i][c]
    out[e] = __bfloat16_as_ushort(__float2bfloat16_rn(W[i * D + c]));
  }
}

template <int KD>
cudaError_t launch_adapter(const sa_adapter_s* ad, const float* X, int64_t rows, uint16_t* Y,
                           uint32_t* flags, cudaStream_t st) {
  using Pl = AdPlan<KD>;
  cudaError_t err = cudaFuncSetAttribute(adapter_kernel<KD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Pl::kSmem);
  if (err != cudaSuccess) return err;
  const dim3 grid(static_cast<unsigned>((rows + 127) / 128), static_cast<unsigned>(ad->D / kAdN));
  adapter_kernel<KD><<<grid, kAdThreads, Pl::kSmem, st>>>(ad->tm_w, X, rows, ad->D, Y, flags);
  return cudaGetLastError();
}

bool al(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The caller's current device is the one the object's memory lives on.
bool on_device(int device) {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev == device;
}

size_t rup(size_t x) { return (x + 255) / 256 * 256; }

sa_status forward_impl(sa_cache_s* c, SaStaging* sg, sa_query q, const sa_cache_key* keys,
                       double now, const void* X, const int64_t* offsets_host, int64_t batch,
                       int64_t total_rows, int k, int d, int dt, float* X_tilde, float* mass,
                       uint8_t* hit, void* workspace, cudaStream_t st) {
  // Hits go straight to the outputs.
  sa_status s = lookup_impl(c, sg, keys, batch, now, hit, X_tilde, mass, st);
  if (s != SA_OK) return s;
  // A run of consecutive missed users owns a contiguous range of X and of
  // the outputs: it is compressed in place by one SA layer over that range
  // (offsets taken relative to the run's first row), and inserted from the
  // outputs.  No rows are copied.
  std::vector<std::pair<int64_t, int64_t>> runs;  // [b0, b1)
  for (int64_t b = 0; b < batch;) {
    if (hit[b]) {
      ++b;
      continue;
    }
    int64_t e = b;
    while (e < batch && !hit[e]) ++e;
    runs.emplace_back(b, e);
    b = e;
  }
  if (runs.empty()) return SA_OK;
  std::vector<int64_t> loc;  // the runs' relative offsets, one after another
  std::vector<size_t> pos;
  for (const auto& r : runs) {
    pos.push_back(loc.size());
    for (int64_t b = r.first; b <= r.second; ++b) loc.push_back(offsets_host[b] - offsets_host[r.first]);
  }
  // The SA pass's workspace comes first, so that its device flags are read
  // with sa_read_device_status on the whole workspace.
  uint8_t* w = static_cast<uint8_t*>(workspace);
  void* ws_sa = w;
  const size_t ws_sa_cap = sa_workspace_bytes(q, batch, total_rows);
  int64_t* d_loc = reinterpret_cast<int64_t*>(w + rup(ws_sa_cap));
  if (!upload(sg, d_loc, loc, st)) return SA_ERR_CUDA;
  const size_t row_bytes = static_cast<size_t>(d) * (dt == SA_BF16 ? 2 : 4);
  const size_t kd = static_cast<size_t>(k) * d;
  for (size_t i = 0; i < runs.size(); ++i) {
    const int64_t b0 = runs[i].first, b1 = runs[i].second;
    const int64_t r0 = offsets_host[b0], nrows = offsets_host[b1] - r0;
    s = sketch_forward_flags(q, static_cast<const uint8_t*>(X) + r0 * row_bytes, d_loc + pos[i],
                             b1 - b0, nrows, X_tilde + b0 * kd, mass + b0 * k, ws_sa, ws_sa_cap, st,
                             i > 0);
    if (s != SA_OK) return s;
    s = insert_impl(c, sg, keys + b0, b1 - b0, now, X_tilde + b0 * kd, mass + b0 * k, st);
    if (s != SA_OK) return s;
  }
  return SA_OK;
}

}  // namespace
}  // namespace sa

extern "C" {

sa_status sa_cache_create(int k, int d, int64_t capacity, double ttl_seconds, sa_cache* out) {
  if (out == nullptr) return SA_ERR_INVALID_ARG;
  *out = nullptr;
  if (k < 1 || d < 4 || d % 4 != 0 || capacity < 1 || !(ttl_seconds > 0.0)) return SA_ERR_INVALID_ARG;
  // The pool's byte count, capacity * k * (d + 1) * 4, must not wrap.
  const uint64_t per_slot = static_cast<uint64_t>(k) * (static_cast<uint64_t>(d) + 1) * 4;
  if (static_cast<uint64_t>(capacity) > SIZE_MAX / per_slot) return SA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
  sa_cache_s* c = new (std::nothrow) sa_cache_s;
  if (c == nullptr) return SA_ERR_CUDA;
  c->device = dev;
  c->k = k;
  c->d = d;
  c->capacity = capacity;
  c->ttl = ttl_seconds;
  c->pool_x = nullptr;
  c->pool_m = nullptr;
  const size_t kd = static_cast<size_t>(k) * d;
  if (cudaMalloc(&c->pool_x, static_cast<size_t>(capacity) * kd * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&c->pool_m, static_cast<size_t>(capacity) * k * sizeof(float)) != cudaSuccess) {
    cudaFree(c->pool_x);
    delete c;
    return SA_ERR_CUDA;
  }
  try {
    c->slot_key.resize(capacity);
    c->used.assign(capacity, false);
    c->t_insert.assign(capacity, 0.0);
    c->t_use.assign(capacity, 0.0);
    for (int64_t s = 0; s < capacity; ++s) c->free_slots.insert(c->free_slots.end(), s);
  } catch (const std::bad_alloc&) {
    cudaFree(c->pool_x);
    cudaFree(c->pool_m);
    delete c;
    return SA_ERR_CUDA;
  }
  *out = c;
  return SA_OK;
}

void sa_cache_free(sa_cache c) {
  if (c == nullptr) return;
  // Kernels enqueued by earlier calls may still read the pool and the slot
  // list: wait for the cache's device (made current for this call only).
  int prev = -1;
  const bool switched = cudaGetDevice(&prev) == cudaSuccess && prev != c->device &&
                        cudaSetDevice(c->device) == cudaSuccess;
  cudaDeviceSynchronize();
  cudaFree(c->pool_x);
  cudaFree(c->pool_m);
  cudaFree(c->d_slots);
  for (auto& s : c->stg) {
    cudaFreeHost(s.host);
    if (s.ev != nullptr) cudaEventDestroy(s.ev);
  }
  if (switched) cudaSetDevice(prev);
  delete c;
}

sa_status sa_cache_lookup(sa_cache c, const sa_cache_key* keys, int64_t batch, double now,
                          uint8_t* hit, float* X_tilde, float* mass, void* stream) {
  if (c == nullptr || batch < 0 || !std::isfinite(now)) return SA_ERR_INVALID_ARG;
  if (batch == 0) return SA_OK;
  if (keys == nullptr || hit == nullptr || X_tilde == nullptr || mass == nullptr ||
      !sa::al(X_tilde, 16) || !sa::al(mass, 4) || !sa::on_device(c->device))
    return SA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(c->mu);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SaStaging* sg = sa::begin_call(c, static_cast<size_t>(batch));
  if (sg == nullptr) return SA_ERR_CUDA;
  sa_status s;
  try {
    s = sa::lookup_impl(c, sg, keys, batch, now, hit, X_tilde, mass, st);
  } catch (const std::bad_alloc&) {
    s = SA_ERR_CUDA;
  }
  return sa::end_call(c, sg, st) ? s : SA_ERR_CUDA;
}

sa_status sa_cache_insert(sa_cache c, const sa_cache_key* keys, int64_t batch, double now,
                          const float* X_tilde, const float* mass, void* stream) {
  if (c == nullptr || batch < 0 || !std::isfinite(now)) return SA_ERR_INVALID_ARG;
  if (batch == 0) return SA_OK;
  if (keys == nullptr || X_tilde == nullptr || mass == nullptr || !sa::al(X_tilde, 16) ||
      !sa::al(mass, 4) || !sa::on_device(c->device))
    return SA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(c->mu);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SaStaging* sg = sa::begin_call(c, static_cast<size_t>(batch));
  if (sg == nullptr) return SA_ERR_CUDA;
  sa_status s;
  try {
    s = sa::insert_impl(c, sg, keys, batch, now, X_tilde, mass, st);
  } catch (const std::bad_alloc&) {
    s = SA_ERR_CUDA;
  }
  return sa::end_call(c, sg, st) ? s : SA_ERR_CUDA;
}

sa_status sa_cache_stats(sa_cache c, int64_t* entries, int64_t* hits, int64_t* misses,
                         int64_t* evictions) {
  if (c == nullptr) return SA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(c->mu);
  if (entries) *entries = static_cast<int64_t>(c->index.size());
  if (hits) *hits = c->hits;
  if (misses) *misses = c->misses;
  if (evictions) *evictions = c->evictions;
  return SA_OK;
}

size_t sa_cache_forward_workspace_bytes(sa_query q, int64_t batch, int64_t total_rows) {
  int k = 0, d = 0, dt = 0, kp = 0;
  if (sa_query_info(q, &k, &d, &dt, &kp) != SA_OK || batch < 0 || total_rows < 0) return 0;
  return sa::rup(sa_workspace_bytes(q, batch, total_rows)) +
         sa::rup((2 * static_cast<size_t>(batch) + 1) * 8);
}

sa_status sa_cache_forward(sa_cache c, sa_query q, const sa_cache_key* keys, double now,
                           const void* X, const int64_t* offsets_host, int64_t batch,
                           int64_t total_rows, float* X_tilde, float* mass, uint8_t* hit,
                           void* workspace, size_t workspace_bytes, void* stream) {
  int k = 0, d = 0, dt = 0, kp = 0;
  if (c == nullptr || sa_query_info(q, &k, &d, &dt, &kp) != SA_OK) return SA_ERR_INVALID_ARG;
  if (k != c->k || d != c->d || batch < 0 || total_rows < 0 || !std::isfinite(now))
    return SA_ERR_INVALID_ARG;
  if (batch == 0) return total_rows == 0 ? SA_OK : SA_ERR_INVALID_ARG;
  if (keys == nullptr || offsets_host == nullptr || X_tilde == nullptr || mass == nullptr ||
      hit == nullptr || workspace == nullptr || (total_rows > 0 && X == nullptr) ||
      !sa::al(workspace, 256) || !sa::al(X, 16) || !sa::on_device(c->device))
    return SA_ERR_INVALID_ARG;
  if (offsets_host[0] != 0 || offsets_host[batch] != total_rows) return SA_ERR_INVALID_ARG;
  for (int64_t b = 0; b < batch; ++b)
    if (offsets_host[b] > offsets_host[b + 1]) return SA_ERR_INVALID_ARG;
  if (workspace_bytes < sa_cache_forward_workspace_bytes(q, batch, total_rows))
    return SA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(c->mu);
  // Lookup slots, the runs' offsets (at most 2 batch + 1) and insert slots.
  SaStaging* sg = sa::begin_call(c, 4 * static_cast<size_t>(batch) + 1);
  if (sg == nullptr) return SA_ERR_CUDA;
  sa_status s;
  try {
    s = sa::forward_impl(c, sg, q, keys, now, X, offsets_host, batch, total_rows, k, d, dt, X_tilde,
                         mass, hit, workspace, st);
  } catch (const std::bad_alloc&) {
    s = SA_ERR_CUDA;
  }
  return sa::end_call(c, sg, st) ? s : SA_ERR_CUDA;
}



sa_status sa_prepare_adapter(const float* W_A, int d, int D, void* stream, sa_adapter* out) {
  if (out == nullptr) return SA_ERR_INVALID_ARG;
  *out = nullptr;
  if (W_A == nullptr || !sa::al(W_A, 4)) return SA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || D < sa::kAdN || D % sa::kAdN != 0) return SA_ERR_INVALID_ARG;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return SA_ERR_CUDA;
  if (major != 10) return SA_ERR_UNSUPPORTED;
  sa_adapter_s* a = new (std::nothrow) sa_adapter_s;
  if (a == nullptr) return SA_ERR_CUDA;
  a->device = dev;
  a->d = d;
  a->D = D;
  a->wt = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool ok = cudaMalloc(&a->wt, static_cast<size_t>(d) * D * sizeof(uint16_t)) == cudaSuccess;
  if (ok) {
    sa::transpose_w_kernel<<<sa::grid_for_elems(static_cast<int64_t>(d) * D), 256, 0, st>>>(W_A, d, D, a->wt);
    ok = cudaGetLastError() == cudaSuccess &&
         sa::make_tmap_bf16(&a->tm_w, a->wt, static_cast<uint64_t>(D), static_cast<uint64_t>(d),
                            sa::kAdN);
  }
  if (!ok) {
    cudaFree(a->wt);
    delete a;
    return SA_ERR_CUDA;
  }
  *out = a;
  return SA_OK;
}

void sa_adapter_free(sa_adapter a) {
  if (a == nullptr) return;
  cudaFree(a->wt);
  delete a;
}

sa_status sa_adapter_forward(sa_adapter a, const float* X_tilde, int64_t rows, void* out,
                             uint32_t* device_flags, void* stream) {
  if (a == nullptr || rows < 0) return SA_ERR_INVALID_ARG;
  if (rows == 0) return SA_OK;
  if (X_tilde == nullptr || out == nullptr || !sa::al(X_tilde, 16) || !sa::al(out, 16) ||
      !sa::al(device_flags, 4))
    return SA_ERR_INVALID_ARG;
  if (rows > (int64_t{1} << 31) * 128 - 128) return SA_ERR_INVALID_ARG;
  if (!sa::on_device(a->device)) return SA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t err =
      a->d == 64 ? sa::launch_adapter<64>(a, X_tilde, rows, static_cast<uint16_t*>(out), device_flags, st)
                 : sa::launch_adapter<128>(a, X_tilde, rows, static_cast<uint16_t*>(out), device_flags, st);
  return err == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

}  // extern "C"
