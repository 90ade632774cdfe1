// C-ABI layer of libsa.so: argument checks, workspace layout, tensor maps
// and kernel launches.  See include/sa.h for the contract of each entry.
#include <math.h>
#include <string.h>

#include <new>

#include "sa.h"
#include "sa_internal.h"

struct sa_query_s {
  int device;
  int sms;
  int pair_units;  // co-resident two-CTA clusters (d == 256, k_pad == 256)
  int ncl;         // CTAs per prototype-split cluster (d <= 128, k > 128), else 1
  int cluster_units;  // co-resident clusters of ncl CTAs
  int k;
  int d;
  int k_pad;  // prototype rows of the bf16 Q' copy (multiple of 64), 0 for fp32
  sa_dtype dtype;
  double scale;      // affinity scale the query was prepared with
  float* q_f32;      // [k][d]
  uint16_t* q_bf16;  // [k_pad][d], rows >= k zero
  float* m_f32;      // [d][d]: W_Q W_K^T * scale * log2(e), for per-user queries
  CUtensorMap tmap_q;       // boxes of k_pad rows (k_pad <= 128), of 128 rows for clusters
  CUtensorMap tmap_q_half;  // boxes of 128 rows (k_pad == 256: one half per CTA of a pair)
};

namespace sa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_tmap_bf16_box(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                        uint32_t box_cols, uint32_t box_rows, int swizzle_bytes) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  CUtensorMapSwizzle sw;
  if (swizzle_bytes == 128 && box_cols == 64) {
    sw = CU_TENSOR_MAP_SWIZZLE_128B;
  } else if (swizzle_bytes == 32 && box_cols == 16) {
    sw = CU_TENSOR_MAP_SWIZZLE_32B;
  } else {
    return false;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
  return make_tmap_bf16_box(m, base, rows, cols, 64, box_rows, 128);
}

}  // namespace sa

namespace {

using sa::PassArgs;
using sa::make_tmap_bf16;

constexpr int64_t kMaxRows = (int64_t{1} << 31) - 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Number of CTA row ranges: one per SM, or one per pair of SMs for the
// two-CTA pass (256 padded prototypes).
int64_t grid_for(const sa_query_s* q, int64_t total_rows) {
  const int64_t T = sa::tiles_of(total_rows);
  const int64_t units = q->ncl > 1 ? q->cluster_units
                        : (q->dtype == SA_BF16 && q->k_pad == 256) ? q->pair_units
                                                                   : q->sms;
  int64_t G = T < units ? T : units;
  return G < 1 ? 1 : G;
}

struct WsLayout {
  size_t part_x_off, part_m_off, total;
};

WsLayout ws_layout(const sa_query_s* q, int64_t total_rows) {
  const size_t G = static_cast<size_t>(grid_for(q, total_rows));
  WsLayout l;
  l.part_x_off = sa::kWsHeaderBytes;
  l.part_m_off = round_up(l.part_x_off + 2 * G * q->k * q->d * sizeof(float), 256);
  l.total = round_up(l.part_m_off + 2 * G * q->k * sizeof(float), 256);
  return l;
}

// Per-user queries: rows per user of the per-call Q' array (k_pad for the
// bf16 copy the tensor-core pass reads, k for fp32) and its bytes, placed
// after the common workspace.
int uq_rows(const sa_query_s* q) { return q->dtype == SA_BF16 ? q->k_pad : q->k; }
size_t uq_bytes(const sa_query_s* q, int64_t batch) {
  const size_t elem = q->dtype == SA_BF16 ? 2 : 4;
  return round_up(static_cast<size_t>(batch) * uq_rows(q) * q->d * elem, 256);
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool same_device(const sa_query_s* q) {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev == q->device;
}

enum class Phase { kBoth, kPartials, kFinalize };

// `queries` (device, [batch][k][d] fp32) selects per-user queries; nullptr
// queries every user with the prepared Q'.
sa_status run(sa_query q, const float* queries, const void* X, const int64_t* offsets,
              int64_t batch, int64_t total_rows, float* X_tilde, float* mass, void* workspace,
              size_t workspace_bytes, void* stream, Phase phase, bool keep_flags = false) {
  if (q == nullptr) return SA_ERR_INVALID_ARG;
  if (batch < 0 || total_rows < 0 || total_rows > kMaxRows) return SA_ERR_INVALID_ARG;
  if (batch == 0) return total_rows == 0 ? SA_OK : SA_ERR_INVALID_ARG;
  if (offsets == nullptr || X_tilde == nullptr || mass == nullptr || workspace == nullptr)
    return SA_ERR_INVALID_ARG;
  if (total_rows > 0 && X == nullptr) return SA_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(X_tilde, 16) || !aligned(mass, 4) || !aligned(offsets, 8) ||
      !aligned(workspace, 256) || !aligned(queries, 4))
    return SA_ERR_INVALID_ARG;
  if (!same_device(q)) return SA_ERR_INVALID_ARG;
  const bool user_q = queries != nullptr;
  if (user_q) {
    // The tensor map's row coordinate b * k_pad is a 32-bit integer.
    if (batch > (int64_t{1} << 31) / (q->k_pad > 0 ? q->k_pad : 1) - 1) return SA_ERR_INVALID_ARG;
  }
  const WsLayout l = ws_layout(q, total_rows);
  if (workspace_bytes < l.total + (user_q ? uq_bytes(q, batch) : 0)) return SA_ERR_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  PassArgs a;
  a.offsets = offsets;
  a.batch = batch;
  a.total_rows = total_rows;
  a.tiles = sa::tiles_of(total_rows);
  a.k = q->k;
  a.d = q->d;
  a.out_x = X_tilde;
  a.out_m = mass;
  a.part_x = reinterpret_cast<float*>(ws + l.part_x_off);
  a.part_m = reinterpret_cast<float*>(ws + l.part_m_off);
  a.header = reinterpret_cast<sa::WsHeader*>(ws);
  a.user_queries = user_q ? 1 : 0;
  a.keep_flags = keep_flags ? 1 : 0;
  const int G = static_cast<int>(grid_for(q, total_rows));

  if (phase != Phase::kFinalize) {
    cudaError_t err;
    void* uq = ws + l.total;  // per-call Q'_b array (per-user queries)
    if (user_q &&
        sa::launch_user_query(queries, q->m_f32, batch, q->k, uq_rows(q), q->d,
                              q->dtype == SA_BF16 ? nullptr : static_cast<float*>(uq),
                              q->dtype == SA_BF16 ? static_cast<uint16_t*>(uq) : nullptr,
                              st) != cudaSuccess)
      return SA_ERR_CUDA;
    if (q->dtype == SA_BF16) {
      CUtensorMap tmq;
      if (user_q && !make_tmap_bf16(&tmq, uq, static_cast<uint64_t>(batch) * q->k_pad,
                                    static_cast<uint64_t>(q->d),
                                    static_cast<uint32_t>(q->k_pad > 128 ? 128 : q->k_pad)))
        return SA_ERR_CUDA;
      CUtensorMap tmx;
      // A zero-row tensor map is not encodable; with N == 0 the kernel
      // issues no loads, so Q' stands in as a valid dummy.
      const bool ok = total_rows > 0
                          ? make_tmap_bf16(&tmx, X, static_cast<uint64_t>(total_rows),
                                           static_cast<uint64_t>(q->d), sa::kTileRows)
                          : make_tmap_bf16(&tmx, q->q_bf16, static_cast<uint64_t>(q->k_pad),
                                           static_cast<uint64_t>(q->d), 64);
      if (!ok) return SA_ERR_CUDA;
      const CUtensorMap& tq = user_q ? tmq : q->tmap_q;
      err = q->ncl > 1 ? sa::launch_fused_bf16_cluster(tmx, tq, a, G, q->ncl, st)
            : q->k_pad == 256 ? sa::launch_fused_bf16_pair(tmx, user_q ? tmq : q->tmap_q_half, a,
                                                           G, st)
                              : sa::launch_fused_bf16(tmx, tq, q->k_pad, a, G, st);
    } else {
      err = sa::launch_simt_fp32(user_q ? static_cast<const float*>(uq) : q->q_f32,
                                 static_cast<const float*>(X), a, G, st);
    }
    if (err != cudaSuccess) return SA_ERR_CUDA;
  }
  if (phase != Phase::kPartials) {
    if (sa::launch_finalize(a, G, st) != cudaSuccess) return SA_ERR_CUDA;
  }
  return SA_OK;
}

}  // namespace

extern "C" {

const char* sa_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID_ARG: return "invalid argument";
    case SA_ERR_UNSUPPORTED: return "unsupported shape, dtype or GPU";
    case SA_ERR_WORKSPACE: return "workspace too small";
    case SA_ERR_CUDA: return "CUDA error";
    case SA_ERR_DEVICE_FLAG: return "device flagged bad offsets or a timed-out wait";
  }
  return "unknown status";
}

sa_status sa_prepare_query(const void* P, const void* W_Q, const void* W_K, int k, int d,
                           float scale, sa_dtype dtype, void* stream, sa_query* out) {
  if (out == nullptr) return SA_ERR_INVALID_ARG;
  *out = nullptr;
  if (P == nullptr || W_Q == nullptr || W_K == nullptr) return SA_ERR_INVALID_ARG;
  if (k < 1 || k > 1024 || !(d == 64 || d == 128 || d == 256) || !isfinite(scale))
    return SA_ERR_INVALID_ARG;
  if (dtype != SA_BF16 && dtype != SA_FP32) return SA_ERR_INVALID_ARG;
  const size_t elem = dtype == SA_BF16 ? 2 : 4;
  if (!aligned(P, elem) || !aligned(W_Q, elem) || !aligned(W_K, elem)) return SA_ERR_INVALID_ARG;

  int dev = 0, major = 0, minor = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return SA_ERR_CUDA;
  if (major != 10 || minor != 0) return SA_ERR_UNSUPPORTED;  // built for sm_100a only

  int k_pad = 0;
  int ncl = 1;
  if (dtype == SA_BF16) {
    // d = 256 with more than 64 prototypes runs on CTA pairs (256 padded);
    // d = 64 or 128 with more than 128 on clusters of ceil(k / 128) CTAs.
    if (d != 256 && k > 128) {
      ncl = (k + 127) / 128;
      k_pad = 128 * ncl;
    } else {
      k_pad = k <= 64 ? 64 : ((k <= 128 && d != 256) ? 128 : 256);
      if (k > 256 || !sa::fused_bf16_supported(d, k_pad)) return SA_ERR_UNSUPPORTED;
    }
  } else if (k > 256) {
    return SA_ERR_UNSUPPORTED;  // the fp32 pass keeps k <= 256 accumulators per thread row
  }

  sa_query_s* q = new (std::nothrow) sa_query_s;
  if (q == nullptr) return SA_ERR_CUDA;
  memset(q, 0, sizeof(*q));
  q->device = dev;
  q->sms = sms;
  q->ncl = ncl;
  if (ncl > 1) {
    const int n = sa::fused_bf16_cluster_max_clusters(d, ncl);
    if (n < 1) {
      delete q;
      return SA_ERR_UNSUPPORTED;
    }
    q->cluster_units = n < sms / ncl ? n : sms / ncl;
  } else if (dtype == SA_BF16 && k_pad == 256) {
    const int n = sa::fused_bf16_pair_max_clusters();
    if (n < 1) {
      delete q;
      return SA_ERR_UNSUPPORTED;
    }
    q->pair_units = n < sms / 2 ? n : sms / 2;
  }
  q->k = k;
  q->d = d;
  q->k_pad = k_pad;
  q->dtype = dtype;
  q->scale = static_cast<double>(scale);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool ok = cudaMalloc(&q->q_f32, static_cast<size_t>(k) * d * sizeof(float)) == cudaSuccess;
  if (ok && dtype == SA_BF16) {
    const size_t qb = static_cast<size_t>(k_pad) * d * sizeof(uint16_t);
    ok = cudaMalloc(&q->q_bf16, qb) == cudaSuccess && cudaMemsetAsync(q->q_bf16, 0, qb, st) == cudaSuccess;
    const bool pair = ncl == 1 && k_pad == 256;
    ok = ok && make_tmap_bf16(pair ? &q->tmap_q_half : &q->tmap_q, q->q_bf16,
                              static_cast<uint64_t>(k_pad), static_cast<uint64_t>(d),
                              static_cast<uint32_t>(k_pad > 128 ? 128 : k_pad));
  }
  ok = ok && cudaMalloc(&q->m_f32, static_cast<size_t>(d) * d * sizeof(float)) == cudaSuccess;
  ok = ok && sa::launch_prepare_query(P, W_Q, W_K, k, d, static_cast<double>(scale),
                                      dtype == SA_BF16, q->q_f32, q->q_bf16, st) == cudaSuccess;
  ok = ok && sa::launch_prepare_projection(W_Q, W_K, d, static_cast<double>(scale),
                                           dtype == SA_BF16, q->m_f32, st) == cudaSuccess;
  if (!ok) {
    cudaFree(q->q_f32);
    cudaFree(q->q_bf16);
    cudaFree(q->m_f32);
    delete q;
    return SA_ERR_CUDA;
  }
  *out = q;
  return SA_OK;
}

void sa_sketch_free(sa_query q) {
  if (q == nullptr) return;
  cudaFree(q->q_f32);
  cudaFree(q->q_bf16);
  cudaFree(q->m_f32);
  delete q;
}

sa_status sa_query_info(sa_query q, int* k, int* d, int* dtype, int* k_pad) {
  if (q == nullptr) return SA_ERR_INVALID_ARG;
  if (k) *k = q->k;
  if (d) *d = q->d;
  if (dtype) *dtype = static_cast<int>(q->dtype);
  if (k_pad) *k_pad = q->k_pad;
  return SA_OK;
}

size_t sa_workspace_bytes(sa_query q, int64_t batch, int64_t total_rows) {
  (void)batch;
  if (q == nullptr || total_rows < 0) return 0;
  return ws_layout(q, total_rows).total;
}

sa_status sa_sketch_forward(sa_query q, const void* X, const int64_t* offsets, int64_t batch,
                            int64_t total_rows, float* X_tilde, float* mass, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return run(q, nullptr, X, offsets, batch, total_rows, X_tilde, mass, workspace, workspace_bytes,
             stream, Phase::kBoth);
}

}  // extern "C"

namespace sa {
sa_status sketch_forward_flags(sa_query q, const void* X, const int64_t* offsets, int64_t batch,
                               int64_t total_rows, float* X_tilde, float* mass, void* workspace,
                               size_t workspace_bytes, void* stream, bool keep_flags) {
  return run(q, nullptr, X, offsets, batch, total_rows, X_tilde, mass, workspace, workspace_bytes,
             stream, Phase::kBoth, keep_flags);
}
}  // namespace sa

extern "C" {

sa_status sa_sketch_partials(sa_query q, const void* X, const int64_t* offsets, int64_t batch,
                             int64_t total_rows, float* X_tilde, float* mass, void* workspace,
                             size_t workspace_bytes, void* stream) {
  return run(q, nullptr, X, offsets, batch, total_rows, X_tilde, mass, workspace, workspace_bytes,
             stream, Phase::kPartials);
}

sa_status sa_sketch_finalize(sa_query q, const void* X, const int64_t* offsets, int64_t batch,
                             int64_t total_rows, float* X_tilde, float* mass, void* workspace,
                             size_t workspace_bytes, void* stream) {
  return run(q, nullptr, X, offsets, batch, total_rows, X_tilde, mass, workspace, workspace_bytes,
             stream, Phase::kFinalize);
}

size_t sa_workspace_bytes_user_queries(sa_query q, int64_t batch, int64_t total_rows) {
  if (q == nullptr || batch < 0 || total_rows < 0) return 0;
  return ws_layout(q, total_rows).total + uq_bytes(q, batch);
}

sa_status sa_sketch_forward_user_queries(sa_query q, const float* queries, const void* X,
                                         const int64_t* offsets, int64_t batch,
                                         int64_t total_rows, float* X_tilde, float* mass,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  if (batch > 0 && queries == nullptr) return SA_ERR_INVALID_ARG;
  return run(q, queries, X, offsets, batch, total_rows, X_tilde, mass, workspace,
             workspace_bytes, stream, Phase::kBoth);
}

sa_status sa_sketch_partials_user_queries(sa_query q, const float* queries, const void* X,
                                          const int64_t* offsets, int64_t batch,
                                          int64_t total_rows, float* X_tilde, float* mass,
                                          void* workspace, size_t workspace_bytes, void* stream) {
  if (batch > 0 && queries == nullptr) return SA_ERR_INVALID_ARG;
  return run(q, queries, X, offsets, batch, total_rows, X_tilde, mass, workspace,
             workspace_bytes, stream, Phase::kPartials);
}

size_t sa_host_path_device_bytes(sa_query q, int64_t batch, int64_t total_rows) {
  if (q == nullptr || batch < 0 || total_rows < 0) return 0;
  const size_t elem = q->dtype == SA_BF16 ? 2 : 4;
  size_t s = round_up(static_cast<size_t>(total_rows) * q->d * elem, 256);
  s += round_up(static_cast<size_t>(batch + 1) * sizeof(int64_t), 256);
  s += round_up(static_cast<size_t>(batch) * q->k * q->d * sizeof(float), 256);
  s += round_up(static_cast<size_t>(batch) * q->k * sizeof(float), 256);
  s += ws_layout(q, total_rows).total;
  return s;
}

sa_status sa_sketch_forward_host(sa_query q, const void* X_host, const int64_t* offsets_host,
                                 int64_t batch, int64_t total_rows, float* X_tilde_host,
                                 float* mass_host, void* device_buffer,
                                 size_t device_buffer_bytes, void* stream) {
  if (q == nullptr || offsets_host == nullptr || batch < 0 || total_rows < 0 ||
      total_rows > kMaxRows)
    return SA_ERR_INVALID_ARG;
  if (batch == 0) return total_rows == 0 ? SA_OK : SA_ERR_INVALID_ARG;
  if (X_tilde_host == nullptr || mass_host == nullptr || device_buffer == nullptr ||
      (total_rows > 0 && X_host == nullptr) || !aligned(device_buffer, 256))
    return SA_ERR_INVALID_ARG;
  if (offsets_host[0] != 0 || offsets_host[batch] != total_rows) return SA_ERR_INVALID_ARG;
  for (int64_t b = 0; b < batch; ++b)
    if (offsets_host[b] > offsets_host[b + 1]) return SA_ERR_INVALID_ARG;
  if (device_buffer_bytes < sa_host_path_device_bytes(q, batch, total_rows))
    return SA_ERR_WORKSPACE;

  const size_t elem = q->dtype == SA_BF16 ? 2 : 4;
  const size_t x_bytes = static_cast<size_t>(total_rows) * q->d * elem;
  const size_t o_bytes = static_cast<size_t>(batch + 1) * sizeof(int64_t);
  const size_t xt_bytes = static_cast<size_t>(batch) * q->k * q->d * sizeof(float);
  const size_t m_bytes = static_cast<size_t>(batch) * q->k * sizeof(float);
  uint8_t* p = static_cast<uint8_t*>(device_buffer);
  void* x_dev = p;
  p += round_up(x_bytes, 256);
  int64_t* o_dev = reinterpret_cast<int64_t*>(p);
  p += round_up(o_bytes, 256);
  float* xt_dev = reinterpret_cast<float*>(p);
  p += round_up(xt_bytes, 256);
  float* m_dev = reinterpret_cast<float*>(p);
  p += round_up(m_bytes, 256);
  void* ws = p;
  const size_t ws_bytes = ws_layout(q, total_rows).total;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (x_bytes > 0 && cudaMemcpyAsync(x_dev, X_host, x_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return SA_ERR_CUDA;
  if (cudaMemcpyAsync(o_dev, offsets_host, o_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return SA_ERR_CUDA;
  sa_status s = run(q, nullptr, x_dev, o_dev, batch, total_rows, xt_dev, m_dev, ws, ws_bytes,
                    stream, Phase::kBoth);
  if (s != SA_OK) return s;
  if (cudaMemcpyAsync(X_tilde_host, xt_dev, xt_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(mass_host, m_dev, m_bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SA_ERR_CUDA;
  return SA_OK;
}

size_t sa_workspace_bytes_refine_layer(sa_query q, int64_t batch, int64_t total_rows) {
  if (q == nullptr || batch < 0 || total_rows < 0) return 0;
  const size_t kd = static_cast<size_t>(q->k) * q->d;
  return round_up(ws_layout(q, total_rows).total + uq_bytes(q, batch), 256) +
         round_up(static_cast<size_t>(batch) * kd * sizeof(float), 256) +
         round_up(static_cast<size_t>(batch) * q->k * sizeof(float), 256);
}

namespace {

// One refinement layer: the SA step (shared query when prev is null, else
// per-user queries prev) into the workspace, then the update into out.
sa_status refine_layer(sa_query q, sa_refine r, const float* prev, const float* P_f32,
                       const void* X, const int64_t* offsets, int64_t batch, int64_t total_rows,
                       float* out, void* workspace, size_t workspace_bytes, void* stream,
                       bool keep_flags) {
  if (q == nullptr || r == nullptr || out == nullptr) return SA_ERR_INVALID_ARG;
  if (q->dtype != SA_BF16) return SA_ERR_UNSUPPORTED;
  if (sa::refine_width(r) != q->d) return SA_ERR_INVALID_ARG;
  if (prev == nullptr && P_f32 == nullptr) return SA_ERR_INVALID_ARG;
  if (batch < 0 || total_rows < 0) return SA_ERR_INVALID_ARG;
  if (batch == 0) return total_rows == 0 ? SA_OK : SA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(prev, 16) || !aligned(P_f32, 16) || !aligned(workspace, 256))
    return SA_ERR_INVALID_ARG;
  if (workspace == nullptr) return SA_ERR_INVALID_ARG;
  if (workspace_bytes < sa_workspace_bytes_refine_layer(q, batch, total_rows))
    return SA_ERR_WORKSPACE;
  const size_t kd = static_cast<size_t>(q->k) * q->d;
  const size_t sa_bytes = round_up(ws_layout(q, total_rows).total + uq_bytes(q, batch), 256);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* xt = reinterpret_cast<float*>(ws + sa_bytes);
  float* m = reinterpret_cast<float*>(ws + sa_bytes +
                                      round_up(static_cast<size_t>(batch) * kd * sizeof(float), 256));
  sa_status s = run(q, prev, X, offsets, batch, total_rows, xt, m, workspace, sa_bytes, stream,
                    Phase::kBoth, keep_flags);
  if (s != SA_OK) return s;
  sa::WsHeader* hdr = reinterpret_cast<sa::WsHeader*>(ws);
  return sa::launch_refine_update(r, prev != nullptr ? prev : P_f32, prev == nullptr, xt, m,
                                  batch, q->k, out, &hdr->timeout_flags,
                                  static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SA_OK
             : SA_ERR_CUDA;
}

}  // namespace

sa_status sa_refine_layer_forward(sa_query q, sa_refine r, const float* prev, const float* P_f32,
                                  const void* X, const int64_t* offsets, int64_t batch,
                                  int64_t total_rows, float* out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  return refine_layer(q, r, prev, P_f32, X, offsets, batch, total_rows, out, workspace,
                      workspace_bytes, stream, false);
}

size_t sa_workspace_bytes_action_sketch(sa_query q, int64_t batch, int64_t total_rows) {
  if (q == nullptr || batch < 0 || total_rows < 0) return 0;
  return round_up(ws_layout(q, total_rows).total, 256) +
         round_up(static_cast<size_t>(total_rows) * q->d * 2, 256);
}

sa_status sa_action_sketch_forward(sa_action act, sa_query q, const void* E, const uint8_t* types,
                                   const int64_t* offsets, int64_t batch, int64_t total_rows,
                                   float* X_tilde, float* mass, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  if (act == nullptr || q == nullptr) return SA_ERR_INVALID_ARG;
  if (q->dtype != SA_BF16) return SA_ERR_UNSUPPORTED;
  int ad = 0, adev = -1;
  sa::action_info(act, &ad, &adev);
  if (ad != q->d || adev != q->device || !same_device(q)) return SA_ERR_INVALID_ARG;
  if (batch < 0 || total_rows < 0 || total_rows >= kMaxRows) return SA_ERR_INVALID_ARG;
  if (batch == 0) return total_rows == 0 ? SA_OK : SA_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned(workspace, 256)) return SA_ERR_INVALID_ARG;
  if (total_rows > 0 && (E == nullptr || types == nullptr || !aligned(E, 16)))
    return SA_ERR_INVALID_ARG;
  if (workspace_bytes < sa_workspace_bytes_action_sketch(q, batch, total_rows))
    return SA_ERR_WORKSPACE;
  // X goes after the SA pass's workspace.  The flag words are cleared here
  // and kept by the SA pass, so that the producer's bits survive it.
  const size_t sa_bytes = round_up(ws_layout(q, total_rows).total, 256);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* X = ws + sa_bytes;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  sa::WsHeader* hdr = reinterpret_cast<sa::WsHeader*>(ws);
  if (cudaMemsetAsync(hdr, 0, 2 * sizeof(uint32_t), st) != cudaSuccess) return SA_ERR_CUDA;
  if (total_rows > 0) {
    const sa_status s =
        sa::action_fuse_enqueue(act, E, types, total_rows, X, &hdr->timeout_flags, st);
    if (s != SA_OK) return s;
  }
  return run(q, nullptr, X, offsets, batch, total_rows, X_tilde, mass, workspace, sa_bytes, stream,
             Phase::kBoth, true);
}

size_t sa_workspace_bytes_refine_stack(sa_query q, int64_t batch, int64_t total_rows) {
  if (q == nullptr || batch < 0 || total_rows < 0) return 0;
  return sa_workspace_bytes_refine_layer(q, batch, total_rows) +
         round_up(static_cast<size_t>(batch) * q->k * q->d * sizeof(float), 256);
}

sa_status sa_refine_stack_forward(int layers, const sa_query* qs, const sa_refine* rs,
                                  const float* P_f32, const void* X, const int64_t* offsets,
                                  int64_t batch, int64_t total_rows, float* out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (layers < 1 || qs == nullptr || rs == nullptr || P_f32 == nullptr) return SA_ERR_INVALID_ARG;
  for (int l = 0; l < layers; ++l) {
    if (qs[l] == nullptr || rs[l] == nullptr) return SA_ERR_INVALID_ARG;
    if (qs[l]->k != qs[0]->k || qs[l]->d != qs[0]->d) return SA_ERR_INVALID_ARG;
  }
  if (batch < 0 || total_rows < 0) return SA_ERR_INVALID_ARG;
  if (batch == 0) return total_rows == 0 ? SA_OK : SA_ERR_INVALID_ARG;
  if (out == nullptr || workspace == nullptr) return SA_ERR_INVALID_ARG;
  if (workspace_bytes < sa_workspace_bytes_refine_stack(qs[0], batch, total_rows))
    return SA_ERR_WORKSPACE;
  // Layer outputs alternate between `out` and a buffer after the layer
  // workspace, so that the last layer writes `out` and no layer writes the
  // sketches it is queried with.
  const size_t layer_bytes = sa_workspace_bytes_refine_layer(qs[0], batch, total_rows);
  float* tmp = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + layer_bytes);
  const float* prev = nullptr;
  for (int l = 0; l < layers; ++l) {
    float* dst = ((layers - 1 - l) % 2 == 0) ? out : tmp;
    const sa_status s = refine_layer(qs[l], rs[l], prev, P_f32, X, offsets, batch, total_rows, dst,
                                     workspace, layer_bytes, stream, l > 0);
    if (s != SA_OK) return s;
    prev = dst;
  }
  return SA_OK;
}

namespace {

struct BwdLayout {
  size_t gb, gp, r, m, rs, tmp, t, uq, total;
};

BwdLayout bwd_layout(const sa_query_s* q, int64_t batch, int64_t total_rows) {
  const size_t B = static_cast<size_t>(batch), k = q->k, d = q->d, kp = q->k_pad;
  BwdLayout l;
  l.gb = round_up(ws_layout(q, total_rows).total, 256);
  l.gp = l.gb + round_up(B * kp * d * 2, 256);
  l.r = l.gp + round_up(B * kp * 4, 256);
  l.m = l.r + round_up(B * k * d * 4, 256);
  l.rs = l.m + round_up(B * k * 4, 256);
  l.tmp = l.rs + round_up(k * d * 4, 256);
  l.t = l.tmp + round_up(B * k * d * 4, 256);
  l.uq = l.t + round_up(d * d * 4, 256);
  l.total = l.uq + round_up(B * kp * d * 2, 256);
  return l;
}

}  // namespace

size_t sa_workspace_bytes_backward(sa_query q, int64_t batch, int64_t total_rows) {
  if (q == nullptr || batch < 0 || total_rows < 0) return 0;
  return bwd_layout(q, batch, total_rows).total;
}

sa_status sa_sketch_backward(sa_query q, const float* queries, const float* P_f32,
                             const float* W_Q_f32, const float* W_K_f32, const void* X,
                             const int64_t* offsets, int64_t batch, int64_t total_rows,
                             const float* G, const float* g, void* dX, float* dP, float* dW_Q,
                             float* dW_K, void* workspace, size_t workspace_bytes, void* stream) {
  if (q == nullptr) return SA_ERR_INVALID_ARG;
  if (q->dtype != SA_BF16 || q->ncl > 1 || !sa::backward_supported(q->d, q->k_pad))
    return SA_ERR_UNSUPPORTED;
  if (batch < 0 || total_rows < 0 || total_rows > kMaxRows) return SA_ERR_INVALID_ARG;
  if (batch == 0) return total_rows == 0 ? SA_OK : SA_ERR_INVALID_ARG;
  const bool user_q = queries != nullptr;
  if (offsets == nullptr || G == nullptr || dP == nullptr || dW_Q == nullptr || dW_K == nullptr ||
      W_Q_f32 == nullptr || W_K_f32 == nullptr || workspace == nullptr ||
      (!user_q && P_f32 == nullptr) || (total_rows > 0 && (X == nullptr || dX == nullptr)))
    return SA_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(dX, 16) || !aligned(offsets, 8) || !aligned(workspace, 256) ||
      !aligned(G, 4) || !aligned(g, 4) || !aligned(queries, 4) || !aligned(P_f32, 4) ||
      !aligned(W_Q_f32, 4) || !aligned(W_K_f32, 4) || !aligned(dP, 4) || !aligned(dW_Q, 4) ||
      !aligned(dW_K, 4))
    return SA_ERR_INVALID_ARG;
  if (!same_device(q)) return SA_ERR_INVALID_ARG;
  if (user_q && batch > (int64_t{1} << 31) / q->k_pad - 1) return SA_ERR_INVALID_ARG;
  const BwdLayout l = bwd_layout(q, batch, total_rows);
  if (workspace_bytes < l.total) return SA_ERR_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const WsLayout wl = ws_layout(q, total_rows);
  uint16_t* gb = reinterpret_cast<uint16_t*>(ws + l.gb);
  float* gp = reinterpret_cast<float*>(ws + l.gp);
  float* R = reinterpret_cast<float*>(ws + l.r);
  float* m = reinterpret_cast<float*>(ws + l.m);
  float* Rs = reinterpret_cast<float*>(ws + l.rs);
  float* tmp = reinterpret_cast<float*>(ws + l.tmp);
  float* T = reinterpret_cast<float*>(ws + l.t);
  uint16_t* uq = reinterpret_cast<uint16_t*>(ws + l.uq);
  const int k = q->k, d = q->d, kp = q->k_pad;

  PassArgs a;
  a.offsets = offsets;
  a.batch = batch;
  a.total_rows = total_rows;
  a.tiles = sa::tiles_of(total_rows);
  a.k = k;
  a.d = d;
  a.out_x = R;
  a.out_m = m;
  a.part_x = reinterpret_cast<float*>(ws + wl.part_x_off);
  a.part_m = reinterpret_cast<float*>(ws + wl.part_m_off);
  a.header = reinterpret_cast<sa::WsHeader*>(ws);
  a.user_queries = user_q ? 1 : 0;
  a.keep_flags = 0;
  const int Gr = static_cast<int>(grid_for(q, total_rows));

  if (sa::launch_bwd_prep(G, g, batch, k, kp, d, gb, gp, st) != cudaSuccess) return SA_ERR_CUDA;
  if (user_q && sa::launch_user_query(queries, q->m_f32, batch, k, kp, d, nullptr, uq, st) !=
                    cudaSuccess)
    return SA_ERR_CUDA;
  CUtensorMap tmx, tmg, tmq;
  const bool ok_maps =
      (total_rows > 0 ? make_tmap_bf16(&tmx, X, static_cast<uint64_t>(total_rows),
                                       static_cast<uint64_t>(d), sa::kTileRows)
                      : make_tmap_bf16(&tmx, q->q_bf16, static_cast<uint64_t>(kp),
                                       static_cast<uint64_t>(d), 64)) &&
      make_tmap_bf16(&tmg, gb, static_cast<uint64_t>(batch) * kp, static_cast<uint64_t>(d),
                     static_cast<uint32_t>(kp)) &&
      (!user_q || make_tmap_bf16(&tmq, uq, static_cast<uint64_t>(batch) * kp,
                                 static_cast<uint64_t>(d), static_cast<uint32_t>(kp)));
  if (!ok_maps) return SA_ERR_CUDA;
  if (sa::launch_backward(tmx, user_q ? tmq : q->tmap_q, tmg, kp, a, gp,
                          static_cast<uint16_t*>(dX), Gr, st) != cudaSuccess ||
      sa::launch_finalize(a, Gr, st) != cudaSuccess)
    return SA_ERR_CUDA;

  // Parameter gradients from R = ln 2 dL/dQ' (Q' = scale P W_Q W_K^T):
  //   dP = c R W_K W_Q^T,  dW_Q = c P^T R W_K,  dW_K = c R^T P W_Q,  c = scale log2 e,
  // summed over users for shared P, per user (dQ_b) with per-user queries.
  const double cgrad = q->scale / 0.6931471805599453;
  const int64_t kd = static_cast<int64_t>(k) * d;
  bool ok = true;
  if (!user_q) {
    ok = sa::launch_sum_users(R, batch, kd, Rs, st) == cudaSuccess &&
         sa::launch_bwd_gemm(Rs, 0, false, W_K_f32, 0, false, tmp, 0, k, d, d, 1.0, false, 1, st) ==
             cudaSuccess &&
         sa::launch_bwd_gemm(tmp, 0, false, W_Q_f32, 0, true, dP, 0, k, d, d, cgrad, false, 1, st) ==
             cudaSuccess &&
         sa::launch_bwd_gemm(P_f32, 0, true, Rs, 0, false, T, 0, d, d, k, 1.0, false, 1, st) ==
             cudaSuccess;
  } else {
    ok = sa::launch_bwd_gemm(R, kd, false, W_K_f32, 0, false, tmp, kd, k, d, d, 1.0, false, batch,
                             st) == cudaSuccess &&
         sa::launch_bwd_gemm(tmp, kd, false, W_Q_f32, 0, true, dP, kd, k, d, d, cgrad, false, batch,
                             st) == cudaSuccess &&
         sa::launch_bwd_gemm(queries, 0, true, R, 0, false, T, 0, d, d,
                             static_cast<int>(batch * k), 1.0, false, 1, st) == cudaSuccess;
  }
  ok = ok &&
       sa::launch_bwd_gemm(T, 0, false, W_K_f32, 0, false, dW_Q, 0, d, d, d, cgrad, false, 1, st) ==
           cudaSuccess &&
       sa::launch_bwd_gemm(T, 0, true, W_Q_f32, 0, false, dW_K, 0, d, d, d, cgrad, false, 1, st) ==
           cudaSuccess;
  return ok ? SA_OK : SA_ERR_CUDA;
}

sa_status sa_read_device_status(void* workspace, size_t workspace_bytes, void* stream,
                                uint32_t* flags_out) {
  if (workspace == nullptr || workspace_bytes < sa::kWsHeaderBytes) return SA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t h[2] = {0, 0};
  if (cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SA_ERR_CUDA;
  const uint32_t bits = h[0] | h[1];
  if (flags_out) *flags_out = bits;
  if (bits == 0) return SA_OK;
  if (cudaMemsetAsync(workspace, 0, sizeof(h), st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SA_ERR_CUDA;
  return SA_ERR_DEVICE_FLAG;
}

}  // extern "C"
