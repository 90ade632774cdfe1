// sa_sketch_forward_noalloc: sa_sketch_forward for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocator) at the point where
// they run the SA layer.  Examples are code inside a custom allocator's own
// hooks, code running under a memory pool that must not grow, and hosts that
// hand the library only fixed, pre-registered buffers.  This entry point
// takes the same inputs and outputs as sa_sketch_forward.  In place of a
// caller-provided workspace it uses a fixed scratch array that lives in this
// library's device image.
//
// When the array is reserved.  The array sits in the module built from this
// file.  With CUDA's default lazy module loading, that module is loaded on a
// device, and the array reserved there, at the first call that needs it:
// the address lookup of the first call on the device.  A call with batch = 0
// does that set-up and nothing else, so a caller can make it at start-up,
// while allocating is still allowed.  From then on the array stays reserved
// on that device until the process exits (or the device is reset), and no
// call allocates.
//
// The array's name is a host-side stand-in, not a device address.  Host code
// must look the address up with cudaGetSymbolAddress, with the device
// current, once per device and context.  That lookup is the set-up below.
#include <mutex>

#include <cuda.h>

#include "sa.h"

namespace {

// Scratch for the partial sketches of users that cross CTA row ranges, plus
// the device-flag header.  32 MiB covers every query with k * d <= 128 * 128
// (and d = 256 with k <= 64) on a GPU with up to 148 SMs.
constexpr size_t kNoAllocScratchBytes = size_t{32} << 20;

static __device__ __align__(256) unsigned char sa_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
// Per device: the scratch address and the context it was looked up in.  A
// device reset (cudaDeviceReset) destroys the context and unloads the
// module; the next call on that device runs in a new context, which has a
// new ID, and looks the address up again.
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique ID of the context current on this thread (0 if none, or if the
// driver does not offer the query).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Address of the scratch array on the current device, looked up once per
// device and context, or nullptr with *err set if the lookup failed.
void* scratch_on_current_device(cudaError_t* err) {
  int dev = -1;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  const unsigned long long ctx = current_context_id();
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, sa_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
    // The lookup makes the runtime's context current if none was.
    g_scratch_ctx[dev] = ctx != 0 ? ctx : current_context_id();
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

sa_status sa_sketch_forward_noalloc(sa_query q, const void* X, const int64_t* offsets,
                                    int64_t batch, int64_t total_rows, float* X_tilde,
                                    float* mass, uint32_t* device_flags_out, void* stream) {
  if (q == nullptr || batch < 0 || total_rows < 0) return SA_ERR_INVALID_ARG;
  const size_t need = sa_workspace_bytes(q, batch, total_rows);
  if (need == 0 || need > kNoAllocScratchBytes) return SA_ERR_WORKSPACE;
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_on_current_device(&err);
  if (scratch == nullptr) return SA_ERR_CUDA;
  // The array keeps the previous call's contents.  What has to start at zero
  // is the flag header, and the first kernel of every call clears it; the
  // partial slots are always written before they are read.
  sa_status s = sa_sketch_forward(q, X, offsets, batch, total_rows, X_tilde, mass, scratch,
                                  kNoAllocScratchBytes, stream);
  if (s != SA_OK) return s;
  if (device_flags_out != nullptr) {
    // Header words 0 and 1: this call's offset-validation and timeout flags.
    // A call with batch == 0 launches no kernel, so its flags are zero.
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e =
        batch == 0 ? cudaMemsetAsync(device_flags_out, 0, 2 * sizeof(uint32_t), st)
                   : cudaMemcpyAsync(device_flags_out, scratch, 2 * sizeof(uint32_t),
                                     cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return SA_ERR_CUDA;
  }
  return SA_OK;
}

}  // extern "C"
