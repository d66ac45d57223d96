// Allocation-free variant of nabla_attn_fwd.
//
// Some callers cannot call cudaMalloc at the point where they run attention: a host
// framework that owns all device memory through its own pool and forbids driver
// allocations on its hot path (cudaMalloc can synchronise the device and would bypass
// the pool's budget), or a latency-critical loop that must not pay for an allocation.
// They still own their inputs and outputs; what they cannot provide is the forward's
// workspace (the device status word and the longest-first tile schedule).  This entry
// point takes that workspace from a fixed array in the library's own device memory.
//
// The array below is a file-scope __device__ array of kNoAllocScratchBytes (1 MiB).
// Every GPU that loads the library holds it until the process exits.  In host code the
// symbol `g_noalloc_scratch` is only a host-side stand-in, never a device address: its
// device address is looked up once per device with cudaGetSymbolAddress (with that
// device current; again if the device's context was re-created, e.g. by cudaDeviceReset)
// and passed to the kernels as an ordinary pointer.
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;   // 1 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Per device: the device address of the array and the unique id of the context it was
// looked up in.  A device reset (cudaDeviceReset) or a re-created primary context gives
// the device a new context id, and the address is then looked up again.
struct DeviceScratch {
  unsigned long long ctx_id;
  void* addr;
};

std::mutex g_setup_mutex;
DeviceScratch g_scratch[kMaxDevices] = {};
PFN_cuCtxGetCurrent_v4000 g_ctx_get_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_get_id = nullptr;

// Unique id of the calling thread's current context (0 when there is none yet).  Called
// with g_setup_mutex held.
bool current_context_id(unsigned long long* id) {
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) {
    void* p = nullptr;
    void* q = nullptr;
    cudaDriverEntryPointQueryResult r1, r2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r1) != cudaSuccess ||
        r1 != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &q, cudaEnableDefault, &r2) != cudaSuccess ||
        r2 != cudaDriverEntryPointSuccess)
      return false;
    g_ctx_get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    g_ctx_get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(q);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return false;
  *id = 0;
  if (ctx == nullptr) return true;
  return g_ctx_get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on the current device.  The set-up (the address
// lookup, with the device current) runs on the first call on a device and again only
// if the device's context has changed since.
nabla_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return NABLA_ERR_CUDA;
  if (dev >= kMaxDevices) return NABLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  unsigned long long id = 0;
  if (!current_context_id(&id)) return NABLA_ERR_CUDA;
  DeviceScratch& ds = g_scratch[dev];
  if (ds.addr == nullptr || id == 0 || ds.ctx_id != id) {
    void* p = nullptr;
    // the lookup also makes the device's primary context current if it was not yet
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return NABLA_ERR_CUDA;
    if (!current_context_id(&id) || id == 0) return NABLA_ERR_CUDA;
    ds.ctx_id = id;
    ds.addr = p;
  }
  *out = ds.addr;
  return NABLA_OK;
}

}  // namespace

extern "C" nabla_status nabla_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                               nabla_dtype v_dtype, const uint32_t* mask_bits,
                                               nabla_shape s, float scale, void* o,
                                               nabla_dtype o_dtype, float* lse,
                                               nabla_layout layout, nabla_stream_t stream) {
  nabla::Dims d;
  nabla_status rc = nabla::check_shape(s, &d);
  if (rc != NABLA_OK) return rc;
  // The problem's workspace must fit the fixed array; larger problems are rejected
  // before anything is enqueued.
  if (nabla_fwd_workspace_bytes(s) > kNoAllocScratchBytes) return NABLA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  rc = scratch_for_current_device(&scratch);
  if (rc != NABLA_OK) return rc;
  // The regular entry point clears the status word before its kernels run, and the
  // schedule kernels overwrite every scratch word that the attention kernel later reads,
  // so nothing left in the array by an earlier call is read.
  return nabla_attn_fwd(q, k, v, v_dtype, mask_bits, s, scale, o, o_dtype, lse, layout, scratch,
                        kNoAllocScratchBytes, stream);
}

extern "C" nabla_status nabla_attn_fwd_noalloc_status(uint32_t* code, nabla_stream_t stream) {
  void* scratch = nullptr;
  const nabla_status rc = scratch_for_current_device(&scratch);
  if (rc != NABLA_OK) return rc;
  return nabla_read_device_status(scratch, code, stream);
}
