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
// device current) and passed to the kernels as an ordinary pointer.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;   // 1 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use).
nabla_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return NABLA_ERR_CUDA;
  if (dev >= kMaxDevices) return NABLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return NABLA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
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
  // The regular entry point clears the status word and the schedule histogram in the
  // scratch before its kernels run, so nothing left by an earlier call is read.
  return nabla_attn_fwd(q, k, v, v_dtype, mask_bits, s, scale, o, o_dtype, lse, layout, scratch,
                        kNoAllocScratchBytes, stream);
}
