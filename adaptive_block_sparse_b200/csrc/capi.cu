// Host-side argument checks and status helpers shared by every C-ABI entry point.
#include <stdio.h>

#include "common.cuh"

namespace nabla {

nabla_status check_shape(const nabla_shape& s, Dims* d) {
  if (s.B < 1 || s.H < 1 || s.T < 1 || s.Hg < 1 || s.W < 1 || s.D < 1 || s.P < 1)
    return NABLA_ERR_INVALID_ARG;
  if (s.P != 8) return NABLA_ERR_UNSUPPORTED;
  if (s.Hg % s.P || s.W % s.P) return NABLA_ERR_INVALID_ARG;
  if (s.D != 64 && s.D != 128) return NABLA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(s.B) * s.H;
  const long long S = static_cast<long long>(s.T) * s.Hg * s.W;
  const long long nb = S / (s.P * s.P);
  if (BH > 65535 || nb > 16384) return NABLA_ERR_UNSUPPORTED;
  d->B = s.B; d->H = s.H; d->T = s.T; d->Hg = s.Hg; d->W = s.W; d->D = s.D; d->P = s.P;
  d->Hb = s.Hg / s.P;
  d->Wb = s.W / s.P;
  d->N = s.P * s.P;
  d->nb = static_cast<int>(nb);
  d->nw = static_cast<int>((nb + 31) / 32);
  d->BH = static_cast<int>(BH);
  d->S = S;
  return NABLA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

nabla_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NABLA_OK : NABLA_ERR_CUDA; }

}  // namespace nabla

using namespace nabla;

extern "C" const char* nabla_status_string(nabla_status s) {
  switch (s) {
    case NABLA_OK: return "NABLA_OK";
    case NABLA_ERR_INVALID_ARG: return "NABLA_ERR_INVALID_ARG";
    case NABLA_ERR_UNSUPPORTED: return "NABLA_ERR_UNSUPPORTED";
    case NABLA_ERR_WORKSPACE: return "NABLA_ERR_WORKSPACE";
    case NABLA_ERR_CUDA: return "NABLA_ERR_CUDA";
    case NABLA_ERR_DEVICE_CHECK: return "NABLA_ERR_DEVICE_CHECK";
  }
  return "NABLA_ERR_UNKNOWN";
}

extern "C" nabla_status nabla_read_device_status(void* workspace, uint32_t* code,
                                                 nabla_stream_t stream) {
  if (!workspace) return NABLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return NABLA_ERR_CUDA;
  if (code) *code = word;
  if (word != 0) {
    e = cudaMemsetAsync(workspace, 0, sizeof(word), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return NABLA_ERR_CUDA;
    return NABLA_ERR_DEVICE_CHECK;
  }
  return NABLA_OK;
}

namespace {

// One warp waits, through the bounded wait every kernel uses, for a barrier phase that
// nothing completes (the barrier expects one arrival and none is made): the wait gives up
// after its time limit, records kDevTimeoutSelftest and the kernel returns normally.
__global__ void __launch_bounds__(32) selftest_bounded_wait_kernel(uint32_t* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncwarp();
  const bool done = __all_sync(0xffffffffu, mbar_wait(&bar, 0, status, kDevTimeoutSelftest));
  if (done && threadIdx.x == 0) record_status(status, kDevSelftestUnexpected);
}

}  // namespace

extern "C" nabla_status nabla_selftest_bounded_wait(void* workspace, size_t workspace_bytes,
                                                    nabla_stream_t stream) {
  if (!workspace || workspace_bytes < kStatusBytes || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return NABLA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_status(e);
  selftest_bounded_wait_kernel<<<1, 32, 0, st>>>(static_cast<uint32_t*>(workspace));
  return cuda_status(cudaGetLastError());
}
