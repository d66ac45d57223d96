// Longest-first ordering of attention work items (tile = pair of consecutive blocks of
// one head).  Heads of one problem can differ by two orders of magnitude in kept tiles,
// so the tiles are dispatched in descending order of their list lengths (an upper bound
// of the union walked by the tile): a counting sort on the device into caller-provided
// scratch.  Ties keep no particular order; the result of every tile is independent of
// the order, so outputs stay deterministic.
#include "common.cuh"

namespace nabla {
namespace {

__global__ void sched_hist_kernel(const int32_t* __restrict__ cnt, int nb, int npairs, long long items,
                                  int32_t* __restrict__ cost_of, int32_t* __restrict__ hist) {
  const long long it = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (it >= items) return;
  const long long bh = it / npairs;
  const int p = static_cast<int>(it - bh * npairs);
  const int i0 = 2 * p;
  int c = min(max(cnt[bh * nb + i0], 0), nb);
  if (i0 + 1 < nb) c += min(max(cnt[bh * nb + i0 + 1], 0), nb);
  cost_of[it] = c;
  atomicAdd(&hist[c], 1);
}

// Exclusive scan in descending cost order: offset[c] = #items with cost > c.
__global__ void __launch_bounds__(1024) sched_scan_kernel(int32_t* __restrict__ hist, int nbins) {
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < nbins; base += 1024) {
    const int c = nbins - 1 - (base + threadIdx.x);   // descending cost
    const int v = (c >= 0) ? hist[c] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += t;
      }
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int prefix = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + incl - v;
    __syncthreads();
    if (c >= 0) hist[c] = prefix;
    if (threadIdx.x == 1023) carry = prefix + v;
    __syncthreads();
  }
}

__global__ void sched_scatter_kernel(const int32_t* __restrict__ cost_of, long long items,
                                     int32_t* __restrict__ offset, int32_t* __restrict__ order) {
  const long long it = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (it >= items) return;
  const int pos = atomicAdd(&offset[cost_of[it]], 1);
  order[pos] = static_cast<int32_t>(it);
}

}  // namespace

size_t schedule_scratch_bytes(const Dims& d) {
  const size_t items = static_cast<size_t>(d.BH) * ((d.nb + 1) / 2);
  const size_t nbins = 2 * static_cast<size_t>(d.nb) + 1;
  return align_up(items * 4, 256) * 2 + align_up(nbins * 4, 256);
}

// Writes the item order (descending cost) to the start of `scratch`; returns it.
cudaError_t build_schedule(const int32_t* cnt, const Dims& d, void* scratch, int32_t** order_out,
                           cudaStream_t st) {
  const long long npairs = (d.nb + 1) / 2;
  const long long items = static_cast<long long>(d.BH) * npairs;
  const int nbins = 2 * d.nb + 1;
  char* base = static_cast<char*>(scratch);
  int32_t* order = reinterpret_cast<int32_t*>(base);
  int32_t* cost_of = reinterpret_cast<int32_t*>(base + align_up(items * 4, 256));
  int32_t* hist = reinterpret_cast<int32_t*>(base + 2 * align_up(items * 4, 256));
  cudaError_t e = cudaMemsetAsync(hist, 0, static_cast<size_t>(nbins) * 4, st);
  if (e != cudaSuccess) return e;
  const unsigned blocks = static_cast<unsigned>((items + 255) / 256);
  sched_hist_kernel<<<blocks, 256, 0, st>>>(cnt, d.nb, static_cast<int>(npairs), items, cost_of, hist);
  sched_scan_kernel<<<1, 1024, 0, st>>>(hist, nbins);
  sched_scatter_kernel<<<blocks, 256, 0, st>>>(cost_of, items, hist, order);
  *order_out = order;
  return cudaGetLastError();
}

}  // namespace nabla
