// Order of attention work items (tile = two query blocks of one head: blocks 2p and 2p+1,
// or with frame pairs the two blocks of tile_blocks()).
//
// Heads are taken one after another (head-major), so the tiles running at the same time
// read K and V of one or two heads and those stay resident in L2.  Inside a head, tiles
// run longest first (descending length of their two kept lists, an upper bound of the
// union a tile walks).  The heads themselves run in descending order of their longest
// tile: the kept-block counts differ by two orders of magnitude between heads (a head
// with flat pooled scores keeps hundreds of blocks per row, a peaked one a handful), and
// a long tile that starts late would leave the other SMs idle at the end.  Two launches:
// one CTA per head sorts the head's tiles with a bitonic sort on (length descending,
// tile index ascending) and records the head's longest tile; then one CTA per head finds
// the head's rank (longest tile descending, head index ascending) and copies its tiles
// to that position.  The order is fully deterministic, and every tile's result is
// independent of the order anyway.
#include "common.cuh"

namespace nabla {
namespace {

// Tile length: with `bits` the exact union size popc(row a | row b); otherwise the sum of
// the two list counts.
__global__ void __launch_bounds__(512) sched_head_sort_kernel(const int32_t* __restrict__ cnt,
                                                              const uint32_t* __restrict__ bits,
                                                              int nb, int nw, int npairs, int npow2,
                                                              int T, int HW, int frame_pairs, int vec4,
                                                              int32_t* __restrict__ sorted,
                                                              int32_t* __restrict__ head_len) {
  extern __shared__ unsigned long long keys[];
  const long long bh = blockIdx.x;
  for (int e = threadIdx.x; e < npow2; e += blockDim.x) {
    unsigned long long key = ~0ull;
    if (e < npairs) {
      int i0 = 2 * e, i1 = i0 + 1 < nb ? i0 + 1 : -1;
      if (frame_pairs) {
        const int2 ab = tile_blocks(e, T, HW, nb);
        i0 = ab.x;
        i1 = ab.y;
      }
      int c = 0;
      if (bits != nullptr) {
        const uint32_t* r0 = bits + (bh * nb + i0) * static_cast<long long>(nw);
        const uint32_t* r1 = i1 >= 0 ? bits + (bh * nb + i1) * static_cast<long long>(nw) : nullptr;
        const uint32_t tail = (nb & 31) ? (1u << (nb & 31)) - 1u : ~0u;
        if (vec4) {
          // rows of whole 16-byte words: eight of them (both rows) in flight at a time
          const uint4* a4 = reinterpret_cast<const uint4*>(r0);
          const uint4* b4 = reinterpret_cast<const uint4*>(r1);
          const int n4 = nw >> 2;
          for (int w4 = 0; w4 < n4; w4 += 8) {
            uint4 xa[8], xb[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              xa[i] = w4 + i < n4 ? __ldg(a4 + w4 + i) : make_uint4(0u, 0u, 0u, 0u);
              xb[i] = (r1 != nullptr && w4 + i < n4) ? __ldg(b4 + w4 + i) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t last = w4 + i == n4 - 1 ? tail : ~0u;   // word nw - 1 is the .w part
              c += __popc(xa[i].x | xb[i].x) + __popc(xa[i].y | xb[i].y) + __popc(xa[i].z | xb[i].z) +
                   __popc((xa[i].w | xb[i].w) & last);
            }
          }
        } else {
          for (int w = 0; w < nw; ++w) {
            uint32_t u = r0[w] | (r1 ? r1[w] : 0u);
            if (w == nw - 1) u &= tail;
            c += __popc(u);
          }
        }
      } else {
        c = min(max(cnt[bh * nb + i0], 0), nb);
        if (i1 >= 0) c += min(max(cnt[bh * nb + i1], 0), nb);
      }
      key = (static_cast<unsigned long long>(0x7FFFFFFF - c) << 32) | static_cast<unsigned>(e);
    }
    keys[e] = key;
  }
  __syncthreads();
  for (int k = 2; k <= npow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int e = threadIdx.x; e < npow2; e += blockDim.x) {
        const int p = e ^ j;
        if (p > e) {
          const unsigned long long a = keys[e], b = keys[p];
          const bool up = (e & k) == 0;
          if ((a > b) == up) {
            keys[e] = b;
            keys[p] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int e = threadIdx.x; e < npairs; e += blockDim.x)
    sorted[bh * npairs + e] = static_cast<int32_t>(bh * npairs + static_cast<long long>(keys[e] & 0xFFFFFFFFull));
  if (threadIdx.x == 0) head_len[bh] = npairs > 0 ? 0x7FFFFFFF - static_cast<int>(keys[0] >> 32) : 0;
}

// Places head bh's sorted tiles at its rank among the heads: longest tile descending,
// head index ascending.
__global__ void __launch_bounds__(256) sched_head_place_kernel(const int32_t* __restrict__ sorted,
                                                               const int32_t* __restrict__ head_len,
                                                               int BH, int npairs,
                                                               int32_t* __restrict__ order) {
  __shared__ int part[8];
  const int bh = blockIdx.x;
  const int mine = head_len[bh];
  int before = 0;
  for (int h = threadIdx.x; h < BH; h += blockDim.x) {
    const int len = head_len[h];
    before += (len > mine || (len == mine && h < bh)) ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = before;
  __syncthreads();
  int rank = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) rank += part[w];
  const long long src = static_cast<long long>(bh) * npairs;
  const long long dst = static_cast<long long>(rank) * npairs;
  for (int e = threadIdx.x; e < npairs; e += blockDim.x) order[dst + e] = sorted[src + e];
}

int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

}  // namespace

size_t schedule_scratch_bytes(const Dims& d) {
  const size_t items = static_cast<size_t>(d.BH) * ((d.nb + 1) / 2);
  // the order, the per-head sorted tiles, the per-head longest tile
  return 2 * align_up(items * 4, 256) + align_up(static_cast<size_t>(d.BH) * 4, 256);
}

// Writes the item order to the start of `scratch`; returns it.  Tile lengths from the
// bitmask when `bits` is given, else from the list counts `cnt`.
cudaError_t build_schedule(const int32_t* cnt, const uint32_t* bits, const Dims& d, void* scratch,
                           int32_t** order_out, cudaStream_t st, bool frame_pairs) {
  const int npairs = (d.nb + 1) / 2;
  const int npow2 = next_pow2(npairs);
  const size_t items_bytes = align_up(static_cast<size_t>(d.BH) * npairs * 4, 256);
  int32_t* order = static_cast<int32_t*>(scratch);
  int32_t* sorted = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) + items_bytes);
  int32_t* head_len = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) + 2 * items_bytes);
  const size_t smem = static_cast<size_t>(npow2) * 8;
  cudaError_t e = cudaFuncSetAttribute(sched_head_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // 16-byte loads of the bitmask rows when every row starts on a 16-byte boundary
  const int vec4 = bits != nullptr && (d.nw & 3) == 0 && (reinterpret_cast<uintptr_t>(bits) & 15) == 0;
  sched_head_sort_kernel<<<d.BH, 512, smem, st>>>(cnt, bits, d.nb, d.nw, npairs, npow2, d.T,
                                                   d.Hb * d.Wb, frame_pairs ? 1 : 0, vec4, sorted, head_len);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sched_head_place_kernel<<<d.BH, 256, 0, st>>>(sorted, head_len, d.BH, npairs, order);
  *order_out = order;
  return cudaGetLastError();
}

}  // namespace nabla
