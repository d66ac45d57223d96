// Fractal-flatten token reorder and block mean pooling (HBM-bound).
//
// "NABLA: Neighborhood Adaptive Block-Level Attention" (gist.science, Chinese edition),
// technical summary, Methodology: "token reordering (fractal flatten)" groups the tokens
// of every P x P spatial patch into one contiguous run with frames kept in order, and
// "adaptive mask construction / downsampling" average-pools Q and K per block.
//
// One CTA moves one block of N = 64 tokens of one (b, h): 64 rows of D bf16.  In
// natural order a patch row (8 tokens of one image row) is one contiguous run of
// 8 * D * 2 bytes, so every warp issues 16-byte loads over 512-byte contiguous spans;
// the reordered block is one contiguous 64 * D * 2-byte run.  The optional pool sums
// the block's 64 rows column by column in fp64, in token order (exact for bf16), and
// divides by 64.  When no copy is written (the pool alone), pool_only_kernel skips the
// shared-memory staging: each lane reads one 16-byte column chunk of its block's tokens
// and keeps the eight column sums itself, in the same order.
#include "common.cuh"

namespace nabla {

namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  const __half2 h = __floats2half2_rn(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// GATHER: the source is in natural order (forward reorder); otherwise the source block
// is contiguous (already reordered).  SCATTER: the destination is natural order
// (inverse reorder).  WRITE: write a destination at all.  POOL: emit fp64 block means of
// the (bf16) source.  TO_F16: convert bf16 -> fp16 on the way.  ESZ: element bytes.
template <int D, int ESZ, bool GATHER, bool SCATTER, bool WRITE, bool POOL, bool TO_F16>
__global__ void __launch_bounds__(kThreads) reorder_pool_kernel(
    const uint4* __restrict__ src, uint4* __restrict__ dst, double* __restrict__ pool_out,
    int Hg, int W, int Hb, int Wb, int nb) {
  constexpr int V = D * ESZ / 16;     // uint4 chunks per token row
  constexpr int kChunks = 64 * V;     // per block
  constexpr int kPer = kChunks / kThreads;
  __shared__ __align__(16) uint4 tile[POOL ? kChunks : 1];

  const int blk = blockIdx.x;
  const long long bh = blockIdx.y;
  const long long S = static_cast<long long>(nb) * 64;
  const int t = blk / (Hb * Wb);
  const int rem = blk - t * (Hb * Wb);
  const int hb = rem / Wb;
  const int wb = rem - hb * Wb;
  const long long head_base = bh * S;   // in tokens

#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int e = threadIdx.x + u * kThreads;
    const int tt = e / V;
    const int c = e - tt * V;
    const long long nat =
        (static_cast<long long>(t) * Hg + hb * 8 + (tt >> 3)) * W + wb * 8 + (tt & 7);
    const long long frac = static_cast<long long>(blk) * 64 + tt;
    const long long s_tok = GATHER ? nat : frac;
    const uint4 val = __ldg(src + (head_base + s_tok) * V + c);
    if constexpr (WRITE) {
      const long long d_tok = SCATTER ? nat : frac;
      uint4 out = val;
      if constexpr (TO_F16) {
        out.x = bf16x2_to_f16x2(val.x);
        out.y = bf16x2_to_f16x2(val.y);
        out.z = bf16x2_to_f16x2(val.z);
        out.w = bf16x2_to_f16x2(val.w);
      }
      dst[(head_base + d_tok) * V + c] = out;
    }
    if constexpr (POOL) tile[e] = val;
  }
  if constexpr (POOL) {
    __syncthreads();
    if (threadIdx.x < D) {
      const __nv_bfloat16* tb = reinterpret_cast<const __nv_bfloat16*>(tile);
      double acc = 0.0;
#pragma unroll 8
      for (int tt = 0; tt < 64; ++tt) acc += static_cast<double>(__bfloat162float(tb[tt * D + threadIdx.x]));
      pool_out[(bh * nb + blk) * D + threadIdx.x] = acc / 64.0;
    }
  }
}

// Pool only (no copy written): lane l of a warp owns the 16-byte column chunk c = l % C
// (C = D / 8 chunks, 8 columns each) of block (l / C) of the warp's 32 / C blocks, reads
// that chunk of the block's 64 tokens straight from memory (the C lanes of a block read
// one token's whole row: 2 x 256-byte runs per load at D = 128) and keeps eight fp64
// sums, each over its column in token order: the same sums, in the same order, as the
// copy-and-pool kernel's, without staging through shared memory.
template <int D, bool GATHER>
__global__ void __launch_bounds__(kThreads) pool_only_kernel(
    const uint4* __restrict__ src, double* __restrict__ pool_out, int Hg, int W, int Hb, int Wb,
    int nb, long long n_blocks) {
  constexpr int C = D / 8;                 // 16-byte chunks per token row
  constexpr int BPW = 32 / C;              // blocks per warp
  const int lane = threadIdx.x & 31;
  const int c = lane % C;
  const long long g = (static_cast<long long>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5)) * BPW + lane / C;
  if (g >= n_blocks) return;               // whole block groups of lanes leave together
  const long long bh = g / nb;
  const int blk = static_cast<int>(g - bh * nb);
  const long long S = static_cast<long long>(nb) * 64;
  const int t = blk / (Hb * Wb);
  const int rem = blk - t * (Hb * Wb);
  const int hb = rem / Wb;
  const int wb = rem - hb * Wb;
  const uint4* base = src + bh * S * C + c;
  double acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.0;
#pragma unroll 2
  for (int r = 0; r < 8; ++r) {            // patch row r: tokens 8 r .. 8 r + 7 of the block
    const long long tok0 = GATHER ? (static_cast<long long>(t) * Hg + hb * 8 + r) * W + wb * 8
                                  : static_cast<long long>(blk) * 64 + 8 * r;
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(base + (tok0 + u) * C);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[2 * k] += static_cast<double>(__uint_as_float(w[k] << 16));
        acc[2 * k + 1] += static_cast<double>(__uint_as_float(w[k] & 0xFFFF0000u));
      }
    }
  }
  double* out = pool_out + g * D + c * 8;   // 8-byte stores: the pool may be 8-byte aligned
#pragma unroll
  for (int k = 0; k < 8; ++k) out[k] = acc[k] / 64.0;
}

template <int D, bool GATHER>
cudaError_t go_pool(const void* src, double* pool, const Dims& d, cudaStream_t st) {
  const long long n_blocks = static_cast<long long>(d.BH) * d.nb;
  constexpr int kBlocksPerCta = (kThreads / 32) * (32 / (D / 8));
  const long long grid = (n_blocks + kBlocksPerCta - 1) / kBlocksPerCta;
  pool_only_kernel<D, GATHER><<<static_cast<unsigned>(grid), kThreads, 0, st>>>(
      static_cast<const uint4*>(src), pool, d.Hg, d.W, d.Hb, d.Wb, d.nb, n_blocks);
  return cudaGetLastError();
}

template <int D, int ESZ, bool GATHER, bool SCATTER, bool WRITE, bool POOL, bool TO_F16>
cudaError_t go(const void* src, void* dst, double* pool, const Dims& d, cudaStream_t st) {
  dim3 grid(d.nb, d.BH);
  reorder_pool_kernel<D, ESZ, GATHER, SCATTER, WRITE, POOL, TO_F16><<<grid, kThreads, 0, st>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), pool, d.Hg, d.W, d.Hb, d.Wb, d.nb);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_reorder(const void* src, void* dst, double* pool, const Dims& d, int inverse,
                           int esz, bool to_f16, cudaStream_t st) {
  if (inverse == 2) {   // natural order kept: the dtype conversion alone (+ the pools)
    if (to_f16)
      return pool ? go<D, 2, true, true, true, true, true>(src, dst, pool, d, st)
                  : go<D, 2, true, true, true, false, true>(src, dst, nullptr, d, st);
    return pool ? go<D, 2, true, true, true, true, false>(src, dst, pool, d, st)
                : go<D, 2, true, true, true, false, false>(src, dst, nullptr, d, st);
  }
  if (inverse) {
    return esz == 4 ? go<D, 4, false, true, true, false, false>(src, dst, nullptr, d, st)
                    : go<D, 2, false, true, true, false, false>(src, dst, nullptr, d, st);
  }
  if (dst == nullptr)   // pool only: the fp64 block means of a natural-order tensor
    return go_pool<D, true>(src, pool, d, st);
  if (to_f16) {
    return pool ? go<D, 2, true, false, true, true, true>(src, dst, pool, d, st)
                : go<D, 2, true, false, true, false, true>(src, dst, nullptr, d, st);
  }
  return pool ? go<D, 2, true, false, true, true, false>(src, dst, pool, d, st)
              : go<D, 2, true, false, true, false, false>(src, dst, nullptr, d, st);
}

}  // namespace

// Pools a bf16 tensor (reordered, or in the natural order) into fp64 block means (used by
// the mask build).
cudaError_t pool_blocks_device(const void* x, double* pool, const Dims& d, cudaStream_t st, bool natural) {
  if (natural) return d.D == 64 ? go_pool<64, true>(x, pool, d, st) : go_pool<128, true>(x, pool, d, st);
  return d.D == 64 ? go_pool<64, false>(x, pool, d, st) : go_pool<128, false>(x, pool, d, st);
}

}  // namespace nabla

using namespace nabla;

extern "C" nabla_status nabla_reorder(const void* src, nabla_dtype src_dtype, void* dst,
                                      nabla_dtype dst_dtype, double* pool_out, nabla_shape s,
                                      int32_t inverse, nabla_stream_t stream) {
  Dims d;
  nabla_status rc = check_shape(s, &d);
  if (rc != NABLA_OK) return rc;
  // inverse: 0 natural -> reordered, 1 reordered -> natural, 2 natural -> natural (the
  // conversion alone).  dst may be NULL for the pool alone (direction 0, pool_out given).
  if (inverse < 0 || inverse > 2) return NABLA_ERR_INVALID_ARG;
  if (!src || (!dst && (inverse || !pool_out))) return NABLA_ERR_INVALID_ARG;
  if (!aligned16(src) || (dst && !aligned16(dst))) return NABLA_ERR_INVALID_ARG;
  const bool dt_ok = inverse == 1 ? (src_dtype == dst_dtype &&
                                     (src_dtype == NABLA_BF16 || src_dtype == NABLA_F16 || src_dtype == NABLA_F32))
                                  : (src_dtype == NABLA_BF16 && (dst_dtype == NABLA_BF16 || dst_dtype == NABLA_F16));
  if (!dt_ok) return NABLA_ERR_INVALID_ARG;
  if (pool_out && (inverse == 1 || (reinterpret_cast<uintptr_t>(pool_out) & 7))) return NABLA_ERR_INVALID_ARG;
  const int esz = src_dtype == NABLA_F32 ? 4 : 2;
  const size_t bytes = static_cast<size_t>(d.BH) * d.S * d.D * esz;
  const char* a = static_cast<const char*>(src);
  const char* b = static_cast<const char*>(dst);
  if (b && a < b + bytes && b < a + bytes) return NABLA_ERR_INVALID_ARG;   // overlap
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool to_f16 = inverse != 1 && dst_dtype == NABLA_F16;
  cudaError_t e = d.D == 64 ? launch_reorder<64>(src, dst, pool_out, d, inverse, esz, to_f16, st)
                            : launch_reorder<128>(src, dst, pool_out, d, inverse, esz, to_f16, st);
  return cuda_status(e);
}
