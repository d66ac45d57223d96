// Fast tier of the adaptive mask build: pooled logits on the tensor cores, then a
// per-row CDF cut in fp32 with a certified error margin.
//
// "NABLA: Neighborhood Adaptive Block-Level Attention" (gist.science, Chinese edition),
// technical summary, Methodology, "reduced attention" + "CDF thresholding": full
// attention on the pooled map, row softmax, keep the blocks whose cumulative
// probability exceeds 1 - thr.
//
// The decision of the method is defined in exact arithmetic (and checked against fp64).
// Computing it in fp64 on CUDA cores is slow, so this tier decides every row whose cut
// is unambiguous at a proven error bound, and hands the others to the fp64 kernel:
//
//  1. pool_split_kernel (from the bf16 tokens: the fp64 block means, written out for the
//     fp64 tier, in the same pass) or split_pools_kernel (from given means): the means
//     q, k are split into fp16 pairs q = q_hi + q_lo + r (|r| <= 2^-22 |q|), padded to a
//     multiple of 256 rows; row norms |q_i| and the per-head maximum |k_j| are kept for
//     the error bound.
//  2. pooled_logits_kernel: A = scale * (q_hi k_hi^T + (q_hi k_lo^T + q_lo k_hi^T)) with
//     tcgen05 (M = 128, N = 128, K = 16 per instruction, fp32 accumulate in TMEM; the
//     dominant q_hi k_hi^T term has its own accumulator), written to an fp32 scratch by
//     a persistent kernel that overlaps the key tiles' copies, the MMAs and the stores.
//  3. mask_select_kernel: one warp per row: softmax in fp32; the cut value P_c (the
//     smallest kept probability) from a bracket of fp32 bit patterns where the mass at
//     or above crosses thr -- first guess one sixteenth of the row maximum, else a lower
//     end from mass(P >= x) >= 1 - nb x and probes interpolated in the key -- narrowed
//     until it holds at most 16 blocks, which are then ranked and walked; then the
//     certificate: with rho the proven relative error of every P_j,
//        thr - E_above > eta,  E_at_or_above - thr > eta,  P_c unique,
//        P_c - P_next > 2 rho P_c,
//     where eta = rho + 3e-6 bounds the error of the ranked masses.  A certified row
//     keeps exactly the blocks with P_j >= P_c (the same set the exact ranking keeps);
//     the others are appended to a per-head list that the fp64 kernel recomputes.
#include <math.h>

#include <type_traits>

#include <cudaTypedefs.h>

#include "common.cuh"

namespace nabla {

bool make_map_16(CUtensorMap* map, const void* base, long long rows, int D, int box_rows,
                 bool fp16);
bool make_map_f32(CUtensorMap* map, const void* base, long long rows, int D);

namespace {

// Per-logit error bound, relative to scale * |q_i| * max_j |k_j|: split residuals
// (3 x 2^-22), eight fp32 accumulations of the leading product (8 x 2^-22, allowing
// truncating adds), the correction products and the final add / scale (~2^-22).
constexpr float kLogitErr = 4.0e-6f;
constexpr int kSelCand = 16;   // the cut's search stops at this many candidates

// ------------------------------------------------------------------------------------
// 1. fp16 split of the pooled means + norms
// ------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) split_pools_kernel(
    const double* __restrict__ qpool, const double* __restrict__ kpool, int nb, int nbp,
    long long rows_pad, __half* __restrict__ qh, __half* __restrict__ ql, __half* __restrict__ kh,
    __half* __restrict__ kl, float* __restrict__ qnorm, uint32_t* __restrict__ kmax_bits,
    int vec16) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);   // padded
  const int lane = threadIdx.x & 31;
  if (row >= rows_pad) return;
  const long long bh = row / nbp;
  const int i = static_cast<int>(row - bh * nbp);
  const bool valid = i < nb;
  // lane l takes the E = D / 32 consecutive columns from l * E: 16-byte loads of the
  // fp64 means (8-byte loads when a pool base is only 8-byte aligned) and one 8- (or 4-)
  // byte store per split tensor
  constexpr int E = D / 32;
  static_assert(E == 2 || E == 4, "D must be 64 or 128");
  double q[E], k[E];
  if (valid && !vec16) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      q[e] = qpool[(bh * nb + i) * D + lane * E + e];
      k[e] = kpool[(bh * nb + i) * D + lane * E + e];
    }
  } else if (valid) {
    const double2* q2 = reinterpret_cast<const double2*>(qpool + (bh * nb + i) * D + lane * E);
    const double2* k2 = reinterpret_cast<const double2*>(kpool + (bh * nb + i) * D + lane * E);
#pragma unroll
    for (int e = 0; e < E / 2; ++e) {
      const double2 a = q2[e], b = k2[e];
      q[2 * e] = a.x;
      q[2 * e + 1] = a.y;
      k[2 * e] = b.x;
      k[2 * e + 1] = b.y;
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) q[e] = k[e] = 0.0;
  }
  double nq = 0.0, nk = 0.0;
  __half qh1[E], ql1[E], kh1[E], kl1[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qh1[e] = __double2half(q[e]);
    kh1[e] = __double2half(k[e]);
    ql1[e] = __double2half(q[e] - static_cast<double>(__half2float(qh1[e])));
    kl1[e] = __double2half(k[e] - static_cast<double>(__half2float(kh1[e])));
    nq = fma(q[e], q[e], nq);
    nk = fma(k[e], k[e], nk);
  }
  const long long off = row * D + lane * E;
  if constexpr (E == 4) {
    *reinterpret_cast<uint2*>(qh + off) = *reinterpret_cast<const uint2*>(qh1);
    *reinterpret_cast<uint2*>(ql + off) = *reinterpret_cast<const uint2*>(ql1);
    *reinterpret_cast<uint2*>(kh + off) = *reinterpret_cast<const uint2*>(kh1);
    *reinterpret_cast<uint2*>(kl + off) = *reinterpret_cast<const uint2*>(kl1);
  } else {
    *reinterpret_cast<uint32_t*>(qh + off) = *reinterpret_cast<const uint32_t*>(qh1);
    *reinterpret_cast<uint32_t*>(ql + off) = *reinterpret_cast<const uint32_t*>(ql1);
    *reinterpret_cast<uint32_t*>(kh + off) = *reinterpret_cast<const uint32_t*>(kh1);
    *reinterpret_cast<uint32_t*>(kl + off) = *reinterpret_cast<const uint32_t*>(kl1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nq += __shfl_xor_sync(0xffffffffu, nq, o);
    nk += __shfl_xor_sync(0xffffffffu, nk, o);
  }
  if (lane == 0 && valid) {
    qnorm[bh * nb + i] = static_cast<float>(sqrt(nq)) * 1.0000001f;
    atomicMax(&kmax_bits[bh], __float_as_uint(static_cast<float>(sqrt(nk)) * 1.0000001f));
  }
}

// 1'. the same from the tokens: block means of bf16 Q or K (natural or reordered order)
// summed in fp64 in token order (exact; the same values as the pooling pass's), written
// as fp64 means (for the exact tier) and as the fp16 split with the norms, in one pass.
// Lane l of a warp owns the 16-byte column chunk l % C (C = D / 8) of row l / C of the
// warp's 32 / C rows of the padded grid [B*H, nbp]; padding rows get zero splits.
// Either `norm` (per row, for Q) or `max_bits` (per head, for K) is given.
template <int D, bool GATHER>
__global__ void __launch_bounds__(128) pool_split_kernel(
    const uint4* __restrict__ src, double* __restrict__ pool, __half* __restrict__ hi,
    __half* __restrict__ lo, float* __restrict__ norm, uint32_t* __restrict__ max_bits, int Hg,
    int W, int Hb, int Wb, int nb, int nbp, long long rows_pad) {
  constexpr int C = D / 8;
  constexpr int RPW = 32 / C;
  const int lane = threadIdx.x & 31;
  const int c = lane % C;
  const long long g = (static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5)) * RPW + lane / C;
  if (g >= rows_pad) return;               // whole rows of lanes leave together
  const long long bh = g / nbp;
  const int blk = static_cast<int>(g - bh * nbp);
  const bool valid = blk < nb;
  double m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = 0.0;
  if (valid) {
    const long long S = static_cast<long long>(nb) * 64;
    const int t = blk / (Hb * Wb);
    const int rem = blk - t * (Hb * Wb);
    const int hb = rem / Wb;
    const int wb = rem - hb * Wb;
    const uint4* base = src + bh * S * C + c;
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
          m[2 * k] += static_cast<double>(__uint_as_float(w[k] << 16));
          m[2 * k + 1] += static_cast<double>(__uint_as_float(w[k] & 0xFFFF0000u));
        }
      }
    }
    double* out = pool + (bh * nb + blk) * D + c * 8;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      m[k] = m[k] / 64.0;
      out[k] = m[k];
    }
  }
  __half h8[8], l8[8];
  double n2 = 0.0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    h8[k] = __double2half(m[k]);
    l8[k] = __double2half(m[k] - static_cast<double>(__half2float(h8[k])));
    n2 = fma(m[k], m[k], n2);
  }
  *reinterpret_cast<uint4*>(hi + g * D + c * 8) = *reinterpret_cast<const uint4*>(h8);
  *reinterpret_cast<uint4*>(lo + g * D + c * 8) = *reinterpret_cast<const uint4*>(l8);
#pragma unroll
  for (int o = C / 2; o > 0; o >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, o);
  if (c == 0 && valid) {
    const float nrm = static_cast<float>(sqrt(n2)) * 1.0000001f;
    if (norm != nullptr) norm[bh * nb + blk] = nrm;
    if (max_bits != nullptr) atomicMax(&max_bits[bh], __float_as_uint(nrm));
  }
}

// ------------------------------------------------------------------------------------
// 2. pooled logits on the tensor cores
// ------------------------------------------------------------------------------------
// Persistent and pipelined: the (head, 128-row query tile, 128-column key tile) units
// are split into equal contiguous ranges, one per CTA.  Warp 0 streams the key tiles
// (fp16 hi and lo) through a two-stage TMA ring and reloads the query tile only when it
// changes; warp 1 issues the MMAs into one of two TMEM accumulator pairs; warps 2-5
// (one TMEM lane quadrant each) add the pair, scale, and store 32 x 32 fp32 boxes with
// tiled TMA stores through swizzled staging, while the next unit's MMAs run.
template <int D>
struct LogitCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = 128 * D * 2;   // one 128-row fp16 operand (hi or lo)
  static constexpr int kOffQh = 0;
  static constexpr int kOffQl = kOffQh + kTileBytes;
  static constexpr int kOffK = kOffQl + kTileBytes;        // 2 stages x (hi, lo)
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kOffStage = kOffK + 2 * kStageBytes; // 4 warps x 2 x 4 KB
  static constexpr int kOffBar = kOffStage + 4 * 2 * 4096;
  static constexpr int kSmemBytes = kOffBar + 128 + 1024;
};
constexpr int kLogitThreads = 192;

__device__ __forceinline__ void bulk_wait_read_le1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

template <int D>
__global__ void __launch_bounds__(kLogitThreads, 1) pooled_logits_kernel(
    const __grid_constant__ CUtensorMap map_qh, const __grid_constant__ CUtensorMap map_ql,
    const __grid_constant__ CUtensorMap map_kh, const __grid_constant__ CUtensorMap map_kl,
    const __grid_constant__ CUtensorMap map_out, int nbp, long long units, float scale,
    uint32_t* status) {
  using C = LogitCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* k_full = bars;          // [2]
  uint64_t* k_empty = bars + 2;     // [2]
  uint64_t* acc_full = bars + 4;    // [2]
  uint64_t* acc_empty = bars + 6;   // [2]
  uint64_t* q_full = bars + 8;
  uint64_t* q_empty = bars + 9;
  uint64_t* mma_done = bars + 10;   // the MMA thread's last commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nt = nbp / 128;                        // query tiles = key tiles per head
  const long long u0 = units * blockIdx.x / gridDim.x;
  const long long u1 = units * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 4);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(mma_done, 1);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      long long cur_q = -1;
      int nq = 0;
      long long k = 0;
      bool ok = true;
      for (long long u = u0; u < u1 && ok; ++u, ++k) {
        const long long qt = u / nt;               // (head, query tile)
        const int jt = static_cast<int>(u - qt * nt);
        const long long bh = qt / nt;
        const int it = static_cast<int>(qt - bh * nt);
        if (qt != cur_q) {
          if (nq > 0) ok = mbar_wait(q_empty, (nq - 1) & 1, status, kDevTimeoutTmaFull);
          if (!ok) break;
          mbar_arrive_expect_tx(q_full, 2 * C::kTileBytes);
          const int arow = static_cast<int>(bh * nbp + it * 128);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn) {
            tma_load_2d(smem + C::kOffQh + pn * 16384, &map_qh, q_full, pn * 64, arow);
            tma_load_2d(smem + C::kOffQl + pn * 16384, &map_ql, q_full, pn * 64, arow);
          }
          cur_q = qt;
          ++nq;
        }
        const int st = static_cast<int>(k & 1);
        const long long use = k >> 1;
        if (use > 0) ok = mbar_wait(&k_empty[st], static_cast<uint32_t>((use - 1) & 1), status, kDevTimeoutKvEmpty);
        if (!ok) break;
        unsigned char* kb = smem + C::kOffK + st * C::kStageBytes;
        mbar_arrive_expect_tx(&k_full[st], 2 * C::kTileBytes);
        const int brow = static_cast<int>(bh * nbp + jt * 128);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn) {
          tma_load_2d(kb + pn * 16384, &map_kh, &k_full[st], pn * 64, brow);
          tma_load_2d(kb + C::kTileBytes + pn * 16384, &map_kl, &k_full[st], pn * 64, brow);
        }
      }
      // drain: every copy issued has landed before the CTA may exit (the MMA warp waits
      // for them on the normal path; after an error it may have stopped early)
      for (long long kk = k > 2 ? k - 2 : 0; kk < k; ++kk)
        mbar_wait(&k_full[kk & 1], static_cast<uint32_t>((kk >> 1) & 1), nullptr, kDevTimeoutDrain);
      if (nq > 0) mbar_wait(q_full, (nq - 1) & 1, nullptr, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, 128, false, false);
      const uint32_t qh = smem_u32(smem + C::kOffQh), ql = smem_u32(smem + C::kOffQl);
      long long cur_q = -1;
      int nq = 0;
      long long k = 0;
      bool ok = true;
      for (long long u = u0; u < u1 && ok; ++u, ++k) {
        const long long qt = u / nt;
        if (qt != cur_q) {
          ok = mbar_wait(q_full, nq & 1, status, kDevTimeoutQFull);
          if (!ok) break;
          cur_q = qt;
          ++nq;
        }
        const int st = static_cast<int>(k & 1);
        const long long use = k >> 1;
        ok = mbar_wait(&k_full[st], static_cast<uint32_t>(use & 1), status, kDevTimeoutTmaFull);
        if (ok && use > 0) ok = mbar_wait(&acc_empty[st], static_cast<uint32_t>((use - 1) & 1), status, kDevTimeoutOBar);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kh = smem_u32(smem + C::kOffK + st * C::kStageBytes);
        const uint32_t kl = kh + C::kTileBytes;
        const uint32_t acc = tmem + static_cast<uint32_t>(st * 256);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2, w = kk & 3;
          mma_bf16_ss(acc, sdesc_sw128(qh + pn * 16384 + w * 32, 16, 1024),
                      sdesc_sw128(kh + pn * 16384 + w * 32, 16, 1024), idesc, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2, w = kk & 3;
          mma_bf16_ss(acc + 128, sdesc_sw128(qh + pn * 16384 + w * 32, 16, 1024),
                      sdesc_sw128(kl + pn * 16384 + w * 32, 16, 1024), idesc, kk > 0);
          mma_bf16_ss(acc + 128, sdesc_sw128(ql + pn * 16384 + w * 32, 16, 1024),
                      sdesc_sw128(kh + pn * 16384 + w * 32, 16, 1024), idesc, 1u);
        }
        mma_commit(&k_empty[st]);
        mma_commit(&acc_full[st]);
        if (u + 1 == u1 || (u + 1) / nt != qt) mma_commit(q_empty);
      }
      // every MMA issued (and every commit before this one) has completed before the
      // accumulators are freed and the CTA exits
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, nullptr, kDevTimeoutDrain);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2-5: TMEM lane quadrant warp % 4) ----------------
    const int q4 = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    unsigned char* stage0 = smem + C::kOffStage + (warp - 2) * 8192;
    long long k = 0;
    int nstore = 0;
    for (long long u = u0; u < u1; ++u, ++k) {
      const long long qt = u / nt;
      const int jt = static_cast<int>(u - qt * nt);
      const long long bh = qt / nt;
      const int it = static_cast<int>(qt - bh * nt);
      const int st = static_cast<int>(k & 1);
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[st], static_cast<uint32_t>((k >> 1) & 1), status,
                                                        kDevTimeoutSFull));
      if (!ok) break;
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + static_cast<uint32_t>(st * 256);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t a0[32], a1[32];
        tmem_ld32(acc + 32 * c, a0);
        tmem_ld32(acc + 128 + 32 * c, a1);
        tmem_wait_ld();
        if (c == 3) {                              // the pair is read: release it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[st]);
        }
        unsigned char* stage = stage0 + (nstore & 1) * 4096;
        if (lane == 0) bulk_wait_read_le1();       // the copy from this buffer has read it
        __syncwarp();
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<float4*>(stage + lane * 128 + ((ch ^ (lane & 7)) << 4)) =
              make_float4((__uint_as_float(a0[4 * ch]) + __uint_as_float(a1[4 * ch])) * scale,
                          (__uint_as_float(a0[4 * ch + 1]) + __uint_as_float(a1[4 * ch + 1])) * scale,
                          (__uint_as_float(a0[4 * ch + 2]) + __uint_as_float(a1[4 * ch + 2])) * scale,
                          (__uint_as_float(a0[4 * ch + 3]) + __uint_as_float(a1[4 * ch + 3])) * scale);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&map_out, stage, jt * 128 + 32 * c, static_cast<int>(bh * nbp + it * 128 + 32 * q4));
          bulk_commit_group();
        }
        ++nstore;
      }
    }
    if (lane == 0) bulk_wait_all();                // the stores have landed
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------
// 3. per-row cut with certificate (one warp per row)
// ------------------------------------------------------------------------------------
struct SelectParams {
  const float* logits;
  const float* qnorm;
  const uint32_t* kmax_bits;
  uint32_t* bits;
  int32_t* row_idx;
  int32_t* row_cnt;
  int32_t* rescue_list;     // [BH, nb]
  int32_t* rescue_cnt;      // [BH]
  int nb, nbp, nw, Hb, Wb;
  int sta_on, wt2, wh2, ww2;
  float thr;
  float scale;
  int thr_mode;             // +1: thr >= 1, -1: thr <= 0, 0: otherwise
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

constexpr int kSelWarps = 8;   // rows (warps) per CTA of the select kernel

// One warp per row.  The row's probabilities live in this warp's slice of shared memory
// and every pass over them is a plain loop, so the kernel's code stays small (the passes
// of a register-resident version, unrolled over the row, overflowed the instruction
// cache) and its register count low.  Block j = lane + 32 t; lane l keeps t = 4 g + c
// in ps4[32 g + l].c, so each access is one conflict-free 16-byte load or store per lane.
// Sums are taken per lane in t order, then by a fixed butterfly.
__global__ void __launch_bounds__(256) mask_select_kernel(const SelectParams prm, long long rows) {
  extern __shared__ float4 psm4[];                     // [kSelWarps][T / 4][32]
  __shared__ uint32_t cand_key[kSelWarps][kSelCand];   // per warp: the cut's candidates
  __shared__ int cand_idx[kSelWarps][kSelCand];
  __shared__ __align__(16) uint32_t words[kSelWarps][64];   // per warp: the row's bitmask
  const long long row = static_cast<long long>(blockIdx.x) * kSelWarps + (threadIdx.x >> 5);
  const int wslot = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int nb = prm.nb;
  const int G = prm.nbp / 128;                         // float4 groups per lane
  const long long bh = row / nb;
  const int i = static_cast<int>(row - bh * nb);
  const float* a = prm.logits + (bh * prm.nbp + i) * static_cast<long long>(prm.nbp);
  float4* ps4 = psm4 + static_cast<size_t>(wslot) * G * 32 + lane;   // ps4[32 g]

  // ---- softmax (fp32): P_j = exp(A_j - max) / sum ------------------------------------
  float m = -INFINITY;
#pragma unroll 2
  for (int g = 0; g < G; ++g) {
    const int j = lane + 128 * g;
    float4 x;
    x.x = j < nb ? a[j] : -INFINITY;
    x.y = j + 32 < nb ? a[j + 32] : -INFINITY;
    x.z = j + 64 < nb ? a[j + 64] : -INFINITY;
    x.w = j + 96 < nb ? a[j + 96] : -INFINITY;
    ps4[32 * g] = x;
    m = fmaxf(m, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
  }
  m = warp_max(m);
  float s = 0.f;
  for (int g = 0; g < G; ++g) {
    float4 x = ps4[32 * g];
    x.x = __expf(x.x - m);
    x.y = __expf(x.y - m);
    x.z = __expf(x.z - m);
    x.w = __expf(x.w - m);
    ps4[32 * g] = x;
    s += x.x;
    s += x.y;
    s += x.z;
    s += x.w;
  }
  s = warp_sum(s);
  const float inv = 1.0f / s;

  const float thr = prm.thr;
  bool certified = false;
  uint32_t kcut = 0;
  // rho: relative error of every probability (two logits' errors, exp, division);
  // eta: error of a ranked mass.
  const float eps = prm.scale * prm.qnorm[bh * nb + i] * __uint_as_float(prm.kmax_bits[bh]) * kLogitErr;
  const float rho = 2.f * eps + 1e-5f;
  const float eta = rho + 3.5e-6f;
  // Bracket [lo, hi) of fp32 keys (bit patterns of probabilities) with
  // mass(P >= lo) >= thr > mass(P >= hi); every block with key >= hi is kept and every
  // block with key < lo dropped.  Probes, in order: one sixteenth of the row maximum
  // (1 / sum; most rows keep a few large blocks, and then [guess, 1] already holds at
  // most kSelCand of them); below it, the lower end from mass(P >= x) >= 1 - nb x (every
  // block below x holds less than x), then 0; then points interpolated linearly in the
  // key between the ends, kept within the middle half of the bracket.  The computed mass
  // is monotone in the key (sums of a subset in a fixed order), so any bracket that
  // satisfies the invariant leads to the same decision.  The first probe's pass also
  // scales the exponentials into probabilities.
  uint32_t lo = 0u, hi = 0x3F800001u;              // 0x3F800001: above 1.0
  float mlo = 0.f, mhi = 0.f;
  int clo = 0, chi = 0;
  int phase = 0;                                   // 0 guess, 1 lower bound, 2 zero, 3 narrow
  bool bracket = false;
  uint32_t probe = max(__float_as_uint(inv), 4u << 23) - (4u << 23);
  for (int it = 0; it < 128; ++it) {
    float mm = 0.f;
    int cm = 0;
    auto acc = [&](float v) {
      const bool ge = __float_as_uint(v) >= probe;
      mm += ge ? v : 0.f;
      cm += ge ? 1 : 0;
    };
    if (it == 0) {
      for (int g = 0; g < G; ++g) {
        float4 x = ps4[32 * g];
        x.x *= inv;
        x.y *= inv;
        x.z *= inv;
        x.w *= inv;
        ps4[32 * g] = x;
        acc(x.x);
        acc(x.y);
        acc(x.z);
        acc(x.w);
      }
    } else {
      for (int g = 0; g < G; ++g) {
        const float4 x = ps4[32 * g];
        acc(x.x);
        acc(x.y);
        acc(x.z);
        acc(x.w);
      }
    }
    if (prm.thr_mode != 0) break;                  // thr >= 1: keep all; thr <= 0: none
    cm = __reduce_add_sync(0xffffffffu, cm);
    mm = warp_sum(mm);
    if (mm >= thr) {
      lo = probe;
      mlo = mm;
      clo = cm;
      phase = 3;
    } else if (phase == 0) {
      hi = probe;
      mhi = mm;
      chi = cm;
      phase = 1;
      probe = __float_as_uint(0.5f * (1.f - thr) / static_cast<float>(nb));
      continue;
    } else if (phase == 1) {
      phase = 2;
      probe = 0u;
      continue;
    } else if (phase == 2) {
      break;                                       // total mass below thr: no bracket
    } else {
      hi = probe;
      mhi = mm;
      chi = cm;
    }
    if (clo - chi <= kSelCand || hi - lo <= 1u) {
      bracket = clo - chi <= kSelCand;
      break;
    }
    const uint32_t w = hi - lo;
    const float f = fminf(fmaxf((mlo - thr) / (mlo - mhi), 0.25f), 0.75f);
    probe = lo + min(max(static_cast<uint32_t>(static_cast<float>(w) * f), 1u), w - 1u);
  }
  if (prm.thr_mode != 0) {
    certified = true;
    kcut = prm.thr_mode > 0 ? 0u : 0xFFFFFFFFu;
  } else if (bracket) {
    // gather the candidates in index order into this warp's slots; the largest value
    // below the bracket is the next value after the last candidate
    uint32_t* ck = cand_key[wslot];
    int* ci = cand_idx[wslot];
    const uint32_t lt_mask = (1u << lane) - 1u;
    int ncand = 0;
    float below = 0.f;
    for (int g = 0; g < G; ++g) {
      const float4 x = ps4[32 * g];
      const float v[4] = {x.x, x.y, x.z, x.w};
      bool in[4];
      bool any = false;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t key = __float_as_uint(v[c]);
        const bool valid = lane + 32 * (4 * g + c) < nb;
        in[c] = valid && key >= lo && key < hi;
        if (valid && key < lo) below = fmaxf(below, v[c]);
        any = any || in[c];
      }
      if (__any_sync(0xffffffffu, any)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t bal = __ballot_sync(0xffffffffu, in[c]);
          if (in[c]) {
            const int pos = ncand + __popc(bal & lt_mask);
            ck[pos] = __float_as_uint(v[c]);
            ci[pos] = lane + 32 * (4 * g + c);
          }
          ncand += __popc(bal);
        }
      }
    }
    below = warp_max(below);
    __syncwarp();
    // lane n < ncand: rank of candidate n (value descending, index ascending) and its
    // exclusive ranked mass, mass(P >= hi) plus the candidates ranked before it (added in
    // index order)
    const uint32_t kn = lane < ncand ? ck[lane] : 0u;
    const int in_ = lane < ncand ? ci[lane] : 0x7FFFFFFF;
    int rank = 0;
    float e = mhi;
    for (int d = 0; d < ncand; ++d) {
      const uint32_t kd = ck[d];
      const bool before = kd > kn || (kd == kn && ci[d] < in_);
      rank += before ? 1 : 0;
      e += before ? __uint_as_float(kd) : 0.f;
    }
    __syncwarp();
    // the cut: the candidate whose exclusive mass is below thr and inclusive mass reaches it
    const float pc = __uint_as_float(kn);
    const uint32_t cb = __ballot_sync(0xffffffffu, lane < ncand && e < thr && e + pc >= thr);
    if (cb != 0u) {
      const int cl = __ffs(cb) - 1;
      const int crank = __shfl_sync(0xffffffffu, rank, cl);
      const float e_above = __shfl_sync(0xffffffffu, e, cl);
      const float p_cut = __shfl_sync(0xffffffffu, pc, cl);
      // next value below the cut: the candidate ranked right after it, else the largest
      // value below the bracket; n_at: candidates equal to the cut value
      const uint32_t nxt = __ballot_sync(0xffffffffu, lane < ncand && rank == crank + 1);
      const float p_next = nxt != 0u ? __shfl_sync(0xffffffffu, pc, __ffs(nxt) - 1) : below;
      const int n_at = __popc(__ballot_sync(0xffffffffu, lane < ncand && pc == p_cut));
      kcut = __float_as_uint(p_cut);
      // Certificate for the cut: the kept set {P >= p_cut} must have exact mass > thr, and
      // without its (exactly) smallest member -- at most e_above + eta + rho p_cut --
      // exact mass < thr.
      certified = (thr - e_above > eta + rho * p_cut) && (e_above + p_cut - thr > eta) &&
                  n_at == 1 && (p_cut - p_next > 2.f * rho * p_cut);
    }
  }
  if (!certified) {
    if (lane == 0) {
      const int pos = atomicAdd(&prm.rescue_cnt[bh], 1);
      prm.rescue_list[bh * nb + pos] = i;
    }
    return;
  }
  // ---- emit: keep P >= P_c, OR the static window ------------------------------------
  // The window test follows block j = lane + 32 t through its (frame, row, column)
  // coordinates by adding those of 32 with carries (no division per block).
  const int nw = prm.nw;
  const bool win = prm.sta_on != 0;
  int ti = 0, hi_ = 0, wi = 0, tj = 0, hj = 0, wj = 0, dt = 0, dh = 0, dw = 0;
  if (win) {
    const int HW = prm.Hb * prm.Wb;
    ti = i / HW;
    hi_ = (i / prm.Wb) % prm.Hb;
    wi = i % prm.Wb;
    tj = lane / HW;
    hj = (lane / prm.Wb) % prm.Hb;
    wj = lane % prm.Wb;
    dt = 32 / HW;
    dh = (32 / prm.Wb) % prm.Hb;
    dw = 32 % prm.Wb;
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  int32_t* ridx = prm.row_idx != nullptr ? prm.row_idx + (bh * nb + i) * static_cast<long long>(nb) : nullptr;
  int run = 0;
  for (int g = 0; 4 * g < nw; ++g) {
    const float4 x = ps4[32 * g];
    const float v[4] = {x.x, x.y, x.z, x.w};
    uint32_t kb[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = lane + 32 * (4 * g + c);
      bool k = j < nb && __float_as_uint(v[c]) >= kcut;
      if (win) {
        k = k || (j < nb && abs(ti - tj) <= prm.wt2 && abs(hi_ - hj) <= prm.wh2 && abs(wi - wj) <= prm.ww2);
        wj += dw;
        const int cw = wj >= prm.Wb ? 1 : 0;
        wj -= cw * prm.Wb;
        hj += dh + cw;
        const int ch = hj >= prm.Hb ? 1 : 0;
        hj -= ch * prm.Hb;
        tj += dt + ch;
      }
      kb[c] = __ballot_sync(0xffffffffu, k);
      if (ridx != nullptr) {
        if (k) ridx[run + __popc(kb[c] & lt_mask)] = j;
        run += __popc(kb[c]);
      }
    }
    if (lane == 0) *reinterpret_cast<uint4*>(&words[wslot][4 * g]) = make_uint4(kb[0], kb[1], kb[2], kb[3]);
  }
  __syncwarp();
  // the row's bitmask words in one coalesced store, and the kept count
  uint32_t* brow = prm.bits + (bh * nb + i) * nw;
  int cnt = 0;
  for (int w = lane; w < nw; w += 32) {
    const uint32_t wv = words[wslot][w];
    brow[w] = wv;
    cnt += __popc(wv);
  }
  if (prm.row_cnt != nullptr) {
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) prm.row_cnt[bh * nb + i] = cnt;
  }
}

size_t select_smem_bytes(int nbp) { return static_cast<size_t>(kSelWarps) * nbp * sizeof(float); }

cudaError_t launch_select(const SelectParams& p, long long rows, cudaStream_t st) {
  const size_t smem = select_smem_bytes(p.nbp);
  cudaError_t e = cudaFuncSetAttribute(mask_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  mask_select_kernel<<<static_cast<unsigned>((rows + kSelWarps - 1) / kSelWarps), kSelWarps * 32, smem, st>>>(
      p, rows);
  return cudaGetLastError();
}

}  // namespace

int mask_fast_nbp(int nb) { return (nb + 255) / 256 * 256; }

size_t mask_fast_scratch_bytes(const Dims& d) {
  const size_t nbp = mask_fast_nbp(d.nb);
  const size_t split = align_up(static_cast<size_t>(d.BH) * nbp * d.D * 2, 256);
  return 4 * split + align_up(static_cast<size_t>(d.BH) * d.nb * 4, 256)      // qnorm
         + align_up(static_cast<size_t>(d.BH) * 4, 256)                       // kmax
         + align_up(static_cast<size_t>(d.BH) * nbp * nbp * 4, 256)           // logits
         + align_up(static_cast<size_t>(d.BH) * d.nb * 4, 256)                // rescue list
         + align_up(static_cast<size_t>(d.BH) * 4, 256);                      // rescue counts
}

bool mask_fast_supported(const Dims& d) { return d.nb <= 2048; }

namespace {

// Scratch layout of the fast tier (see mask_fast_scratch_bytes).
struct FastScratch {
  __half *qh, *ql, *kh, *kl;
  float* qnorm;
  uint32_t* kmax;
  float* logits;
  int32_t* rlist;
  int32_t* rc;
};

FastScratch fast_scratch(const Dims& d, void* scratch) {
  const int nbp = mask_fast_nbp(d.nb);
  const size_t split = align_up(static_cast<size_t>(d.BH) * nbp * d.D * 2, 256);
  char* base = static_cast<char*>(scratch);
  FastScratch f;
  f.qh = reinterpret_cast<__half*>(base);
  f.ql = reinterpret_cast<__half*>(base + split);
  f.kh = reinterpret_cast<__half*>(base + 2 * split);
  f.kl = reinterpret_cast<__half*>(base + 3 * split);
  char* c = base + 4 * split;
  f.qnorm = reinterpret_cast<float*>(c);
  c += align_up(static_cast<size_t>(d.BH) * d.nb * 4, 256);
  f.kmax = reinterpret_cast<uint32_t*>(c);
  c += align_up(static_cast<size_t>(d.BH) * 4, 256);
  f.logits = reinterpret_cast<float*>(c);
  c += align_up(static_cast<size_t>(d.BH) * nbp * nbp * 4, 256);
  f.rlist = reinterpret_cast<int32_t*>(c);
  c += align_up(static_cast<size_t>(d.BH) * d.nb * 4, 256);
  f.rc = reinterpret_cast<int32_t*>(c);
  return f;
}

}  // namespace

namespace {
// Tier 2a: the pooled logits from the split (independent of thr).
cudaError_t mask_fast_logits(const Dims& d, double scale, const FastScratch& f, uint32_t* status,
                             cudaStream_t st) {
  const int nbp = mask_fast_nbp(d.nb);
  const long long rows_pad = static_cast<long long>(d.BH) * nbp;
  CUtensorMap mqh, mql, mkh, mkl, mout;
  if (!(make_map_16(&mqh, f.qh, rows_pad, d.D, 128, true) && make_map_16(&mql, f.ql, rows_pad, d.D, 128, true) &&
        make_map_16(&mkh, f.kh, rows_pad, d.D, 128, true) && make_map_16(&mkl, f.kl, rows_pad, d.D, 128, true) &&
        make_map_f32(&mout, f.logits, rows_pad, nbp)))
    return cudaErrorInvalidValue;
  const long long units = static_cast<long long>(d.BH) * (nbp / 128) * (nbp / 128);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned grid = static_cast<unsigned>(units < sms ? units : sms);
  cudaError_t e;
  if (d.D == 64) {
    e = cudaFuncSetAttribute(pooled_logits_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             LogitCfg<64>::kSmemBytes);
    if (e != cudaSuccess) return e;
    pooled_logits_kernel<64><<<grid, kLogitThreads, LogitCfg<64>::kSmemBytes, st>>>(
        mqh, mql, mkh, mkl, mout, nbp, units, static_cast<float>(scale), status);
  } else {
    e = cudaFuncSetAttribute(pooled_logits_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             LogitCfg<128>::kSmemBytes);
    if (e != cudaSuccess) return e;
    pooled_logits_kernel<128><<<grid, kLogitThreads, LogitCfg<128>::kSmemBytes, st>>>(
        mqh, mql, mkh, mkl, mout, nbp, units, static_cast<float>(scale), status);
  }
  return cudaGetLastError();
}

template <int D, bool GATHER>
void launch_pool_split(const void* x, double* pool, __half* hi, __half* lo, float* norm, uint32_t* max_bits,
                       const Dims& d, cudaStream_t st) {
  const int nbp = mask_fast_nbp(d.nb);
  const long long rows_pad = static_cast<long long>(d.BH) * nbp;
  constexpr int kRowsPerCta = 4 * (32 / (D / 8));
  pool_split_kernel<D, GATHER><<<static_cast<unsigned>((rows_pad + kRowsPerCta - 1) / kRowsPerCta), 128, 0, st>>>(
      static_cast<const uint4*>(x), pool, hi, lo, norm, max_bits, d.Hg, d.W, d.Hb, d.Wb, d.nb, nbp, rows_pad);
}
}  // namespace

// Tiers 1-2a from fp64 pools: split of the pooled means, then the pooled logits.
cudaError_t mask_fast_prepare(const double* qp, const double* kp, const Dims& d, double scale,
                              void* scratch, uint32_t* status, cudaStream_t st) {
  const int nbp = mask_fast_nbp(d.nb);
  const FastScratch f = fast_scratch(d, scratch);
  cudaError_t e = cudaMemsetAsync(f.kmax, 0, static_cast<size_t>(d.BH) * 4, st);
  if (e != cudaSuccess) return e;
  const long long rows_pad = static_cast<long long>(d.BH) * nbp;
  const int vec16 = ((reinterpret_cast<uintptr_t>(qp) | reinterpret_cast<uintptr_t>(kp)) & 15) == 0;
  if (d.D == 64)
    split_pools_kernel<64><<<static_cast<unsigned>((rows_pad + 7) / 8), 256, 0, st>>>(
        qp, kp, d.nb, nbp, rows_pad, f.qh, f.ql, f.kh, f.kl, f.qnorm, f.kmax, vec16);
  else
    split_pools_kernel<128><<<static_cast<unsigned>((rows_pad + 7) / 8), 256, 0, st>>>(
        qp, kp, d.nb, nbp, rows_pad, f.qh, f.ql, f.kh, f.kl, f.qnorm, f.kmax, vec16);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return mask_fast_logits(d, scale, f, status, st);
}

// Tiers 1-2a from the bf16 tokens (natural order when `natural`, else reordered): the
// pools (written to qp_out / kp_out for the exact tier), their split and norms in one
// pass per tensor, then the pooled logits.
cudaError_t mask_fast_prepare_tokens(const void* q, const void* k, bool natural, double* qp_out,
                                     double* kp_out, const Dims& d, double scale, void* scratch,
                                     uint32_t* status, cudaStream_t st) {
  const FastScratch f = fast_scratch(d, scratch);
  cudaError_t e = cudaMemsetAsync(f.kmax, 0, static_cast<size_t>(d.BH) * 4, st);
  if (e != cudaSuccess) return e;
  if (d.D == 64) {
    if (natural) {
      launch_pool_split<64, true>(q, qp_out, f.qh, f.ql, f.qnorm, nullptr, d, st);
      launch_pool_split<64, true>(k, kp_out, f.kh, f.kl, nullptr, f.kmax, d, st);
    } else {
      launch_pool_split<64, false>(q, qp_out, f.qh, f.ql, f.qnorm, nullptr, d, st);
      launch_pool_split<64, false>(k, kp_out, f.kh, f.kl, nullptr, f.kmax, d, st);
    }
  } else {
    if (natural) {
      launch_pool_split<128, true>(q, qp_out, f.qh, f.ql, f.qnorm, nullptr, d, st);
      launch_pool_split<128, true>(k, kp_out, f.kh, f.kl, nullptr, f.kmax, d, st);
    } else {
      launch_pool_split<128, false>(q, qp_out, f.qh, f.ql, f.qnorm, nullptr, d, st);
      launch_pool_split<128, false>(k, kp_out, f.kh, f.kl, nullptr, f.kmax, d, st);
    }
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return mask_fast_logits(d, scale, f, status, st);
}

// Tier 2b: the certified cut for one thr from the logits mask_fast_prepare wrote.  Rows
// that are not certified are listed per head in rescue_list / rescue_cnt (returned) for
// the fp64 kernel; the lists are rebuilt by every call.
cudaError_t mask_fast_select(const Dims& d, double scale, double thr, const nabla_window& w,
                             uint32_t* bits, int32_t* ridx, int32_t* rcnt, void* scratch,
                             int32_t** rescue_list, int32_t** rescue_cnt, cudaStream_t st) {
  const int nbp = mask_fast_nbp(d.nb);
  const FastScratch f = fast_scratch(d, scratch);
  cudaError_t e = cudaMemsetAsync(f.rc, 0, static_cast<size_t>(d.BH) * 4, st);
  if (e != cudaSuccess) return e;
  SelectParams p;
  p.logits = f.logits;
  p.qnorm = f.qnorm;
  p.kmax_bits = f.kmax;
  p.bits = bits;
  p.row_idx = ridx;
  p.row_cnt = rcnt;
  p.rescue_list = f.rlist;
  p.rescue_cnt = f.rc;
  p.nb = d.nb;
  p.nbp = nbp;
  p.nw = d.nw;
  p.Hb = d.Hb;
  p.Wb = d.Wb;
  p.sta_on = (w.t | w.h | w.w) != 0;
  p.wt2 = w.t / 2;
  p.wh2 = w.h / 2;
  p.ww2 = w.w / 2;
  p.thr = static_cast<float>(thr);
  p.thr_mode = thr >= 1.0 ? 1 : (thr <= 0.0 ? -1 : 0);
  p.scale = static_cast<float>(scale);
  const long long rows = static_cast<long long>(d.BH) * d.nb;
  e = launch_select(p, rows, st);
  *rescue_list = f.rlist;
  *rescue_cnt = f.rc;
  return e;
}

}  // namespace nabla
