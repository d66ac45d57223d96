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
//  1. split_pools_kernel: the fp64 block means q, k are split into fp16 pairs
//     q = q_hi + q_lo + r (|r| <= 2^-22 |q|), padded to a multiple of 256 rows; row
//     norms |q_i| and the per-head maximum |k_j| are kept for the error bound.
//  2. pooled_logits_kernel: A = scale * (q_hi k_hi^T + (q_hi k_lo^T + q_lo k_hi^T)) with
//     tcgen05 (M = 128, N = 256, K = 16 per instruction, fp32 accumulate in TMEM; the
//     dominant q_hi k_hi^T term has its own accumulator), written to an fp32 scratch.
//  3. mask_select_kernel: one warp per row: softmax in fp32; the cut value P_c (the
//     smallest kept probability) by extracting maxima while the running mass is below
//     thr (rows keeping a few blocks), else by bisection over the fp32 bit patterns until
//     the interval where the mass at or above crosses thr holds at most 16 blocks, which
//     are then ranked and walked; then the certificate: with rho the proven relative
//     error of every P_j,
//        thr - E_above > eta,  E_at_or_above - thr > eta,  P_c unique,
//        P_c - P_next > 2 rho P_c,
//     where eta = rho + 3e-6 bounds the error of the ranked masses.  A certified row
//     keeps exactly the blocks with P_j >= P_c (the same set the exact ranking keeps);
//     the others are appended to a per-head list that the fp64 kernel recomputes.
#include <math.h>

#include <cudaTypedefs.h>

#include "common.cuh"

namespace nabla {

bool make_map_16(CUtensorMap* map, const void* base, long long rows, int D, int box_rows,
                 bool fp16);

namespace {

// Per-logit error bound, relative to scale * |q_i| * max_j |k_j|: split residuals
// (3 x 2^-22), eight fp32 accumulations of the leading product (8 x 2^-22, allowing
// truncating adds), the correction products and the final add / scale (~2^-22).
constexpr float kLogitErr = 4.0e-6f;
constexpr int kSelCand = 16;   // the cut's bisection stops at this many candidates

// ------------------------------------------------------------------------------------
// 1. fp16 split of the pooled means + norms
// ------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) split_pools_kernel(
    const double* __restrict__ qpool, const double* __restrict__ kpool, int nb, int nbp,
    long long rows_pad, __half* __restrict__ qh, __half* __restrict__ ql, __half* __restrict__ kh,
    __half* __restrict__ kl, float* __restrict__ qnorm, uint32_t* __restrict__ kmax_bits) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);   // padded
  const int lane = threadIdx.x & 31;
  if (row >= rows_pad) return;
  const long long bh = row / nbp;
  const int i = static_cast<int>(row - bh * nbp);
  const bool valid = i < nb;
  constexpr int E = D / 32;
  double nq = 0.0, nk = 0.0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int d = lane * E + e;
    const double q = valid ? qpool[(bh * nb + i) * D + d] : 0.0;
    const double k = valid ? kpool[(bh * nb + i) * D + d] : 0.0;
    const __half q1 = __double2half(q);
    const __half k1 = __double2half(k);
    qh[row * D + d] = q1;
    kh[row * D + d] = k1;
    ql[row * D + d] = __double2half(q - static_cast<double>(__half2float(q1)));
    kl[row * D + d] = __double2half(k - static_cast<double>(__half2float(k1)));
    nq = fma(q, q, nq);
    nk = fma(k, k, nk);
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

// ------------------------------------------------------------------------------------
// 2. pooled logits on the tensor cores
// ------------------------------------------------------------------------------------
template <int D>
struct LogitCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kABytes = 128 * D * 2;    // one 128-row fp16 operand
  static constexpr int kBBytes = 256 * D * 2;    // one 256-row fp16 operand
  static constexpr int kOffQh = 0;
  static constexpr int kOffQl = kOffQh + kABytes;
  static constexpr int kOffKh = kOffQl + kABytes;
  static constexpr int kOffKl = kOffKh + kBBytes;
  static constexpr int kOffBar = kOffKl + kBBytes;
  static constexpr int kSmemBytes = kOffBar + 64 + 1024;
};

template <int D>
__global__ void __launch_bounds__(128, 1) pooled_logits_kernel(
    const __grid_constant__ CUtensorMap map_qh, const __grid_constant__ CUtensorMap map_ql,
    const __grid_constant__ CUtensorMap map_kh, const __grid_constant__ CUtensorMap map_kl,
    float* __restrict__ logits, int nbp, float scale, uint32_t* status) {
  using C = LogitCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* done = full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int it = blockIdx.x, jt = blockIdx.y;
  const long long bh = blockIdx.z;

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const int arow = static_cast<int>(bh * nbp + it * 128);
      const int brow = static_cast<int>(bh * nbp + jt * 256);
      mbar_arrive_expect_tx(full, 2 * C::kABytes + 2 * C::kBBytes);
#pragma unroll
      for (int pn = 0; pn < C::kPanels; ++pn) {
        tma_load_2d(smem + C::kOffQh + pn * 16384, &map_qh, full, pn * 64, arow);
        tma_load_2d(smem + C::kOffQl + pn * 16384, &map_ql, full, pn * 64, arow);
        tma_load_2d(smem + C::kOffKh + pn * 32768, &map_kh, full, pn * 64, brow);
        tma_load_2d(smem + C::kOffKl + pn * 32768, &map_kl, full, pn * 64, brow);
      }
      const bool ok = mbar_wait(full, 0, status, kDevTimeoutTmaFull);
      tc_fence_after();
      if (ok) {
        constexpr uint32_t idesc = idesc_f16_f32(128, 256, false, false);
        const uint32_t qh = smem_u32(smem + C::kOffQh), ql = smem_u32(smem + C::kOffQl);
        const uint32_t kh = smem_u32(smem + C::kOffKh), kl = smem_u32(smem + C::kOffKl);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2, w = kk & 3;
          mma_bf16_ss(tmem, sdesc_sw128(qh + pn * 16384 + w * 32, 16, 1024),
                      sdesc_sw128(kh + pn * 32768 + w * 32, 16, 1024), idesc, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2, w = kk & 3;
          mma_bf16_ss(tmem + 256, sdesc_sw128(qh + pn * 16384 + w * 32, 16, 1024),
                      sdesc_sw128(kl + pn * 32768 + w * 32, 16, 1024), idesc, kk > 0);
          mma_bf16_ss(tmem + 256, sdesc_sw128(ql + pn * 16384 + w * 32, 16, 1024),
                      sdesc_sw128(kh + pn * 32768 + w * 32, 16, 1024), idesc, 1u);
        }
      }
      mma_commit(done);
    }
    __syncwarp();
  }
  const bool ok = __all_sync(0xffffffffu, mbar_wait(done, 0, status, kDevTimeoutSFull));
  tc_fence_after();
  if (ok) {
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int row = warp * 32 + lane;
    float* dst = logits + (bh * nbp + it * 128 + row) * static_cast<long long>(nbp) + jt * 256;
#pragma unroll 1
    for (int c0 = 0; c0 < 256; c0 += 32) {
      uint32_t a0[32], a1[32];
      tmem_ld32(tmem + lane_base + c0, a0);
      tmem_ld32(tmem + lane_base + 256 + c0, a1);
      tmem_wait_ld();
      float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        d4[c] = make_float4((__uint_as_float(a0[4 * c]) + __uint_as_float(a1[4 * c])) * scale,
                            (__uint_as_float(a0[4 * c + 1]) + __uint_as_float(a1[4 * c + 1])) * scale,
                            (__uint_as_float(a0[4 * c + 2]) + __uint_as_float(a1[4 * c + 2])) * scale,
                            (__uint_as_float(a0[4 * c + 3]) + __uint_as_float(a1[4 * c + 3])) * scale);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
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

template <int TPL>
__global__ void __launch_bounds__(256) mask_select_kernel(const SelectParams prm, long long rows) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int nb = prm.nb;
  const long long bh = row / nb;
  const int i = static_cast<int>(row - bh * nb);
  const float* a = prm.logits + (bh * prm.nbp + i) * static_cast<long long>(prm.nbp);

  float p[TPL];
  float m = -INFINITY;
#pragma unroll
  for (int t = 0; t < TPL; ++t) {
    const int j = lane + 32 * t;
    p[t] = (j < nb) ? a[j] : -INFINITY;
    m = fmaxf(m, p[t]);
  }
  m = warp_max(m);
  float s = 0.f;
#pragma unroll
  for (int t = 0; t < TPL; ++t) {
    p[t] = __expf(p[t] - m);
    s += p[t];
  }
  s = warp_sum(s);
  const float inv = 1.0f / s;
#pragma unroll
  for (int t = 0; t < TPL; ++t) p[t] *= inv;

  // Largest key k (fp32 bit pattern of a probability) with mass(P >= k) >= thr.
  const float thr = prm.thr;
  auto mass_ge = [&](uint32_t k) {
    float acc = 0.f;
#pragma unroll
    for (int t = 0; t < TPL; ++t) acc += (__float_as_uint(p[t]) >= k) ? p[t] : 0.f;
    return warp_sum(acc);
  };
  bool certified = false;
  uint32_t kcut = 0;
  // rho: relative error of every probability (two logits' errors, exp, division);
  // eta: error of a ranked mass.
  const float eps = prm.scale * prm.qnorm[bh * nb + i] * __uint_as_float(prm.kmax_bits[bh]) * kLogitErr;
  const float rho = 2.f * eps + 1e-5f;
  const float eta = rho + 3.5e-6f;
  // Certificate for a cut at value p_cut with ranked masses e_above (strictly above) and
  // e_at (at or above), the next smaller value p_next and n_at values equal to p_cut.
  // The kept set {P >= p_cut} must have exact mass > thr, and without its (exactly)
  // smallest member -- at most e_above + eta + rho p_cut -- exact mass < thr.
  auto certify = [&](float e_above, float e_at, float p_cut, float p_next, int n_at) {
    return (thr - e_above > eta + rho * p_cut) && (e_at - thr > eta) && n_at == 1 &&
           (p_cut - p_next > 2.f * rho * p_cut);
  };
  if (prm.thr_mode != 0) {            // thr >= 1: keep every block; thr <= 0: none
    certified = true;
    kcut = prm.thr_mode > 0 ? 0u : 0xFFFFFFFFu;
  } else {
    // Fast path: take maxima in descending order (ties: lower block index first) while
    // the running mass is below thr; most rows keep only a few blocks.
    constexpr int kMaxExtract = 16;
    uint64_t taken = 0;                 // bit t: p[t] of this lane already taken
    float acc = 0.f, acc_prev = 0.f;
    bool found = false;
    float p_cut = 0.f;
    for (int e = 0; e <= kMaxExtract; ++e) {
      float best = -1.f;
      int bj = 0x7FFFFFFF;
#pragma unroll
      for (int t = 0; t < TPL; ++t)
        if (!((taken >> t) & 1ull) && p[t] > best) { best = p[t]; bj = lane + 32 * t; }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
        if (ov > best || (ov == best && oj < bj)) { best = ov; bj = oj; }
      }
      if (found) {                      // one more maximum: the first value below the cut
        certified = certify(acc_prev, acc, p_cut, fmaxf(best, 0.f), best == p_cut ? 2 : 1);
        break;
      }
      if (bj == 0x7FFFFFFF || e == kMaxExtract) break;
      if ((bj & 31) == lane) taken |= 1ull << (bj >> 5);
      acc_prev = acc;
      acc += best;
      if (acc >= thr) {
        found = true;
        p_cut = best;
        kcut = __float_as_uint(best);
      }
    }
    if (!found) {
      // General path: bisection over the fp32 bit patterns until the interval [lo, hi)
      // where the mass at or above crosses thr holds at most kSelCand blocks, then the
      // candidates are ranked (value descending, index ascending) and walked from
      // mass(P >= hi); the last kept candidate is the cut.
      auto mass_cnt_ge = [&](uint32_t k, int* cnt) {
        float acc = 0.f;
        int c = 0;
#pragma unroll
        for (int t = 0; t < TPL; ++t) {
          const bool ge = __float_as_uint(p[t]) >= k;
          acc += ge ? p[t] : 0.f;
          c += ge ? 1 : 0;
        }
        *cnt = __reduce_add_sync(0xffffffffu, c);
        return warp_sum(acc);
      };
      int clo = 0, chi = 0;
      if (mass_cnt_ge(0u, &clo) >= thr) {
        uint32_t lo = 0u, hi = 0x3F800001u;      // mass_ge(lo) >= thr > mass_ge(hi)
        float mass_hi = 0.f;
        while (clo - chi > kSelCand && hi - lo > 1u) {
          const uint32_t mid = lo + ((hi - lo) >> 1);
          int cm = 0;
          const float mm = mass_cnt_ge(mid, &cm);
          if (mm >= thr) {
            lo = mid;
            clo = cm;
          } else {
            hi = mid;
            chi = cm;
            mass_hi = mm;
          }
        }
        if (clo - chi <= kSelCand) {
          // gather the candidates in index order: candidate n goes to lane n (each lane
          // holds the blocks lane + 32 t)
          uint32_t ck = 0u;
          int ci = 0x7FFFFFFF;
          int ncand = 0;
          float below = 0.f;                      // largest value below the interval
#pragma unroll
          for (int t = 0; t < TPL; ++t) {
            const uint32_t key = __float_as_uint(p[t]);
            const bool valid = lane + 32 * t < nb;
            const bool in = valid && key >= lo && key < hi;
            if (valid && key < lo) below = fmaxf(below, p[t]);
            uint32_t bal = __ballot_sync(0xffffffffu, in);
            while (bal != 0u) {                   // warp-uniform
              const int src = __ffs(bal) - 1;
              bal &= bal - 1u;
              const uint32_t kv = __shfl_sync(0xffffffffu, key, src);
              if (lane == ncand) {
                ck = kv;
                ci = src + 32 * t;
              }
              ++ncand;
            }
          }
          below = warp_max(below);
          // rank and exclusive mass of each candidate (lanes 0..ncand-1)
          int rank = 0;
          for (int d = 0; d < ncand; ++d) {
            const uint32_t kd = __shfl_sync(0xffffffffu, ck, d);
            const int id = __shfl_sync(0xffffffffu, ci, d);
            rank += (lane < ncand && (kd > ck || (kd == ck && id < ci))) ? 1 : 0;
          }
          float e = mass_hi;
          for (int d = 0; d < ncand; ++d) {
            const int rd = __shfl_sync(0xffffffffu, rank, d);
            const float pd = __uint_as_float(__shfl_sync(0xffffffffu, ck, d));
            if (lane < ncand && rd < rank) e += pd;
          }
          // the cut: the candidate whose exclusive mass is below thr and inclusive mass
          // reaches it
          const float pc = __uint_as_float(ck);
          const bool is_cut = lane < ncand && e < thr && e + pc >= thr;
          const uint32_t cb = __ballot_sync(0xffffffffu, is_cut);
          if (cb != 0u) {
            const int cl = __ffs(cb) - 1;
            const int crank = __shfl_sync(0xffffffffu, rank, cl);
            const float e_above = __shfl_sync(0xffffffffu, e, cl);
            const float p_cut = __uint_as_float(__shfl_sync(0xffffffffu, ck, cl));
            // next value below the cut: the candidate ranked right after it, else the
            // largest value below the interval
            float p_next = below;
            int n_at = 0;
            for (int d = 0; d < ncand; ++d) {
              const int rd = __shfl_sync(0xffffffffu, rank, d);
              const float pd = __uint_as_float(__shfl_sync(0xffffffffu, ck, d));
              if (rd == crank + 1) p_next = pd;
              n_at += pd == p_cut ? 1 : 0;
            }
            kcut = __float_as_uint(p_cut);
            certified = certify(e_above, e_above + p_cut, p_cut, p_next, n_at);
          }
        }
      }
    }
  }
  if (!certified) {
    if (lane == 0) {
      const int pos = atomicAdd(&prm.rescue_cnt[bh], 1);
      prm.rescue_list[bh * nb + pos] = i;
    }
    return;
  }
  // Emit: keep P >= P_c, OR the static window.
  const int ti = i / (prm.Hb * prm.Wb), hi_ = (i / prm.Wb) % prm.Hb, wi = i % prm.Wb;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int run = 0;
  uint32_t word[(TPL + 31) / 32];                     // lane l keeps bitmask word l + 32 w
#pragma unroll
  for (int w = 0; w < (TPL + 31) / 32; ++w) word[w] = 0u;
#pragma unroll
  for (int t = 0; t < TPL; ++t) {
    if (t >= prm.nw) break;
    const int j = lane + 32 * t;
    bool k = (j < nb) && (__float_as_uint(p[t]) >= kcut);
    if (prm.sta_on && j < nb) {
      const int tj = j / (prm.Hb * prm.Wb), hj = (j / prm.Wb) % prm.Hb, wj = j % prm.Wb;
      k = k || (abs(ti - tj) <= prm.wt2 && abs(hi_ - hj) <= prm.wh2 && abs(wi - wj) <= prm.ww2);
    }
    const uint32_t kb = __ballot_sync(0xffffffffu, k);
    if (lane == (t & 31)) word[t >> 5] = kb;
    if (prm.row_idx != nullptr && k) prm.row_idx[(bh * nb + i) * static_cast<long long>(nb) + run + __popc(kb & lt_mask)] = j;
    run += __popc(kb);
  }
  // the row's bitmask words in one coalesced store
  uint32_t* brow = prm.bits + (bh * nb + i) * prm.nw;
#pragma unroll
  for (int w = 0; w < (TPL + 31) / 32; ++w)
    if (lane + 32 * w < prm.nw) brow[lane + 32 * w] = word[w];
  if (prm.row_cnt != nullptr && lane == 0) prm.row_cnt[bh * nb + i] = run;
}

template <int TPL>
cudaError_t launch_select(const SelectParams& p, long long rows, cudaStream_t st) {
  mask_select_kernel<TPL><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(p, rows);
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

// Tiers 1-2a: split of the pooled means and the pooled logits (independent of thr).
cudaError_t mask_fast_prepare(const double* qp, const double* kp, const Dims& d, double scale,
                              void* scratch, uint32_t* status, cudaStream_t st) {
  const int nbp = mask_fast_nbp(d.nb);
  const FastScratch f = fast_scratch(d, scratch);
  cudaError_t e = cudaMemsetAsync(f.kmax, 0, static_cast<size_t>(d.BH) * 4, st);
  if (e != cudaSuccess) return e;
  const long long rows_pad = static_cast<long long>(d.BH) * nbp;
  if (d.D == 64)
    split_pools_kernel<64><<<static_cast<unsigned>((rows_pad + 7) / 8), 256, 0, st>>>(
        qp, kp, d.nb, nbp, rows_pad, f.qh, f.ql, f.kh, f.kl, f.qnorm, f.kmax);
  else
    split_pools_kernel<128><<<static_cast<unsigned>((rows_pad + 7) / 8), 256, 0, st>>>(
        qp, kp, d.nb, nbp, rows_pad, f.qh, f.ql, f.kh, f.kl, f.qnorm, f.kmax);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  CUtensorMap mqh, mql, mkh, mkl;
  if (!(make_map_16(&mqh, f.qh, rows_pad, d.D, 128, true) && make_map_16(&mql, f.ql, rows_pad, d.D, 128, true) &&
        make_map_16(&mkh, f.kh, rows_pad, d.D, 256, true) && make_map_16(&mkl, f.kl, rows_pad, d.D, 256, true)))
    return cudaErrorInvalidValue;
  dim3 grid(nbp / 128, nbp / 256, d.BH);
  if (d.D == 64) {
    e = cudaFuncSetAttribute(pooled_logits_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             LogitCfg<64>::kSmemBytes);
    if (e != cudaSuccess) return e;
    pooled_logits_kernel<64><<<grid, 128, LogitCfg<64>::kSmemBytes, st>>>(
        mqh, mql, mkh, mkl, f.logits, nbp, static_cast<float>(scale), status);
  } else {
    e = cudaFuncSetAttribute(pooled_logits_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             LogitCfg<128>::kSmemBytes);
    if (e != cudaSuccess) return e;
    pooled_logits_kernel<128><<<grid, 128, LogitCfg<128>::kSmemBytes, st>>>(
        mqh, mql, mkh, mkl, f.logits, nbp, static_cast<float>(scale), status);
  }
  return cudaGetLastError();
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
  const int tpl = nbp / 32;
  switch (tpl) {
    case 8: e = launch_select<8>(p, rows, st); break;
    case 16: e = launch_select<16>(p, rows, st); break;
    case 24: e = launch_select<24>(p, rows, st); break;
    case 32: e = launch_select<32>(p, rows, st); break;
    case 40: e = launch_select<40>(p, rows, st); break;
    case 48: e = launch_select<48>(p, rows, st); break;
    case 56: e = launch_select<56>(p, rows, st); break;
    default: e = launch_select<64>(p, rows, st); break;
  }
  *rescue_list = f.rlist;
  *rescue_cnt = f.rc;
  return e;
}

// Runs tiers 1-2 (split, logits, certified select) for one thr.
cudaError_t mask_fast_run(const double* qp, const double* kp, const Dims& d, double scale, double thr,
                          const nabla_window& w, uint32_t* bits, int32_t* ridx, int32_t* rcnt,
                          void* scratch, uint32_t* status, int32_t** rescue_list,
                          int32_t** rescue_cnt, cudaStream_t st) {
  cudaError_t e = mask_fast_prepare(qp, kp, d, scale, scratch, status, st);
  if (e != cudaSuccess) return e;
  return mask_fast_select(d, scale, thr, w, bits, ridx, rcnt, scratch, rescue_list, rescue_cnt, st);
}

}  // namespace nabla
