// Block-sparse flash-attention forward over the kept 64 x 64 tiles (sm_100a).
//
// "NABLA: Neighborhood Adaptive Block-Level Attention" (gist.science, Chinese edition),
// technical summary, Methodology, "expansion": each kept entry (i, j) of the pooled
// block mask is one full N x N tile of the token attention matrix, computed exactly;
// the pages run this through FlexAttention.  Here it is a hand-written kernel:
//
//  * work tile = 128 query rows = two consecutive query blocks (2p, 2p+1) of one head
//    (M = 128 MMAs).  The tile walks the ascending union of the two blocks' kept key
//    blocks, read from the mask bitmask, two key blocks per step (N = 128 keys per
//    MMA); a half of the rows whose block does not keep a key block is masked (-inf);
//  * persistent: one CTA per SM takes tiles in a head-major, longest-first order through
//    an atomic counter; Q is double-buffered so the next tile's Q and first K/V tiles
//    load while the current tile finishes;
//  * warp 0 streams K and V with TMA (128-byte swizzle) through a ring of stages of two
//    key blocks each; warp 1 (one lane) issues tcgen05.mma: S = Q K^T (128 x 128) into
//    one of two TMEM score buffers, one step of look-ahead, and O += P V with P read
//    from TMEM;
//  * two softmax warpgroups (warps 4-7, 8-11) take alternate steps of the same tile, each
//    with its own score buffer, running max / sum and TMEM accumulator, one query row per
//    thread (TMEM lane = row).  Exponentials run on the MUFU unit with a quarter on the
//    FMA pipe (polynomial); P is rounded to the V operand's 16-bit type and the row sum
//    takes the rounded weights; O is rescaled only when a row maximum grows by more than
//    2^8.  The epilogue merges the two partial results (m, l, O);
//  * every barrier wait is bounded; on a timeout a kernel records a status code, stops,
//    drains its own copies and MMAs and frees TMEM.
#include <math.h>

#include <cudaTypedefs.h>

#include "common.cuh"

namespace nabla {
namespace {

constexpr int kThreads = 512;             // 16 warps
constexpr int kSoftmaxWarp0 = 4;          // warps 4..7 = group 0, 8..11 = group 1
constexpr int kEpilogueWarp0 = 12;        // warps 12..15
constexpr int kMaxWords = 512;            // bitmask words per row (nb <= 16384)

template <int D>
struct FwdCfg {
  static constexpr int kPanels = D / 64;                  // 128-byte swizzle panels
  static constexpr int kQBytes = 128 * D * 2;             // 128 rows
  static constexpr int kPairBytes = 128 * D * 2;          // two K (or V) blocks, 128 rows
  static constexpr int kStageBytes = 2 * kPairBytes;      // K pair + V pair
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kOffQ = 0;                         // two Q buffers
  static constexpr int kOffStage = kOffQ + 2 * kQBytes;
  static constexpr int kOffWords = kOffStage + kStages * kStageBytes;   // [2 tiles][2 rows][kMaxWords]
  static constexpr int kOffML = kOffWords + 2 * 2 * kMaxWords * 4;     // m, l: [2 tiles][2 groups][128]
  static constexpr int kOffBar = kOffML + 2 * 2 * 2 * 128 * 4;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
};

struct FwdParams {
  const int32_t* order;      // work items (head * npairs + pair)
  int items;
  int npairs;
  const uint32_t* bits;      // [B*H, nb, nw]
  int nw;
  void* o;
  float* lse;
  uint32_t* status;          // word 0: status, word 1: work counter
  int nb;
  long long S;
  float scale_log2;
  int o_f32;
};

// Walks the set bits of w0 | w1 (two rows' bitmask words in shared memory) in ascending
// order; f = bit0: kept by the first row, bit1: kept by the second.
struct BitWalk {
  const uint32_t* w0;
  const uint32_t* w1;
  int nw, w;
  uint32_t cur;
  __device__ void init(const uint32_t* a, const uint32_t* b, int n) {
    w0 = a; w1 = b; nw = n; w = 0; cur = n > 0 ? (a[0] | b[0]) : 0u;
  }
  __device__ int next(uint32_t* f) {
    while (cur == 0u) {
      if (++w >= nw) return -1;
      cur = w0[w] | w1[w];
    }
    const int bit = __ffs(cur) - 1;
    cur &= cur - 1u;
    *f = ((w0[w] >> bit) & 1u) | (((w1[w] >> bit) & 1u) << 1);
    return 32 * w + bit;
  }
};

// Roles (one CTA per SM, tiles taken in turn; tile t uses buffer set qb = t & 1):
//   warp 2      tile loader: takes the next tile, copies its two bitmask rows to shared
//               memory, counts the union and loads Q (q_full[qb]);
//   warp 0      K/V streamer: walks the union two key blocks per step into the stages;
//   warp 1      MMA issuer;
//   warps 4-11  two softmax groups on alternate steps; at the end of a tile each writes
//               its running (max, sum) and moves on (ml_ready[qb]);
//   warps 12-15 epilogue: merges the two groups' accumulators and stores O and LSE,
//               then frees the accumulators and the tile's buffer set (o_free[qb]).
template <int D, bool VF16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const FwdParams prm) {
  using C = FwdCfg<D>;
  constexpr int NST = C::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sStage = smem + C::kOffStage;
  uint32_t* sWords = reinterpret_cast<uint32_t*>(smem + C::kOffWords);
  float* ml = reinterpret_cast<float*>(smem + C::kOffML);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;                 // [NST]
  uint64_t* empty = full + NST;          // [NST]
  uint64_t* q_full = empty + NST;        // [2] loader -> all
  uint64_t* q_empty = q_full + 2;        // [2] MMA: Q buffer no longer read
  uint64_t* s_full = q_empty + 2;        // [2] per softmax group
  uint64_t* p_full = s_full + 2;         // [2] per softmax group
  uint64_t* tile_done = p_full + 2;      // [2] MMA: the tile's last PV landed
  uint64_t* ml_ready = tile_done + 2;    // [2] softmax groups -> epilogue
  uint64_t* o_free = ml_ready + 2;       // [2] epilogue: accumulators read, tile retired
  uint64_t* drain = o_free + 2;
  int32_t* qmeta = reinterpret_cast<int32_t*>(drain + 1);    // [2][2]: item, steps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qmeta + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nb = prm.nb;
  const int nw = prm.nw;
  uint32_t* status = prm.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
      mbar_init(&tile_done[b], 1);
      mbar_init(&ml_ready[b], 256);
      mbar_init(&o_free[b], 128);
    }
    mbar_init(drain, 1);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 2) {
    // ------------------------------------------------------------------ tile loader
    if (lane == 0) tma_prefetch_desc(&map_q);
    for (int tc = 0;; ++tc) {
      const int qb = tc & 1;
      int slot = 0;
      bool ok = true;
      if (lane == 0) {
        if (tc >= 2) {
          const uint32_t par = ((tc - 2) >> 1) & 1;
          ok = mbar_wait(&q_empty[qb], par, status, kDevTimeoutQFull) &&
               mbar_wait(&o_free[qb], par, status, kDevTimeoutOBar);
        }
        slot = ok ? atomicAdd(status + 1, 1) : prm.items;
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      slot = __shfl_sync(0xffffffffu, slot, 0);
      if (!ok) break;
      if (slot >= prm.items) {
        if (lane == 0) {
          qmeta[2 * qb] = -1;
          qmeta[2 * qb + 1] = 0;
          mbar_arrive(&q_full[qb]);
        }
        break;
      }
      const int item = prm.order[slot];
      const long long bh = item / prm.npairs;
      const int i0 = 2 * (item - static_cast<int>(bh) * prm.npairs);
      const bool has_i1 = i0 + 1 < nb;
      uint32_t* u0 = sWords + (qb * 2) * kMaxWords;
      uint32_t* u1 = u0 + kMaxWords;
      const uint32_t* r0 = prm.bits + (bh * nb + i0) * static_cast<long long>(nw);
      int cnt = 0;
      for (int w = lane; w < nw; w += 32) {
        uint32_t a = r0[w];
        uint32_t b = has_i1 ? r0[nw + w] : 0u;
        if (w == nw - 1 && (nb & 31)) {
          a &= (1u << (nb & 31)) - 1u;
          b &= (1u << (nb & 31)) - 1u;
        }
        u0[w] = a;
        u1[w] = b;
        cnt += __popc(a | b);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      __syncwarp();
      if (lane == 0) {
        qmeta[2 * qb] = item;
        qmeta[2 * qb + 1] = (cnt + 1) >> 1;
        mbar_arrive_expect_tx(&q_full[qb], C::kQBytes);
        const int qrow = static_cast<int>(bh * prm.S + static_cast<long long>(i0) * 64);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_2d(sQ + qb * C::kQBytes + pn * 16384, &map_q, &q_full[qb], pn * 64, qrow);
      }
      __syncwarp();
    }
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------------ K/V streamer
    if (lane == 0) {
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      long long g = 0;   // global stage counter
      bool ok = true;
      for (int tc = 0; ok; ++tc) {
        const int qb = tc & 1;
        if (!mbar_wait(&q_full[qb], (tc >> 1) & 1, status, kDevTimeoutQFull)) break;
        const int item = qmeta[2 * qb];
        const int steps = qmeta[2 * qb + 1];
        if (item < 0) break;
        const long long bh = item / prm.npairs;
        BitWalk wk;
        wk.init(sWords + (qb * 2) * kMaxWords, sWords + (qb * 2 + 1) * kMaxWords, nw);
        for (int k = 0; k < steps; ++k, ++g) {
          uint32_t fa = 0, fb = 0;
          const int ja = wk.next(&fa);
          int jb = wk.next(&fb);
          if (jb < 0) { jb = ja; fb = 0; }          // odd tail: a masked duplicate
          const int s = static_cast<int>(g % NST);
          const long long r = g / NST;
          if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1, status, kDevTimeoutKvEmpty)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], C::kStageBytes);
          unsigned char* kp = sStage + s * C::kStageBytes;
          unsigned char* vp = kp + C::kPairBytes;
          const int ra = static_cast<int>(bh * prm.S + static_cast<long long>(ja) * 64);
          const int rb = static_cast<int>(bh * prm.S + static_cast<long long>(jb) * 64);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn) {
            tma_load_2d(kp + pn * 16384, &map_k, &full[s], pn * 64, ra);
            tma_load_2d(kp + pn * 16384 + 8192, &map_k, &full[s], pn * 64, rb);
            tma_load_2d(vp + pn * 16384, &map_v, &full[s], pn * 64, ra);
            tma_load_2d(vp + pn * 16384 + 8192, &map_v, &full[s], pn * 64, rb);
          }
        }
      }
      // Drain: copies still in flight must land before the CTA exits.
      for (long long x = g > NST ? g - NST : 0; x < g; ++x)
        mbar_wait(&full[x % NST], (x / NST) & 1, status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = VF16 ? idesc_f16_f32(128, D, false, true)
                                        : idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t st_addr = smem_u32(sStage);
      long long g = 0;
      int pcount[2] = {0, 0};
      bool ok = true;
      auto issue_s = [&](int qb, long long gs, int b) {
        const uint32_t kp = st_addr + static_cast<uint32_t>(gs % NST) * C::kStageBytes;
        const uint32_t d_tmem = tmem + (b ? C::kColS1 : C::kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2, w = kk & 3;
          const uint64_t ad = sdesc_sw128(q_addr + qb * C::kQBytes + pn * 16384 + w * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(kp + pn * 16384 + w * 32, 16, 1024);
          mma_bf16_ss(d_tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[b]);
      };
      for (int tc = 0; ok; ++tc) {
        const int qb = tc & 1;
        if (!mbar_wait(&q_full[qb], (tc >> 1) & 1, status, kDevTimeoutQFull)) break;
        const int item = qmeta[2 * qb];
        const int n = qmeta[2 * qb + 1];
        if (item < 0) break;
        tc_fence_after();
        if (n > 0) {
          if (!mbar_wait(&full[g % NST], (g / NST) & 1, status, kDevTimeoutTmaFull)) break;
          tc_fence_after();
          issue_s(qb, g, 0);
          for (int k = 0; k < n; ++k) {
            if (k + 1 < n) {
              const long long g1 = g + k + 1;
              if (!mbar_wait(&full[g1 % NST], (g1 / NST) & 1, status, kDevTimeoutTmaFull)) { ok = false; break; }
              tc_fence_after();
              issue_s(qb, g1, (k + 1) & 1);
            }
            if (k == 0 && tc > 0) {
              // The accumulators hold an earlier tile until its epilogue frees them; the
              // epilogue retires tiles in order, so waiting for the previous tile suffices
              // (its buffer set's previous use was retired before this tile was loaded).
              const int pb = (tc - 1) & 1;
              if (!mbar_wait(&o_free[pb], ((tc - 1) >> 1) & 1, status, kDevTimeoutOBar)) { ok = false; break; }
              tc_fence_after();
            }
            const int b = k & 1;
            if (!mbar_wait(&p_full[b], pcount[b] & 1, status, kDevTimeoutPFull)) { ok = false; break; }
            ++pcount[b];
            tc_fence_after();
            // O_b += P V: P (16-bit, 128 keys) in the first 64 columns of score buffer b,
            // V pair MN-major (panel stride 16 KB along D, 8-row groups 1 KB apart).
            const long long gk = g + k;
            const int st = static_cast<int>(gk % NST);
            const uint32_t vp = st_addr + static_cast<uint32_t>(st) * C::kStageBytes + C::kPairBytes;
            const uint32_t p_tmem = tmem + (b ? C::kColS1 : C::kColS0);
            const uint32_t o_tmem = tmem + (b ? C::kColO1 : C::kColO0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t bd = sdesc_sw128(vp + kk * 2048, 16384, 1024);
              mma_bf16_ts(o_tmem, p_tmem + kk * 8, bd, idesc_o, (k >= 2 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&empty[st]);
          }
          if (!ok) break;
          g += n;
        }
        mma_commit(&q_empty[qb]);
        mma_commit(&tile_done[qb]);
      }
      mma_commit(drain);
      mbar_wait(drain, 0, status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp >= kSoftmaxWarp0 && warp < kEpilogueWarp0) {
    // ------------------------------------------------------------------ softmax groups
    const int grp = (warp - kSoftmaxWarp0) >> 2;                  // 0 or 1
    const int row = ((warp - kSoftmaxWarp0) & 3) * 32 + lane;      // 0..127 = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(((warp - kSoftmaxWarp0) & 3) * 32) << 16;
    const bool upper = row >= 64;
    const float sl2 = prm.scale_log2;
    const uint32_t s_col = tmem + lane_base + (grp ? C::kColS1 : C::kColS0);
    int my_iter = 0;
    bool ok = true;
    for (int tc = 0; ok; ++tc) {
      const int qb = tc & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&q_full[qb], (tc >> 1) & 1, status, kDevTimeoutQFull));
      if (!ok) break;
      const int item = qmeta[2 * qb];
      const int n = qmeta[2 * qb + 1];
      if (item < 0) break;
      float m_ref = -INFINITY;
      float l = 0.f;
      // The step's key blocks and flags come from the tile's bitmask words (stable in
      // shared memory for the whole tile), walked the same way as the K/V streamer does;
      // the group then waits only on its own score buffer, never on a K/V stage whose
      // previous phase it has not observed.
      BitWalk wk;
      wk.init(sWords + (qb * 2) * kMaxWords, sWords + (qb * 2 + 1) * kMaxWords, nw);
      for (int k = 0; k < n; ++k) {
        uint32_t fa = 0, fb = 0;
        wk.next(&fa);
        if (wk.next(&fb) < 0) fb = 0;
        if ((k & 1) != grp) continue;
        const bool keep_a = upper ? (fa >> 1) : (fa & 1u);
        const bool keep_b = upper ? (fb >> 1) : (fb & 1u);
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[grp], my_iter & 1, status, kDevTimeoutSFull));
        if (!ok) break;
        ++my_iter;
        tc_fence_after();
        // pass 1: row maximum over the kept half-rows
        float mx = -INFINITY;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h == 0 ? keep_a : keep_b) {
            uint32_t x[32], y[32];
            tmem_ld32(s_col + h * 64, x);
            tmem_ld32(s_col + h * 64 + 32, y);
            tmem_wait_ld();
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 32; ++c)
              m4[c & 3] = fmaxf(m4[c & 3], fmaxf(__uint_as_float(x[c]), __uint_as_float(y[c])));
            mx = fmaxf(mx, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
          }
        }
        const float rm = mx * sl2;
        float factor = 1.f;
        bool rescale = false;
        if ((keep_a || keep_b) && rm > m_ref + 8.0f) {
          if (m_ref != -INFINITY) {
            factor = fast_exp2(m_ref - rm);
            rescale = true;
          }
          m_ref = rm;
        }
        // The group's previous PV has completed (it was issued before this step's S), so
        // O can be rescaled in place; warp-uniform (tcgen05.ld/st are warp-collective).
        if (__any_sync(0xffffffffu, rescale)) {
          l *= factor;
          const uint32_t o_col = tmem + lane_base + (grp ? C::kColO1 : C::kColO0);
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t ov[32];
            tmem_ld32(o_col + c0, ov);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * factor);
            tmem_st32(o_col + c0, ov);
          }
          tmem_wait_st();
        }
        // pass 2: P = 2^(s*scale*log2e - m) as 16-bit pairs into the first 64 columns of the
        // score buffer (chunk c of 32 scores -> columns 16c..16c+15, already read).
        float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const bool kp = c < 2 ? keep_a : keep_b;
          uint32_t packed[16];
          if (kp) {
            uint32_t sv[32];
            tmem_ld32(s_col + c * 32, sv);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * e]), sl2, -m_ref));
              const float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * e + 1]), sl2, -m_ref));
              const float p2 = fast_exp2(fmaf(__uint_as_float(sv[2 * e + 2]), sl2, -m_ref));
              const float p3 = poly_exp2(fmaf(__uint_as_float(sv[2 * e + 3]), sl2, -m_ref));
              // The row sum takes the rounded weights that enter the PV product, so the
              // output is an exact convex combination of those weights.
              if constexpr (VF16) {
                packed[e] = pack_f16x2(p0, p1);
                packed[e + 1] = pack_f16x2(p2, p3);
                sum0 += f16lo(packed[e]) + f16hi(packed[e]);
                sum1 += f16lo(packed[e + 1]) + f16hi(packed[e + 1]);
              } else {
                packed[e] = pack_bf16x2(p0, p1);
                packed[e + 1] = pack_bf16x2(p2, p3);
                sum0 += bf16lo(packed[e]) + bf16hi(packed[e]);
                sum1 += bf16lo(packed[e + 1]) + bf16hi(packed[e + 1]);
              }
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) packed[e] = 0u;
          }
          tmem_st16(s_col + c * 16, packed);
        }
        l += sum0 + sum1;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[grp]);
      }
      if (!ok) break;
      // Hand the running (max, sum) to the epilogue and move on to the next tile.
      ml[(qb * 2 + grp) * 128 + row] = m_ref;
      ml[512 + (qb * 2 + grp) * 128 + row] = l;
      mbar_arrive(&ml_ready[qb]);
    }
  } else if (warp >= kEpilogueWarp0) {
    // ------------------------------------------------------------------ epilogue group
    const int row = (warp - kEpilogueWarp0) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((warp - kEpilogueWarp0) * 32) << 16;
    const bool upper = row >= 64;
    bool ok = true;
    for (int tc = 0; ok; ++tc) {
      const int qb = tc & 1;
      const uint32_t par = (tc >> 1) & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&q_full[qb], par, status, kDevTimeoutQFull));
      if (!ok) break;
      const int item = qmeta[2 * qb];
      const int n = qmeta[2 * qb + 1];
      if (item < 0) break;
      ok = __all_sync(0xffffffffu, mbar_wait(&tile_done[qb], par, status, kDevTimeoutOBar) &&
                                       mbar_wait(&ml_ready[qb], par, status, kDevTimeoutOBar));
      if (!ok) break;
      tc_fence_after();
      const float m0 = ml[(qb * 2) * 128 + row], m1 = ml[(qb * 2 + 1) * 128 + row];
      const float l0 = ml[512 + (qb * 2) * 128 + row], l1 = ml[512 + (qb * 2 + 1) * 128 + row];
      const float M = fmaxf(m0, m1);
      const float f0 = l0 > 0.f ? fast_exp2(m0 - M) : 0.f;
      const float f1 = l1 > 0.f ? fast_exp2(m1 - M) : 0.f;
      const float L = l0 * f0 + l1 * f1;
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const float w0 = f0 * inv, w1 = f1 * inv;
      const bool has0 = n > 0, has1 = n > 1;       // whether each group wrote O in this tile
      const long long bh = item / prm.npairs;
      const int i0 = 2 * (item - static_cast<int>(bh) * prm.npairs);
      const bool valid_row = upper ? (i0 + 1 < nb) : true;
      const long long tok = bh * prm.S + static_cast<long long>(i0) * 64 + row;
      const uint32_t o0 = tmem + lane_base + C::kColO0, o1 = tmem + lane_base + C::kColO1;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t a0[32], a1[32];
        if (has0) tmem_ld32(o0 + c0, a0);
        if (has1) tmem_ld32(o1 + c0, a1);
        tmem_wait_ld();
        float* v = reinterpret_cast<float*>(a0);   // merged in place
#pragma unroll
        for (int c = 0; c < 32; ++c)
          v[c] = (has0 ? __uint_as_float(a0[c]) * w0 : 0.f) + (has1 ? __uint_as_float(a1[c]) * w1 : 0.f);
        if (valid_row) {
          if (prm.o_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(prm.o) + tok * D + c0);
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.o) + tok * D + c0);
#pragma unroll
            for (int c = 0; c < 4; ++c)
              dst[c] = make_uint4(pack_bf16x2(v[8 * c], v[8 * c + 1]), pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                                  pack_bf16x2(v[8 * c + 4], v[8 * c + 5]), pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
          }
        }
      }
      if (valid_row && prm.lse != nullptr)
        prm.lse[tok] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      mbar_arrive(&o_free[qb]);
    }
  }
  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace

// ------------------------------------------------------------------------------------
// Tensor maps (host)
// ------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map of 16-bit elements (bf16, or fp16 when `fp16`) over [rows, D] (row stride
// D*2 bytes), box = 64 columns x box_rows rows, 128-byte swizzle, zero fill out of bounds.
bool make_map_16(CUtensorMap* map, const void* base, long long rows, int D, int box_rows,
                 bool fp16) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {
template <int D, bool VF16>
cudaError_t launch_fwd(const void* q, const void* k, const void* v, const Dims& d,
                       const FwdParams& prm, cudaStream_t st, bool* map_ok) {
  CUtensorMap mq, mk, mv;
  const long long rows = static_cast<long long>(d.BH) * d.S;
  *map_ok = make_map_16(&mq, q, rows, D, 128, false) && make_map_16(&mk, k, rows, D, 64, false) &&
            make_map_16(&mv, v, rows, D, 64, VF16);   // K / V: one 64-row block per copy
  if (!*map_ok) return cudaErrorInvalidValue;
  using C = FwdCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, VF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = prm.items < sms ? prm.items : sms;
  attn_fwd_kernel<D, VF16><<<grid, kThreads, C::kSmemBytes, st>>>(mq, mk, mv, prm);
  return cudaGetLastError();
}
}  // namespace

}  // namespace nabla

using namespace nabla;

extern "C" size_t nabla_fwd_workspace_bytes(nabla_shape s) {
  Dims d;
  if (check_shape(s, &d) != NABLA_OK) return 0;
  return kStatusBytes + schedule_scratch_bytes(d);
}

extern "C" nabla_status nabla_attn_fwd(const void* q, const void* k, const void* v,
                                       nabla_dtype v_dtype, const uint32_t* mask_bits,
                                       nabla_shape s, float scale, void* o, nabla_dtype o_dtype,
                                       float* lse, void* workspace, size_t workspace_bytes,
                                       nabla_stream_t stream) {
  Dims d;
  nabla_status rc = check_shape(s, &d);
  if (rc != NABLA_OK) return rc;
  if (!q || !k || !v || !o || !mask_bits) return NABLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return NABLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(mask_bits) & 3) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
    return NABLA_ERR_INVALID_ARG;
  if (o_dtype != NABLA_BF16 && o_dtype != NABLA_F32) return NABLA_ERR_INVALID_ARG;
  if (v_dtype != NABLA_BF16 && v_dtype != NABLA_F16) return NABLA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return NABLA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < nabla_fwd_workspace_bytes(s) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return NABLA_ERR_WORKSPACE;
  if (static_cast<long long>(d.BH) * d.S >= (1ll << 31)) return NABLA_ERR_UNSUPPORTED;
  FwdParams prm;
  prm.bits = mask_bits;
  prm.nw = d.nw;
  prm.o = o;
  prm.lse = lse;
  prm.status = static_cast<uint32_t*>(workspace);
  prm.nb = d.nb;
  prm.S = d.S;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.o_f32 = o_dtype == NABLA_F32;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t ce = cudaMemsetAsync(workspace, 0, kStatusBytes, st);
  if (ce != cudaSuccess) return cuda_status(ce);
  int32_t* order = nullptr;
  ce = build_schedule(nullptr, mask_bits, d, static_cast<char*>(workspace) + kStatusBytes, &order, st);
  if (ce != cudaSuccess) return cuda_status(ce);
  prm.order = order;
  prm.npairs = (d.nb + 1) / 2;
  prm.items = d.BH * prm.npairs;
  bool map_ok = true;
  const bool vf16 = v_dtype == NABLA_F16;
  cudaError_t e = d.D == 64 ? (vf16 ? launch_fwd<64, true>(q, k, v, d, prm, st, &map_ok)
                                    : launch_fwd<64, false>(q, k, v, d, prm, st, &map_ok))
                            : (vf16 ? launch_fwd<128, true>(q, k, v, d, prm, st, &map_ok)
                                    : launch_fwd<128, false>(q, k, v, d, prm, st, &map_ok));
  return cuda_status(e);
}
