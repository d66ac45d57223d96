// Block-sparse flash-attention forward over the kept 64 x 64 tiles (sm_100a).
//
// "NABLA: Neighborhood Adaptive Block-Level Attention" (gist.science, Chinese edition),
// technical summary, Methodology, "expansion": each kept entry (i, j) of the pooled
// block mask is one full N x N tile of the token attention matrix, computed exactly;
// the pages run this through FlexAttention.  Here it is a hand-written kernel:
//
//  * work tile = 128 query rows = two query blocks of one head (M = 128 MMAs): the same
//    patch in frames 2u and 2u + 1 (tile_blocks()).  The tile walks the ascending union
//    of the two blocks' kept key blocks, read from the mask bitmask, two key blocks per
//    step (N = 128 keys per MMA); a half of the rows whose block does not keep a key
//    block is masked (-inf);
//  * persistent: one CTA per SM takes tiles in a head-major, longest-first order through
//    an atomic counter.  A loader warp fetches tile descriptors into a ring several tiles
//    ahead; Q is double-buffered; K and V stream through separate rings, so a K stage is
//    refilled as soon as its S = Q K^T has run and does not wait for the softmax and P V;
//  * warp 1 (one lane) issues tcgen05.mma: S into one of two TMEM score buffers, one step
//    of look-ahead (into the next tile too), and O_g += P_g V_g with P read from TMEM;
//  * two softmax warpgroups (warps 4-7, 8-11) work on every step at once, group g on the
//    step's key block g (64 of the 128 score columns), each with its own running max /
//    sum and TMEM accumulator, one query row per thread (TMEM lane = row): two warps per
//    scheduler run the exponentials side by side.  Which group sums which key blocks
//    depends only on the tile, so results are bitwise reproducible whatever CTA runs it.
//    P is rounded to the V operand's 16-bit type and the row sum takes the rounded
//    weights; O is rescaled only when a row maximum grows by more than 2^8.  The
//    epilogue warpgroup merges the two partial results;
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
constexpr int kMetaRing = 4;              // tile descriptors fetched ahead
constexpr int kMetaInts = 8;              // item, bh, block a, block b, steps

template <int D>
struct FwdCfg {
  static constexpr int kPanels = D / 64;                  // 128-byte swizzle panels
  static constexpr int kQBytes = 128 * D * 2;             // 128 rows
  static constexpr int kPairBytes = 128 * D * 2;          // two K (or V) blocks, 128 rows
  static constexpr int kKStages = (D == 128) ? 2 : 4;
  static constexpr int kVStages = (D == 128) ? 2 : 4;
  static constexpr int kOffQ = 0;                         // two Q buffers
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffV = kOffK + kKStages * kPairBytes;
  static constexpr int kOffML = kOffV + kVStages * kPairBytes;   // m, l: [2 tiles][2 groups][128]
  static constexpr int kOffX = kOffML + 2 * 2 * 2 * 128 * 4;      // row max exchange [2][2][128]
  static constexpr int kOffMeta = kOffX + 2 * 2 * 128 * 4;
  static constexpr int kOffBar = kOffMeta + kMetaRing * kMetaInts * 4;
  static constexpr int kSmemBytes = kOffBar + 512 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  // two score buffers (by step parity), two accumulators (by tile parity)
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
};

struct FwdParams {
  const int32_t* order;      // work items (head * npairs + tile)
  int items;
  int npairs;
  const uint32_t* bits;      // [B*H, nb, nw]
  int nw;
  void* o;
  float* lse;
  uint32_t* status;          // word 0: status, word 1: work counter
  int nb;
  int T, HW;                 // frames, blocks per frame
  long long S;
  float scale_log2;
  int o_f32;
};

// Walks the set bits of rows a | b of the bitmask (global memory, read-only) in
// ascending order; f = bit0: kept by row a, bit1: kept by row b (b may be absent).
// Padding bits past nb are ignored.  Warp-cooperative (all 32 lanes call next() together
// and get the same answer): to reach the next non-empty word the lanes load 32 words at
// once and a ballot picks the first, so a run of empty words costs one round trip.
struct WarpBitWalk {
  const uint32_t* ra;
  const uint32_t* rb;
  int nw, w;
  uint32_t tail, a, b, cur;
  __device__ void init(const uint32_t* row_a, const uint32_t* row_b, int n_words, int nb) {
    ra = row_a; rb = row_b; nw = n_words; w = -1; cur = 0u; a = b = 0u;
    tail = (nb & 31) ? (1u << (nb & 31)) - 1u : ~0u;
  }
  __device__ int next(uint32_t* f) {
    while (cur == 0u) {
      const int base = w + 1;
      if (base >= nw) return -1;
      const int ww = base + static_cast<int>(threadIdx.x & 31);
      uint32_t xa = 0u, xb = 0u;
      if (ww < nw) {
        const uint32_t m = (ww == nw - 1) ? tail : ~0u;
        xa = __ldg(ra + ww) & m;
        xb = rb ? (__ldg(rb + ww) & m) : 0u;
      }
      const uint32_t nz = __ballot_sync(0xffffffffu, (xa | xb) != 0u);
      if (nz == 0u) {
        w = base + 31;
        continue;
      }
      const int src = __ffs(nz) - 1;
      w = base + src;
      a = __shfl_sync(0xffffffffu, xa, src);
      b = __shfl_sync(0xffffffffu, xb, src);
      cur = a | b;
    }
    const int bit = __ffs(cur) - 1;
    cur &= cur - 1u;
    *f = ((a >> bit) & 1u) | (((b >> bit) & 1u) << 1);
    return 32 * w + bit;
  }
};

struct TileMeta {
  int item, bh, ia, ib, n;
};

__device__ __forceinline__ TileMeta read_meta(const int32_t* m) {
  TileMeta t;
  t.item = m[0]; t.bh = m[1]; t.ia = m[2]; t.ib = m[3]; t.n = m[4];
  return t;
}

// Roles (one CTA per SM, tiles taken in turn; tile c uses descriptor slot c % kMetaRing
// and Q / (m, l) buffer c & 1):
//   warp 2      tile loader: takes the next tile, counts the union of its two bitmask rows
//               and publishes its descriptor (meta_full);
//   warp 3      Q loader: loads the tile's two Q blocks (q_full);
//   warp 0      K/V streamer: walks the union two key blocks per step; V one step behind K;
//   warp 1      MMA issuer;
//   warps 4-11  two softmax groups, one per key block of each step; at the end of a tile
//               each writes its running (max, sum) and moves on (ml_ready);
//   warps 12-15 epilogue: merges the two groups' accumulators and stores O and LSE,
//               then frees the accumulators (o_free) and the descriptor (meta_empty).
template <int D, bool VF16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const FwdParams prm) {
  using C = FwdCfg<D>;
  constexpr int NK = C::kKStages;
  constexpr int NV = C::kVStages;
  constexpr int R = kMetaRing;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sK = smem + C::kOffK;
  unsigned char* sV = smem + C::kOffV;
  float* ml = reinterpret_cast<float*>(smem + C::kOffML);
  float* xmax = reinterpret_cast<float*>(smem + C::kOffX);
  int32_t* meta = reinterpret_cast<int32_t*>(smem + C::kOffMeta);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* k_full = bars;               // [NK]
  uint64_t* k_empty = k_full + NK;       // [NK]
  uint64_t* v_full = k_empty + NK;       // [NV]
  uint64_t* v_empty = v_full + NV;       // [NV]
  uint64_t* meta_full = v_empty + NV;    // [R] tile loader -> all
  uint64_t* meta_empty = meta_full + R;  // [R] epilogue -> tile loader
  uint64_t* q_full = meta_empty + R;     // [2] Q loader -> MMA
  uint64_t* q_empty = q_full + 2;        // [2] MMA: the tile's last S has read Q
  uint64_t* s_full = q_empty + 2;        // [2] per softmax group
  uint64_t* p_full = s_full + 2;         // [2] per softmax group
  uint64_t* tile_done = p_full + 2;      // [2] MMA: the tile's last PV landed
  uint64_t* ml_ready = tile_done + 2;    // [2] softmax groups -> epilogue
  uint64_t* o_free = ml_ready + 2;       // [2] epilogue: accumulators read, tile retired
  uint64_t* pv_done = o_free + 2;        // [2] MMA: the step's P V landed (per score buffer)
  uint64_t* xbar = pv_done + 2;          // [4 warp pairs][2] softmax row max exchange
  uint64_t* drain = xbar + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nb = prm.nb;
  const int nw = prm.nw;
  uint32_t* status = prm.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int r = 0; r < R; ++r) {
      mbar_init(&meta_full[r], 1);
      mbar_init(&meta_empty[r], 128);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 256);
      mbar_init(&tile_done[b], 1);
      mbar_init(&ml_ready[b], 256);
      mbar_init(&o_free[b], 128);
      mbar_init(&pv_done[b], 1);
      for (int i = 0; i < 4; ++i) mbar_init(&xbar[i * 2 + b], 2);
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

  if (warp < 4) {
    if (warp == 2) {
      // ------------------------------------------------------------------ tile loader
      for (int c = 0;; ++c) {
        const int r = c % R;
        int32_t* mt = meta + r * kMetaInts;
        int slot = 0;
        bool ok = true;
        if (lane == 0) {
          if (c >= R) ok = mbar_wait(&meta_empty[r], ((c / R) - 1) & 1, status, kDevTimeoutMeta);
          slot = ok ? atomicAdd(status + 1, 1) : prm.items;
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        slot = __shfl_sync(0xffffffffu, slot, 0);
        if (!ok) break;
        if (slot >= prm.items) {
          if (lane == 0) {
            mt[0] = -1;
            mt[4] = 0;
            mbar_arrive(&meta_full[r]);
          }
          break;
        }
        const int item = prm.order[slot];
        const int bh = item / prm.npairs;
        const int2 ab = tile_blocks(item - bh * prm.npairs, prm.T, prm.HW, nb);
        const uint32_t* ra = prm.bits + (static_cast<long long>(bh) * nb + ab.x) * nw;
        const uint32_t* rb = ab.y >= 0 ? prm.bits + (static_cast<long long>(bh) * nb + ab.y) * nw : nullptr;
        int cnt = 0;
        for (int w = lane; w < nw; w += 32) {
          uint32_t u = __ldg(ra + w) | (rb ? __ldg(rb + w) : 0u);
          if (w == nw - 1 && (nb & 31)) u &= (1u << (nb & 31)) - 1u;
          cnt += __popc(u);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
        if (lane == 0) {
          mt[0] = item;
          mt[1] = bh;
          mt[2] = ab.x;
          mt[3] = ab.y;
          mt[4] = (cnt + 1) >> 1;
          mbar_arrive(&meta_full[r]);
        }
        __syncwarp();
      }
      __syncwarp();
    } else if (warp == 3) {
      // ------------------------------------------------------------------ Q loader
      if (lane == 0) {
        tma_prefetch_desc(&map_q);
        for (int c = 0;; ++c) {
          const int qb = c & 1;
          if (!mbar_wait(&meta_full[c % R], (c / R) & 1, status, kDevTimeoutMeta)) break;
          const TileMeta t = read_meta(meta + (c % R) * kMetaInts);
          if (t.item < 0) break;
          if (c >= 2 && !mbar_wait(&q_empty[qb], ((c - 2) >> 1) & 1, status, kDevTimeoutQFull)) break;
          mbar_arrive_expect_tx(&q_full[qb], C::kQBytes);
          const int rowa = static_cast<int>(t.bh * prm.S + static_cast<long long>(t.ia) * 64);
          const int rowb = static_cast<int>(t.bh * prm.S + static_cast<long long>(t.ib >= 0 ? t.ib : t.ia) * 64);
          unsigned char* qd = sQ + qb * C::kQBytes;
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn) {
            tma_load_2d(qd + pn * 16384, &map_q, &q_full[qb], pn * 64, rowa);
            tma_load_2d(qd + pn * 16384 + 8192, &map_q, &q_full[qb], pn * 64, rowb);
          }
        }
      }
      __syncwarp();
    } else if (warp == 0) {
      // ------------------------------------------------------------------ K/V streamer
      // The whole warp walks the bitmask and waits; lane 0 issues the copies.
      if (lane == 0) {
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
      }
      long long gk = 0, gv = 0;   // K pairs and V pairs issued (one pair per step)
      int pva = -1, pvb = -1;     // rows of the V pair still to issue (step gk - 1)
      bool ok = true;
      auto wait_all = [&](uint64_t* bar, uint32_t parity, uint32_t code) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, status, code));
      };
      auto load_v = [&](int ra, int rb) -> bool {
        const int s = static_cast<int>(gv % NV);
        const long long r = gv / NV;
        if (r > 0 && !wait_all(&v_empty[s], (r - 1) & 1, kDevTimeoutKvEmpty)) return false;
        if (lane == 0) {
          mbar_arrive_expect_tx(&v_full[s], C::kPairBytes);
          unsigned char* vp = sV + s * C::kPairBytes;
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn) {
            tma_load_2d(vp + pn * 16384, &map_v, &v_full[s], pn * 64, ra);
            tma_load_2d(vp + pn * 16384 + 8192, &map_v, &v_full[s], pn * 64, rb);
          }
        }
        __syncwarp();
        ++gv;
        return true;
      };
      for (int c = 0; ok; ++c) {
        if (!wait_all(&meta_full[c % R], (c / R) & 1, kDevTimeoutMeta)) break;
        const TileMeta t = read_meta(meta + (c % R) * kMetaInts);
        if (t.item < 0) break;
        WarpBitWalk wk;
        wk.init(prm.bits + (static_cast<long long>(t.bh) * nb + t.ia) * nw,
                t.ib >= 0 ? prm.bits + (static_cast<long long>(t.bh) * nb + t.ib) * nw : nullptr, nw, nb);
        for (int k = 0; k < t.n; ++k) {
          uint32_t fa = 0, fb = 0;
          const int ja = wk.next(&fa);
          int jb = wk.next(&fb);
          if (jb < 0) jb = ja;                      // odd tail: a masked duplicate
          const int ra = static_cast<int>(t.bh * prm.S + static_cast<long long>(ja) * 64);
          const int rb = static_cast<int>(t.bh * prm.S + static_cast<long long>(jb) * 64);
          const int s = static_cast<int>(gk % NK);
          const long long r = gk / NK;
          if (r > 0 && !wait_all(&k_empty[s], (r - 1) & 1, kDevTimeoutKvEmpty)) { ok = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(&k_full[s], C::kPairBytes);
            unsigned char* kp = sK + s * C::kPairBytes;
#pragma unroll
            for (int pn = 0; pn < C::kPanels; ++pn) {
              tma_load_2d(kp + pn * 16384, &map_k, &k_full[s], pn * 64, ra);
              tma_load_2d(kp + pn * 16384 + 8192, &map_k, &k_full[s], pn * 64, rb);
            }
          }
          __syncwarp();
          ++gk;
          // V of the previous step: its stage frees later (after P V), so K runs first.
          if (pva >= 0 && !load_v(pva, pvb)) { ok = false; break; }
          pva = ra;
          pvb = rb;
        }
      }
      if (ok && pva >= 0) load_v(pva, pvb);
      // Drain: copies still in flight must land before the CTA exits.
      for (long long x = gk > NK ? gk - NK : 0; x < gk; ++x)
        mbar_wait(&k_full[x % NK], (x / NK) & 1, status, kDevTimeoutDrain);
      for (long long x = gv > NV ? gv - NV : 0; x < gv; ++x)
        mbar_wait(&v_full[x % NV], (x / NV) & 1, status, kDevTimeoutDrain);
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t idesc_o = VF16 ? idesc_f16_f32(128, D, false, true)
                                          : idesc_bf16_f32(128, D, false, true);
        const uint32_t q_addr = smem_u32(sQ);
        const uint32_t k_addr = smem_u32(sK);
        const uint32_t v_addr = smem_u32(sV);
        long long g = 0;             // global step of the tile's first step
        int pcount[2] = {0, 0};
        bool ok = true;
        bool s0_issued = false;      // S of the tile's first step issued by look-ahead
        // S for global step gs (K stage gs % NK) into score buffer sb from Q buffer qb.
        auto issue_s = [&](int qb, long long gs, int sb) -> bool {
          const int ks = static_cast<int>(gs % NK);
          if (!mbar_wait(&k_full[ks], (gs / NK) & 1, status, kDevTimeoutTmaFull)) return false;
          tc_fence_after();
          const uint32_t kp = k_addr + static_cast<uint32_t>(ks) * C::kPairBytes;
          const uint32_t d_tmem = tmem + (sb ? C::kColS1 : C::kColS0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int pn = kk >> 2, w = kk & 3;
            const uint64_t ad = sdesc_sw128(q_addr + qb * C::kQBytes + pn * 16384 + w * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(kp + pn * 16384 + w * 32, 16, 1024);
            mma_bf16_ss(d_tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&s_full[sb]);
          mma_commit(&k_empty[ks]);
          return true;
        };
        for (int c = 0; ok; ++c) {
          const int qb = c & 1;
          if (!mbar_wait(&meta_full[c % R], (c / R) & 1, status, kDevTimeoutMeta)) break;
          const TileMeta t = read_meta(meta + (c % R) * kMetaInts);
          if (t.item < 0) break;
          const int n = t.n;
          if (n == 0) {
            // Nothing to compute: release Q once it has landed; retire the tile once the
            // epilogue has retired tile c - 2 (so it sees tile_done phases one at a time).
            if (!mbar_wait(&q_full[qb], (c >> 1) & 1, status, kDevTimeoutQFull)) break;
            mma_commit(&q_empty[qb]);
            if (c >= 2 && !mbar_wait(&o_free[qb], ((c - 2) >> 1) & 1, status, kDevTimeoutOBar)) break;
            mma_commit(&tile_done[qb]);
            s0_issued = false;
            continue;
          }
          if (!s0_issued) {
            if (!mbar_wait(&q_full[qb], (c >> 1) & 1, status, kDevTimeoutQFull)) break;
            tc_fence_after();
            if (!issue_s(qb, g, static_cast<int>(g & 1))) break;
            if (n == 1) mma_commit(&q_empty[qb]);
          }
          s0_issued = false;
          for (int k = 0; k < n; ++k) {
            const long long gk = g + k;
            if (k + 1 < n) {
              if (!issue_s(qb, gk + 1, static_cast<int>((gk + 1) & 1))) { ok = false; break; }
              if (k + 2 == n) mma_commit(&q_empty[qb]);
            } else {
              // Look-ahead into the next tile: its first S goes to the other score buffer,
              // whose P (the step before) has been handed to its P V already.
              const int c1 = c + 1;
              if (!mbar_wait(&meta_full[c1 % R], (c1 / R) & 1, status, kDevTimeoutMeta)) { ok = false; break; }
              const TileMeta t1 = read_meta(meta + (c1 % R) * kMetaInts);
              if (t1.item >= 0 && t1.n > 0) {
                if (!mbar_wait(&q_full[c1 & 1], (c1 >> 1) & 1, status, kDevTimeoutQFull)) { ok = false; break; }
                tc_fence_after();
                if (!issue_s(c1 & 1, gk + 1, static_cast<int>((gk + 1) & 1))) { ok = false; break; }
                if (t1.n == 1) mma_commit(&q_empty[c1 & 1]);
                s0_issued = true;
              }
            }
            if (k == 0 && c >= 2) {
              // The accumulator of this tile parity holds tile c - 2 until its epilogue
              // frees it; tile c - 1 uses the other one.
              if (!mbar_wait(&o_free[qb], ((c - 2) >> 1) & 1, status, kDevTimeoutOBar)) { ok = false; break; }
              tc_fence_after();
            }
            const int b = static_cast<int>(gk & 1);
            if (!mbar_wait(&p_full[b], pcount[b] & 1, status, kDevTimeoutPFull)) { ok = false; break; }
            ++pcount[b];
            const int vs = static_cast<int>(gk % NV);
            if (!mbar_wait(&v_full[vs], (gk / NV) & 1, status, kDevTimeoutTmaFull)) { ok = false; break; }
            tc_fence_after();
            // O += P_a V_a + P_b V_b: each group's P (16-bit, 64 keys) in 32 columns of
            // score buffer b (group 0 at column 0, group 1 at column 64); the V pair
            // MN-major (panel stride 16 KB along D, 8-row groups 1 KB apart), block a in
            // keys 0-63, block b in keys 64-127.  O is the accumulator of this tile parity.
            const uint32_t vp = v_addr + static_cast<uint32_t>(vs) * C::kPairBytes;
            const uint32_t p_tmem = tmem + (b ? C::kColS1 : C::kColS0);
            const uint32_t o_tmem = tmem + (qb ? C::kColO1 : C::kColO0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t bd = sdesc_sw128(vp + kk * 2048, 16384, 1024);
              const uint32_t a_tmem = p_tmem + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8);
              mma_bf16_ts(o_tmem, a_tmem, bd, idesc_o, (k > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&v_empty[vs]);
            mma_commit(&pv_done[b]);
          }
          if (!ok) break;
          mma_commit(&tile_done[qb]);
          g += n;
        }
        mma_commit(drain);
        mbar_wait(drain, 0, status, kDevTimeoutDrain);
      }
      __syncwarp();
    }
  } else if (warp < kEpilogueWarp0) {
    // ------------------------------------------------------------------ softmax groups
    // Group grp takes key block grp of every step: score columns 64 grp .. 64 grp + 63 of
    // the step's buffer; its P goes to the first 32 of those columns (already read).
    const int grp = (warp - kSoftmaxWarp0) >> 2;                  // 0 or 1
    const int row = ((warp - kSoftmaxWarp0) & 3) * 32 + lane;      // 0..127 = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(((warp - kSoftmaxWarp0) & 3) * 32) << 16;
    const bool upper = row >= 64;
    const float sl2 = prm.scale_log2;
    const float2 sl2v = make_float2(sl2, sl2);
    const int pair = (warp - kSoftmaxWarp0) & 3;                   // warp pair sharing rows
    int scount[2] = {0, 0}, pvcount[2] = {0, 0}, xcount[2] = {0, 0};
    long long g = 0;             // global step of the tile's first step
    bool ok = true;
    for (int c = 0; ok; ++c) {
      const int qb = c & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&meta_full[c % R], (c / R) & 1, status, kDevTimeoutMeta));
      if (!ok) break;
      const TileMeta t = read_meta(meta + (c % R) * kMetaInts);
      if (t.item < 0) break;
      const int n = t.n;
      // This group rescales its half of the tile's accumulator columns.
      const uint32_t o_col = tmem + lane_base + (qb ? C::kColO1 : C::kColO0) + static_cast<uint32_t>(grp * (D / 2));
      float m_ref = -INFINITY;
      float l = 0.f;
      // The step's key blocks and flags come from the tile's bitmask rows, walked the same
      // way as the K/V streamer does.
      WarpBitWalk wk;
      wk.init(prm.bits + (static_cast<long long>(t.bh) * nb + t.ia) * nw,
              t.ib >= 0 ? prm.bits + (static_cast<long long>(t.bh) * nb + t.ib) * nw : nullptr, nw, nb);
      for (int k = 0; k < n; ++k) {
        uint32_t fa = 0, fb = 0;
        wk.next(&fa);
        if (wk.next(&fb) < 0) fb = 0;
        const uint32_t f = grp ? fb : fa;
        const bool keep = upper ? (f >> 1) : (f & 1u);   // warp-uniform
        const long long gk = g + k;
        const int b = static_cast<int>(gk & 1);
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], scount[b] & 1, status, kDevTimeoutSFull));
        if (!ok) break;
        ++scount[b];
        tc_fence_after();
        const uint32_t s_col = tmem + lane_base + (b ? C::kColS1 : C::kColS0) + static_cast<uint32_t>(grp * 64);
        // The row's 64 scores of this key block in registers: one TMEM round trip.
        uint32_t sv[64];
        uint32_t(&c0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t(&c1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        if (keep) {
          tmem_ld32(s_col, c0);
          tmem_ld32(s_col + 32, c1);
        }
        tmem_wait_ld();
        float lm = -INFINITY;
        if (keep) {
          reg_fence32(c0);
          reg_fence32(c1);
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int cc = 0; cc < 64; ++cc) m4[cc & 3] = fmaxf(m4[cc & 3], __uint_as_float(sv[cc]));
          lm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
        // Both groups accumulate into one O, so they share the row's reference maximum:
        // partner threads (same row) swap their block maxima through shared memory
        // (buffered by step parity) and take the same decisions.
        const int xb = static_cast<int>(gk & 1);
        xmax[(xb * 2 + grp) * 128 + row] = lm;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xbar[pair * 2 + xb]);
        ok = __all_sync(0xffffffffu, mbar_wait(&xbar[pair * 2 + xb], xcount[xb] & 1, status, kDevTimeoutSFull));
        if (!ok) break;
        ++xcount[xb];
        const float mx = fmaxf(lm, xmax[(xb * 2 + (grp ^ 1)) * 128 + row]);
        float factor = 1.f;
        bool rescale = false;
        if (mx != -INFINITY && mx * sl2 > m_ref + 8.0f) {
          const float rm = mx * sl2;
          if (m_ref != -INFINITY) {
            factor = fast_exp2(m_ref - rm);
            rescale = true;
          }
          m_ref = rm;
        }
        // P = 2^(s*scale*log2e - m) as 16-bit pairs (keys 2e, 2e+1 -> column e).
        const float2 negm = make_float2(-m_ref, -m_ref);
        float2 acc = make_float2(0.f, 0.f);
        if (keep) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float2 xa = __ffma2_rn(make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])),
                                         sl2v, negm);
            const float2 pr = make_float2(fast_exp2(xa.x), fast_exp2(xa.y));
            // The row sum takes the rounded weights that enter the PV product, so the
            // output is an exact convex combination of them.
            uint32_t pk;
            if constexpr (VF16) {
              // Non-negative fp16 halves widened exactly with integer ops: the fp16 bits
              // moved to f32 bits 13..27 read as the value times 2^-112 (fp16 subnormals
              // land on f32 subnormals); the sum is rescaled once below.
              pk = pack_f16x2(pr.x, pr.y);
              acc = __fadd2_rn(acc, make_float2(__uint_as_float((pk << 13) & 0x0FFFE000u),
                                                __uint_as_float((pk >> 3) & 0x0FFFE000u)));
            } else {
              pk = pack_bf16x2(pr.x, pr.y);
              acc = __fadd2_rn(acc, make_float2(bf16lo(pk), bf16hi(pk)));
            }
            sv[e] = pk;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) sv[e] = 0u;
        }
        tmem_st32(s_col, c0);
        // This group's previous P V (issued after this step's S) must have landed before
        // O is touched, and before this step's P V is released.  Waited every step, so
        // the phases are followed one by one.
        if (gk > 0) {
          const int pb = static_cast<int>((gk - 1) & 1);
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[pb], pvcount[pb] & 1, status, kDevTimeoutPFull));
          if (!ok) break;
          ++pvcount[pb];
          tc_fence_after();
        }
        // Rescale this group's half of O in place (warp-uniform: tcgen05.ld/st are
        // warp-collective); the partner does the other half with the same factor.
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int o0 = 0; o0 < D / 2; o0 += 16) {
            uint32_t ov[16];
            tmem_ld16(o_col + o0, ov);
            tmem_wait_ld();
            reg_fence16(ov);
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) ov[cc] = __float_as_uint(__uint_as_float(ov[cc]) * factor);
            tmem_st16(o_col + o0, ov);
          }
        }
        l = l * factor + (acc.x + acc.y) * (VF16 ? 0x1p112f : 1.0f);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
      }
      if (!ok) break;
      g += n;
      // Hand the running (max, sum) to the epilogue and move on to the next tile.  The
      // (m, l) buffer of this tile parity was last read by the epilogue of tile c - 2.
      if (c >= 2)
        ok = __all_sync(0xffffffffu, mbar_wait(&o_free[qb], ((c - 2) >> 1) & 1, status, kDevTimeoutOBar));
      if (!ok) break;
      ml[(qb * 2 + grp) * 128 + row] = m_ref;
      ml[512 + (qb * 2 + grp) * 128 + row] = l;
      mbar_arrive(&ml_ready[qb]);
    }
  } else {
    // ------------------------------------------------------------------ epilogue group
    const int row = (warp - kEpilogueWarp0) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((warp - kEpilogueWarp0) * 32) << 16;
    const bool upper = row >= 64;
    bool ok = true;
    for (int c = 0; ok; ++c) {
      const int qb = c & 1;
      const uint32_t par = (c >> 1) & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&meta_full[c % R], (c / R) & 1, status, kDevTimeoutMeta));
      if (!ok) break;
      const TileMeta t = read_meta(meta + (c % R) * kMetaInts);
      if (t.item < 0) break;
      const int n = t.n;
      ok = __all_sync(0xffffffffu, mbar_wait(&tile_done[qb], par, status, kDevTimeoutOBar) &&
                                       mbar_wait(&ml_ready[qb], par, status, kDevTimeoutOBar));
      if (!ok) break;
      tc_fence_after();
      // Both groups ran with the same reference maximum: L is the sum of their row sums.
      const float M = ml[(qb * 2) * 128 + row];
      const float L = ml[512 + (qb * 2) * 128 + row] + ml[512 + (qb * 2 + 1) * 128 + row];
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const bool has = n >= 1;                        // whether O was written in this tile
      const int blk = upper ? t.ib : t.ia;
      const bool valid_row = blk >= 0;
      const long long tok = static_cast<long long>(t.bh) * prm.S + static_cast<long long>(valid_row ? blk : 0) * 64 + (row & 63);
      const uint32_t oacc = tmem + lane_base + (qb ? C::kColO1 : C::kColO0);
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t a0[16];
        if (has) {
          tmem_ld16(oacc + c0, a0);
          tmem_wait_ld();
          reg_fence16(a0);
        }
        float v[16];
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) v[cc] = has ? __uint_as_float(a0[cc]) * inv : 0.f;
        if (valid_row) {
          if (prm.o_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(prm.o) + tok * D + c0);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) dst[cc] = make_float4(v[4 * cc], v[4 * cc + 1], v[4 * cc + 2], v[4 * cc + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.o) + tok * D + c0);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc)
              dst[cc] = make_uint4(pack_bf16x2(v[8 * cc], v[8 * cc + 1]), pack_bf16x2(v[8 * cc + 2], v[8 * cc + 3]),
                                   pack_bf16x2(v[8 * cc + 4], v[8 * cc + 5]), pack_bf16x2(v[8 * cc + 6], v[8 * cc + 7]));
          }
        }
      }
      if (valid_row && prm.lse != nullptr)
        prm.lse[tok] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
      tc_fence_before();
      mbar_arrive(&o_free[qb]);
      mbar_arrive(&meta_empty[c % R]);
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
  *map_ok = make_map_16(&mq, q, rows, D, 64, false) && make_map_16(&mk, k, rows, D, 64, false) &&
            make_map_16(&mv, v, rows, D, 64, VF16);   // one 64-row block per copy
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
  prm.T = d.T;
  prm.HW = d.Hb * d.Wb;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.o_f32 = o_dtype == NABLA_F32;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t ce = cudaMemsetAsync(workspace, 0, kStatusBytes, st);
  if (ce != cudaSuccess) return cuda_status(ce);
  int32_t* order = nullptr;
  ce = build_schedule(nullptr, mask_bits, d, static_cast<char*>(workspace) + kStatusBytes, &order, st,
                      /*frame_pairs=*/true);
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
