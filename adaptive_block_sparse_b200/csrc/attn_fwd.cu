// Block-sparse flash-attention forward over the kept 64 x 64 tiles (sm_100a).
//
// "NABLA: Neighborhood Adaptive Block-Level Attention" (gist.science, Chinese edition),
// technical summary, Methodology, "expansion": each kept entry (i, j) of the pooled
// block mask is one full N x N tile of the token attention matrix, computed exactly;
// the pages run this through FlexAttention.  Here it is a hand-written kernel:
//
//  * work tile = 128 query rows = two query blocks of one head (M = 128 MMAs): the same
//    patch in frames 2u and 2u + 1 (tile_blocks()).  The tile walks the ascending union
//    of the two blocks' kept key blocks, read from the mask bitmask, one key block per
//    step (N = 64 keys per S MMA); the half of the rows whose block does not keep a key
//    block skips its softmax (P = 0);
//  * persistent: one CTA per SM runs two independent pipelines ("slots"), each taking
//    tiles through an atomic counter in the schedule's order (heads by their longest
//    tile, tiles longest first inside a head).  A slot owns a Q buffer, two K and two V
//    stages, two TMEM score buffers and a TMEM accumulator; per step its chain is
//    S = Q K^T (tcgen05.mma) -> softmax -> O += P V with P read from TMEM, and S of the
//    next step is issued before P V of this one, into the other score buffer.  The two
//    chains share the tensor core: while one slot runs its softmax, the other's MMAs
//    run, and a tile change in one slot is covered by the other;
//  * per slot: a streamer warp fetches the tiles (the union of the two bitmask rows is
//    counted and walked warp-cooperatively, the tile's Q prefetched into L2) and loads
//    Q, K and V with TMA (128-byte swizzle, one copy per K or V block); one lane of an
//    issuer warp issues the MMAs; a softmax warpgroup (one query row per thread, TMEM
//    lane = row) holds the row's 64 scores of a step in registers, rescales O only when
//    a row maximum grows by more than 2^8, rounds P to the V operand's 16-bit type (the
//    row sum takes the rounded weights), and at the end of the tile normalises O,
//    releases the accumulator and writes O through a shared-memory staging area with
//    tiled TMA stores, and the LSE;
//  * the producer warps give registers to the softmax warpgroups (setmaxnreg);
//  * every barrier wait is bounded; on a timeout a kernel records a status code, stops,
//    drains its own copies and MMAs and frees TMEM.
#include <math.h>

#include <cudaTypedefs.h>

#include "common.cuh"

namespace nabla {
namespace {

constexpr int kThreads = 384;             // 12 warps
constexpr int kSoftmaxWarp0 = 4;          // warps 4..7 = slot 0, 8..11 = slot 1
constexpr int kMetaRing = 3;              // tile descriptors per slot
constexpr int kMetaInts = 8;              // item, bh, block a, block b, steps
// Registers per thread: the block launches with kLaunchRegs x 384; the producer warps
// (0-3) give registers up to the softmax warps (a row's 64 scores of a step, the packed
// weights, the epilogue's packed O row).
constexpr int kLaunchRegs = 168;
constexpr int kRegProducer = 64;
constexpr int kRegSoftmax = 216;
static_assert(128 * kRegProducer + 256 * kRegSoftmax <= kThreads * kLaunchRegs,
              "register split exceeds the block's launch budget");

template <int D>
struct FwdCfg {
  static constexpr int kPanels = D / 64;                  // 128-byte swizzle panels
  static constexpr int kTileBytes = 128 * D * 2;          // 128 rows of Q
  static constexpr int kStageBytes = 64 * D * 2;          // one key block of K or V
  static constexpr int kSlotBytes = kTileBytes + 4 * kStageBytes;   // Q, 2 K stages, 2 V stages
  static constexpr int kOffMeta = 2 * kSlotBytes;         // [2 slots][kMetaRing][kMetaInts]
  static constexpr int kOffBar = kOffMeta + 2 * kMetaRing * kMetaInts * 4;
  // bf16 O staging for the epilogue's tiled stores: per softmax warp 32 rows x 128 bytes
  // (64 dims), 1 KB aligned for the 128-byte swizzle
  static constexpr int kOffOStage = (kOffBar + 512 + 1023) / 1024 * 1024;
  static constexpr int kOStageWarpBytes = 32 * 128;
  static constexpr int kSmemBytes = kOffOStage + 8 * kOStageWarpBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;
  // slot s: score buffers b = 0, 1 at column 128 s + 64 b, accumulator at 256 + 128 s
  static __device__ __forceinline__ uint32_t col_s(int s, int b) {
    return static_cast<uint32_t>(s) * 128u + static_cast<uint32_t>(b) * 64u;
  }
  static __device__ __forceinline__ uint32_t col_o(int s) { return 256u + static_cast<uint32_t>(s) * 128u; }
};

struct FwdParams {
  const int32_t* order;      // work items (head * npairs + tile)
  int items;
  int npairs;
  const uint32_t* bits;      // [B*H, nb, nw]
  int nw;
  const void* q;             // for L2 prefetches of a tile's Q rows
  void* o;
  float* lse;
  uint32_t* status;          // word 0: status, word 1: work counter
  int nb;
  int T, HW;                 // frames, blocks per frame
  int Hb, Wb, Hg, W;         // blocks per frame row / column; latent height and width
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
  // rows of up to 64 words are held in registers for the whole tile: lane l keeps words
  // l and l + 32 of both rows, so moving to the next non-empty word takes a ballot and a
  // shuffle instead of a dependent global load
  bool reg;
  uint32_t a0, a1, b0, b1;
  __device__ void init(const uint32_t* row_a, const uint32_t* row_b, int n_words, int nb) {
    ra = row_a; rb = row_b; nw = n_words; w = -1; cur = 0u; a = b = 0u;
    tail = (nb & 31) ? (1u << (nb & 31)) - 1u : ~0u;
    reg = n_words <= 64;
    a0 = a1 = b0 = b1 = 0u;
    if (reg) {
      const int l = static_cast<int>(threadIdx.x & 31);
      if (l < nw) {
        const uint32_t m = (l == nw - 1) ? tail : ~0u;
        a0 = __ldg(ra + l) & m;
        b0 = rb ? (__ldg(rb + l) & m) : 0u;
      }
      if (l + 32 < nw) {
        const uint32_t m = (l + 32 == nw - 1) ? tail : ~0u;
        a1 = __ldg(ra + l + 32) & m;
        b1 = rb ? (__ldg(rb + l + 32) & m) : 0u;
      }
    }
  }
  __device__ int next(uint32_t* f) {
    while (cur == 0u) {
      const int base = w + 1;
      if (base >= nw) return -1;
      if (reg) {
        const int l = static_cast<int>(threadIdx.x & 31);
        const uint32_t nz0 = __ballot_sync(0xffffffffu, l >= base && (a0 | b0) != 0u);
        const uint32_t nz1 = __ballot_sync(0xffffffffu, l + 32 >= base && (a1 | b1) != 0u);
        if (nz0 != 0u) {
          const int src = __ffs(nz0) - 1;
          w = src;
          a = __shfl_sync(0xffffffffu, a0, src);
          b = __shfl_sync(0xffffffffu, b0, src);
        } else if (nz1 != 0u) {
          const int src = __ffs(nz1) - 1;
          w = 32 + src;
          a = __shfl_sync(0xffffffffu, a1, src);
          b = __shfl_sync(0xffffffffu, b1, src);
        } else {
          w = nw;
          return -1;
        }
        cur = a | b;
        continue;
      }
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

// Per-slot barriers (all in shared memory).
struct SlotBars {
  uint64_t q_full, q_empty;          // Q landed / the tile's last S has read Q
  uint64_t k_full[2], k_empty[2];    // K stage landed / S has read it
  uint64_t v_full[2], v_empty[2];    // V stage landed / P V has read it
  uint64_t s_full[2], p_full[2];     // score buffer: S landed / the softmax wrote P
  uint64_t pv_done;                  // completes once per P V (O may then be rescaled)
  uint64_t tile_done, o_free;        // the tile's last P V landed / the epilogue read O
  uint64_t meta_full[kMetaRing], meta_empty[kMetaRing];
  uint64_t drain;
};

// Roles (one CTA per SM; slot s = 0, 1):
//   warp 2 s      streamer of slot s: fetches tiles, publishes their descriptors
//                 (meta_full), loads Q, K, V;
//   warp 2 s + 1  MMA issuer of slot s (one lane);
//   warps 4-7 (slot 0), 8-11 (slot 1): softmax and epilogue of the slot's tiles.
// NAT: q, k, v, o, lse in the latent's natural token order; a block (an 8 x 8 patch of a
// frame) is then fetched with a 4-D copy (channels, patch columns, patch rows, frames of
// the head) that lands in shared memory exactly as the 64 reordered rows would.
template <int D, bool VF16, bool NAT>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v,
                    const __grid_constant__ CUtensorMap map_o, const FwdParams prm) {
  using C = FwdCfg<D>;
  constexpr int R = kMetaRing;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  SlotBars* bars = reinterpret_cast<SlotBars*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nb = prm.nb;
  const int nw = prm.nw;
  uint32_t* status = prm.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      SlotBars& B = bars[s];
      mbar_init(&B.q_full, 1);
      mbar_init(&B.q_empty, 1);
      for (int b = 0; b < 2; ++b) {
        mbar_init(&B.k_full[b], 1);
        mbar_init(&B.k_empty[b], 1);
        mbar_init(&B.v_full[b], 1);
        mbar_init(&B.v_empty[b], 1);
        mbar_init(&B.s_full[b], 1);
        mbar_init(&B.p_full[b], 128);
      }
      mbar_init(&B.pv_done, 1);
      mbar_init(&B.tile_done, 1);
      mbar_init(&B.o_free, 128);
      for (int r = 0; r < R; ++r) {
        mbar_init(&B.meta_full[r], 1);
        mbar_init(&B.meta_empty[r], 128);
      }
      mbar_init(&B.drain, 1);
    }
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

  if (warp < kSoftmaxWarp0) {
    reg_dealloc<kRegProducer>();
    const int slot = warp >> 1;
    SlotBars& B = bars[slot];
    unsigned char* sQ = smem + slot * C::kSlotBytes;
    unsigned char* sK = sQ + C::kTileBytes;             // stage b at sK + b * kStageBytes
    unsigned char* sV = sK + 2 * C::kStageBytes;
    int32_t* meta = reinterpret_cast<int32_t*>(smem + C::kOffMeta) + slot * R * kMetaInts;
    if ((warp & 1) == 0) {
      // ---------------------------------------------------------------- streamer of the slot
      // The whole warp fetches and walks; lane 0 issues the copies.  A step is one key
      // block; K and V each have two stages, K running a step ahead of V: K of step g + 1
      // once S of step g - 1 has read its stage, V of step g once P V of step g - 2 has.
      if (lane == 0) {
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
      }
      auto wait_all = [&](uint64_t* bar, uint32_t parity, uint32_t code) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, status, code));
      };
      // Block index -> (frame, patch row, patch column) without integer division: the
      // quotients come from float reciprocals, exact here (blk < 2^14, so (blk + 0.5) / n
      // stays more than 0.5 / n from an integer while its float error is below 2^-9 / n).
      const float inv_hw = 1.0f / static_cast<float>(prm.HW);
      const float inv_wb = 1.0f / static_cast<float>(prm.Wb);
      auto decode = [&](int blk) {
        const int tf = static_cast<int>((static_cast<float>(blk) + 0.5f) * inv_hw);
        const int r = blk - tf * prm.HW;
        const int hb = static_cast<int>((static_cast<float>(r) + 0.5f) * inv_wb);
        return make_int3(tf, hb, r - hb * prm.Wb);
      };
      // one 64-column panel of block blk of head bh: 64 rows of 128 bytes
      auto load_block = [&](unsigned char* dst, const CUtensorMap* map, uint64_t* bar, int pn, int bh,
                            int blk) {
        if constexpr (NAT) {
          const int3 c3 = decode(blk);
          const int tf = c3.x, hb = c3.y, wb = c3.z;
          tma_load_4d(dst, map, bar, pn * 64, wb * 8, hb * 8, bh * prm.T + tf);
        } else {
          tma_load_2d(dst, map, bar, pn * 64, static_cast<int>(bh * prm.S + static_cast<long long>(blk) * 64));
        }
      };
      // K or V of block blk of head bh, all D columns in one copy: the map's outermost
      // dimension walks the 64-column panels, so the copy lands as the panels one after
      // the other (8 KB apart), as per-panel copies would
      auto load_kv = [&](unsigned char* dst, const CUtensorMap* map, uint64_t* bar, int bh, int blk) {
        if constexpr (NAT) {
          const int3 c3 = decode(blk);
          const int tf = c3.x, hb = c3.y, wb = c3.z;
          tma_load_5d(dst, map, bar, 0, wb * 8, hb * 8, bh * prm.T + tf, 0);
        } else {
          tma_load_3d(dst, map, bar, 0, static_cast<int>(bh * prm.S + static_cast<long long>(blk) * 64), 0);
        }
      };
      // the rows of block blk of head bh into L2 (contiguous in the reordered order; eight
      // patch rows of 8 tokens in the natural one)
      auto prefetch_block = [&](int bh, int blk) {
        const char* qg = static_cast<const char*>(prm.q);
        if constexpr (NAT) {
          const int3 c3 = decode(blk);
          const int tf = c3.x, hb = c3.y, wb = c3.z;
#pragma unroll 1
          for (int hh = 0; hh < 8; ++hh)
            l2_prefetch(qg + ((static_cast<long long>(bh * prm.T + tf) * prm.Hg + hb * 8 + hh) * prm.W + wb * 8) * D * 2,
                        8 * D * 2);
        } else {
          l2_prefetch(qg + (static_cast<long long>(bh) * prm.S + static_cast<long long>(blk) * 64) * D * 2, 64 * D * 2);
        }
      };
      // Takes the next work item for tile c of this slot and publishes its descriptor in
      // ring entry c % R.  Returns 1 (tile), 0 (end of the work: terminator published) or
      // -1 (error).
      auto fetch = [&](int c) -> int {
        const int r = c % R;
        if (c >= R && !wait_all(&B.meta_empty[r], ((c / R) - 1) & 1, kDevTimeoutMeta)) return -1;
        int it = 0;
        if (lane == 0) it = atomicAdd(status + 1, 1);
        it = __shfl_sync(0xffffffffu, it, 0);
        int32_t* mt = meta + r * kMetaInts;
        if (it >= prm.items) {
          if (lane == 0) {
            mt[0] = -1;
            mt[4] = 0;
            mbar_arrive(&B.meta_full[r]);
          }
          __syncwarp();
          return 0;
        }
        const int item = prm.order[it];
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
          // the tile's Q rows into L2 ahead of their TMA copy
          prefetch_block(bh, ab.x);
          if (ab.y >= 0) prefetch_block(bh, ab.y);
          mt[0] = item;
          mt[1] = bh;
          mt[2] = ab.x;
          mt[3] = ab.y;
          mt[4] = cnt;
          mbar_arrive(&B.meta_full[r]);
        }
        __syncwarp();
        return 1;
      };
      long long gk = 0, gv = 0;   // K and V blocks issued
      int nq = 0;                 // Q tiles issued
      int fetched = 0;            // descriptors published
      bool end = false, ok = true;
      for (int c = 0; ok; ++c) {
        // the descriptor of this tile (normally fetched one tile ahead)
        while (!end && fetched <= c) {
          const int f = fetch(fetched);
          if (f < 0) { ok = false; break; }
          ++fetched;
          if (f == 0) end = true;
        }
        if (!ok || c >= fetched) break;
        const TileMeta t = read_meta(meta + (c % R) * kMetaInts);
        if (t.item < 0) break;
        // Q: the buffer frees once the previous tile's last S has run.  It is copied before
        // the next descriptor is fetched (three dependent global round trips), which would
        // otherwise delay every tile's first S.
        if (c > 0 && !wait_all(&B.q_empty, (c - 1) & 1, kDevTimeoutQFull)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(&B.q_full, C::kTileBytes);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn) {
            load_block(sQ + pn * 16384, &map_q, &B.q_full, pn, t.bh, t.ia);
            load_block(sQ + pn * 16384 + 8192, &map_q, &B.q_full, pn, t.bh, t.ib >= 0 ? t.ib : t.ia);
          }
        }
        __syncwarp();
        ++nq;
        WarpBitWalk wk;
        wk.init(prm.bits + (static_cast<long long>(t.bh) * nb + t.ia) * nw,
                t.ib >= 0 ? prm.bits + (static_cast<long long>(t.bh) * nb + t.ib) * nw : nullptr, nw, nb);
        auto load_k = [&](int j) -> bool {
          const int st = static_cast<int>(gk & 1);
          if (gk >= 2 && !wait_all(&B.k_empty[st], ((gk >> 1) - 1) & 1, kDevTimeoutKvEmpty)) return false;
          if (lane == 0) {
            mbar_arrive_expect_tx(&B.k_full[st], C::kStageBytes);
            load_kv(sK + st * C::kStageBytes, &map_k, &B.k_full[st], t.bh, j);
          }
          __syncwarp();
          ++gk;
          return true;
        };
        auto load_v = [&](int j) -> bool {
          const int st = static_cast<int>(gv & 1);
          if (gv >= 2 && !wait_all(&B.v_empty[st], ((gv >> 1) - 1) & 1, kDevTimeoutKvEmpty)) return false;
          if (lane == 0) {
            mbar_arrive_expect_tx(&B.v_full[st], C::kStageBytes);
            load_kv(sV + st * C::kStageBytes, &map_v, &B.v_full[st], t.bh, j);
          }
          __syncwarp();
          ++gv;
          return true;
        };
        uint32_t f = 0;
        int j_next = t.n > 0 ? wk.next(&f) : -1;
        if (t.n > 0 && !load_k(j_next)) { ok = false; break; }
        for (int k = 0; k < t.n; ++k) {
          const int j = j_next;
          if (k + 1 < t.n) {
            j_next = wk.next(&f);
            if (!load_k(j_next)) { ok = false; break; }
          }
          if (!load_v(j)) { ok = false; break; }
          // the next tile's descriptor, once this tile's first K, V (and second K) are on
          // their way
          if (k == 0 && !end && fetched == c + 1) {
            const int fr = fetch(fetched);
            if (fr < 0) { ok = false; break; }
            ++fetched;
            if (fr == 0) end = true;
          }
        }
        if (!ok) break;
        if (!end && fetched == c + 1) {     // a tile without steps
          const int fr = fetch(fetched);
          if (fr < 0) break;
          ++fetched;
          if (fr == 0) end = true;
        }
      }
      // Drain: copies still in flight must land before the CTA exits.
      if (nq > 0) mbar_wait(&B.q_full, (nq - 1) & 1, status, kDevTimeoutDrain);
      for (long long x = gk > 2 ? gk - 2 : 0; x < gk; ++x)
        mbar_wait(&B.k_full[x & 1], (x >> 1) & 1, status, kDevTimeoutDrain);
      for (long long x = gv > 2 ? gv - 2 : 0; x < gv; ++x)
        mbar_wait(&B.v_full[x & 1], (x >> 1) & 1, status, kDevTimeoutDrain);
      __syncwarp();
    } else {
      // ---------------------------------------------------------------- MMA issuer of the slot
      // Step g (one key block): S_g = Q K_g^T into score buffer g & 1, issued before
      // O += P_{g-1} V_{g-1}, so that S of the next step runs while the softmax of this
      // one does.  The buffer S_g overwrites held P_{g-2}, read by the P V issued before
      // (tcgen05 MMAs of one thread run in order).  Every P V commits pv_done, which the
      // softmax waits for before it rescales O.
      if (lane == 0) {
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
        constexpr uint32_t idesc_o = VF16 ? idesc_f16_f32(128, D, false, true)
                                          : idesc_bf16_f32(128, D, false, true);
        const uint32_t q_addr = smem_u32(sQ);
        const uint32_t k_addr = smem_u32(sK);
        const uint32_t v_addr = smem_u32(sV);
        const uint32_t o_tmem = tmem + C::col_o(slot);
        long long g = 0;   // steps whose S has been issued
        bool ok = true;
        auto issue_s = [&](bool last_of_tile) -> bool {
          const int b = static_cast<int>(g & 1);
          if (!mbar_wait(&B.k_full[b], (g >> 1) & 1, status, kDevTimeoutTmaFull)) return false;
          tc_fence_after();
          const uint32_t ks = k_addr + b * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int pn = kk >> 2, w = kk & 3;
            const uint64_t ad = sdesc_sw128(q_addr + pn * 16384 + w * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(ks + pn * 8192 + w * 32, 16, 1024);
            mma_bf16_ss(tmem + C::col_s(slot, b), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&B.s_full[b]);
          mma_commit(&B.k_empty[b]);
          if (last_of_tile) mma_commit(&B.q_empty);   // the tile's last S has read Q
          ++g;
          return true;
        };
        for (int c = 0; ok; ++c) {
          if (!mbar_wait(&B.meta_full[c % R], (c / R) & 1, status, kDevTimeoutMeta)) break;
          const TileMeta t = read_meta(meta + (c % R) * kMetaInts);
          if (t.item < 0) break;
          if (!mbar_wait(&B.q_full, c & 1, status, kDevTimeoutQFull)) break;
          tc_fence_after();
          if (t.n == 0) {
            // Nothing to compute: release Q; retire the tile after the previous one.
            mma_commit(&B.q_empty);
            if (c > 0 && !mbar_wait(&B.o_free, (c - 1) & 1, status, kDevTimeoutOBar)) break;
            mma_commit(&B.tile_done);
            continue;
          }
          if (!issue_s(t.n == 1)) break;
          for (int k = 0; k < t.n; ++k) {
            if (k + 1 < t.n && !issue_s(k + 2 == t.n)) { ok = false; break; }
            // P V of step k of the tile (global step gs: S of the next step, if any, is
            // already issued)
            const long long gs = (k + 1 < t.n) ? g - 2 : g - 1;
            const int b = static_cast<int>(gs & 1);
            if (!mbar_wait(&B.p_full[b], (gs >> 1) & 1, status, kDevTimeoutPFull)) { ok = false; break; }
            if (k == 0 && c > 0) {
              // The accumulator holds the previous tile until its epilogue has read it.
              if (!mbar_wait(&B.o_free, (c - 1) & 1, status, kDevTimeoutOBar)) { ok = false; break; }
            }
            if (!mbar_wait(&B.v_full[b], (gs >> 1) & 1, status, kDevTimeoutTmaFull)) { ok = false; break; }
            tc_fence_after();
            // O += P V: P (16-bit, 64 keys) in the first 32 columns of score buffer b, V stage
            // b MN-major (panel stride 8 KB along D, 8-row groups 1 KB apart).
            const uint32_t vs = v_addr + b * C::kStageBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = sdesc_sw128(vs + kk * 2048, 8192, 1024);
              mma_bf16_ts(o_tmem, tmem + C::col_s(slot, b) + kk * 8, bd, idesc_o, (k > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&B.v_empty[b]);
            mma_commit(&B.pv_done);
          }
          if (!ok) break;
          mma_commit(&B.tile_done);
        }
        mma_commit(&B.drain);
        mbar_wait(&B.drain, 0, status, kDevTimeoutDrain);
      }
      __syncwarp();
    }
  } else {
    reg_alloc<kRegSoftmax>();
    // ------------------------------------------------------------------ softmax of the slot
    const int slot = (warp - kSoftmaxWarp0) >> 2;
    SlotBars& B = bars[slot];
    const int32_t* meta = reinterpret_cast<const int32_t*>(smem + C::kOffMeta) + slot * R * kMetaInts;
    const int row = ((warp - kSoftmaxWarp0) & 3) * 32 + lane;      // 0..127 = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(((warp - kSoftmaxWarp0) & 3) * 32) << 16;
    const bool upper = row >= 64;
    const float sl2 = prm.scale_log2;
    const float2 sl2v = make_float2(sl2, sl2);
    const uint32_t o_col = tmem + lane_base + C::col_o(slot);
    long long g = 0;   // steps processed
    bool ok = true;
    for (int c = 0; ok; ++c) {
      ok = __all_sync(0xffffffffu, mbar_wait(&B.meta_full[c % R], (c / R) & 1, status, kDevTimeoutMeta));
      if (!ok) break;
      const TileMeta t = read_meta(meta + (c % R) * kMetaInts);
      if (t.item < 0) break;
      const int n = t.n;
      float m_ref = -INFINITY;
      float l = 0.f;
      // The step's key block and flags come from the tile's bitmask rows, walked the same
      // way as the streamer does.
      WarpBitWalk wk;
      wk.init(prm.bits + (static_cast<long long>(t.bh) * nb + t.ia) * nw,
              t.ib >= 0 ? prm.bits + (static_cast<long long>(t.bh) * nb + t.ib) * nw : nullptr, nw, nb);
      for (int k = 0; k < n; ++k, ++g) {
        uint32_t f = 0;
        wk.next(&f);
        // warp-uniform: rows 0-63 (block a) and 64-127 (block b) sit in different warps
        const bool keep = upper ? (f >> 1) : (f & 1u);
        const int b = static_cast<int>(g & 1);
        const uint32_t s_col = tmem + lane_base + C::col_s(slot, b);
        ok = __all_sync(0xffffffffu, mbar_wait(&B.s_full[b], (g >> 1) & 1, status, kDevTimeoutSFull));
        if (!ok) break;
        tc_fence_after();
        // The row's 64 scores of the step in registers: one TMEM round trip.
        uint32_t sv[64];
        uint32_t(&c0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t(&c1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        float mx = -INFINITY;
        if (keep) {
          tmem_ld32(s_col, c0);
          tmem_ld32(s_col + 32, c1);
          tmem_wait_ld();
          reg_fence32(c0);
          reg_fence32(c1);
          float m8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) m8[i] = -INFINITY;
#pragma unroll
          for (int cc = 0; cc < 64; cc += 2)
            m8[(cc >> 1) & 7] = fmax3(m8[(cc >> 1) & 7], __uint_as_float(sv[cc]), __uint_as_float(sv[cc + 1]));
          mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                     fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        }
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
        // P = 2^(s*scale*log2e - m) as 16-bit pairs (keys 2e, 2e+1 -> column e) into the
        // first 32 columns of the score buffer (those scores are already in registers).
        const float2 negm = make_float2(-m_ref, -m_ref);
        float2 acc = make_float2(0.f, 0.f);
        if (keep) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float2 xa = __ffma2_rn(make_float2(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])), sl2v, negm);
            const float2 pr = make_float2(fast_exp2(xa.x), fast_exp2(xa.y));
            // The row sum takes the rounded weights that enter the PV product, so the
            // output is an exact convex combination of them.
            uint32_t pk;
            if constexpr (VF16) {
              pk = pack_f16x2(pr.x, pr.y);
              add_halves_f16(acc, pk);
            } else {
              pk = pack_bf16x2(pr.x, pr.y);
              add_halves_bf16(acc, pk);
            }
            sv[e] = pk;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) sv[e] = 0u;
        }
        tmem_st32(s_col, c0);
        // O may be rescaled in place once every earlier P V of the slot has landed (the
        // previous step's, of this tile: a tile's first step never rescales), before this
        // step's P V (issued once p_full completes); warp-uniform.
        if (__any_sync(0xffffffffu, rescale)) {
          ok = __all_sync(0xffffffffu, mbar_wait(&B.pv_done, (g - 1) & 1, status, kDevTimeoutPFull));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int o0 = 0; o0 < D; o0 += 16) {
            uint32_t ov[16];
            tmem_ld16(o_col + o0, ov);
            tmem_wait_ld();
            reg_fence16(ov);
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) ov[cc] = __float_as_uint(__uint_as_float(ov[cc]) * factor);
            tmem_st16(o_col + o0, ov);
          }
        }
        l = l * factor + (acc.x + acc.y);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&B.p_full[b]);
      }
      if (!ok) break;
      // ---- epilogue of the tile: O / l and the LSE, once its last P V has landed
      ok = __all_sync(0xffffffffu, mbar_wait(&B.tile_done, c & 1, status, kDevTimeoutOBar));
      if (!ok) break;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int blk = upper ? t.ib : t.ia;
      const bool valid_row = blk >= 0;
      long long tok;   // the row's token: reordered index, or natural (t, h, w) index
      if constexpr (NAT) {
        const int bb = valid_row ? blk : 0;
        const int tf = bb / prm.HW, hb = (bb / prm.Wb) % prm.Hb, wb = bb % prm.Wb;
        tok = static_cast<long long>(t.bh) * prm.S +
              (static_cast<long long>(tf) * prm.Hg + hb * 8 + ((row & 63) >> 3)) * prm.W + wb * 8 + (row & 7);
      } else {
        tok = static_cast<long long>(t.bh) * prm.S + static_cast<long long>(valid_row ? blk : 0) * 64 + (row & 63);
      }
      // Each warp stages its 32 rows, 128 bytes of each at a time (64 bf16 or 32 f32 dims),
      // in the 128-byte-swizzled layout of a tiled copy, and one lane stores them with TMA
      // (a 4 x 8 token part of the patch, or 32 consecutive reordered rows), instead of
      // 16-byte stores scattered over 32 rows.
      const int wq = (warp - kSoftmaxWarp0) & 3;
      unsigned char* stage = smem + C::kOffOStage + ((warp - kSoftmaxWarp0) >> 2) * 4 * C::kOStageWarpBytes +
                             wq * C::kOStageWarpBytes;
      const int r32 = row & 31;
      // stage 8 x 16 bytes of this row, then one lane copies the warp's 32 rows to
      // columns [x0, x0 + 128 bytes) of O
      auto stage_and_store = [&](const uint4 (&ch8)[8], int x0) {
        if (lane == 0) bulk_wait_read_all();       // the previous copy has read the staging
        __syncwarp();
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(stage + r32 * 128 + ((ch ^ (r32 & 7)) << 4)) = ch8[ch];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && valid_row) {               // warp-uniform: a warp's rows are one block
          if constexpr (NAT) {
            const int tf = blk / prm.HW, hb = (blk / prm.Wb) % prm.Hb, wb = blk % prm.Wb;
            tma_store_4d(&map_o, stage, x0, wb * 8, hb * 8 + 4 * (wq & 1), t.bh * prm.T + tf);
          } else {
            tma_store_2d(&map_o, stage, x0,
                         static_cast<int>(static_cast<long long>(t.bh) * prm.S + static_cast<long long>(blk) * 64 +
                                          32 * (wq & 1)));
          }
          bulk_commit_group();
        }
      };
      if (prm.o_f32) {
        // 32 dims per copy; the accumulator is released after its last columns are read
#pragma unroll 1
        for (int d0 = 0; d0 < D; d0 += 32) {
          uint32_t a0[32];
          if (n > 0) {
            tmem_ld32(o_col + d0, a0);
            tmem_wait_ld();
            reg_fence32(a0);
          } else {
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) a0[cc] = 0u;
          }
          if (d0 + 32 == D) {
            tc_fence_before();
            mbar_arrive(&B.o_free);
          }
          uint4 ch8[8];
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            ch8[cc] = make_uint4(__float_as_uint(__uint_as_float(a0[4 * cc]) * inv),
                                 __float_as_uint(__uint_as_float(a0[4 * cc + 1]) * inv),
                                 __float_as_uint(__uint_as_float(a0[4 * cc + 2]) * inv),
                                 __float_as_uint(__uint_as_float(a0[4 * cc + 3]) * inv));
          stage_and_store(ch8, d0);
        }
      } else {
        // bf16 output: the whole row is read and packed first (D / 2 registers), so that the
        // next tile's P V may overwrite the accumulator while the row is being stored.
        uint32_t packed[D / 2];
#pragma unroll
        for (int d0 = 0; d0 < D; d0 += 32) {
          uint32_t a0[32];
          if (n > 0) {
            tmem_ld32(o_col + d0, a0);
            tmem_wait_ld();
            reg_fence32(a0);
          } else {
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) a0[cc] = 0u;
          }
#pragma unroll
          for (int cc = 0; cc < 16; ++cc)
            packed[d0 / 2 + cc] = pack_bf16x2(__uint_as_float(a0[2 * cc]) * inv, __uint_as_float(a0[2 * cc + 1]) * inv);
        }
        tc_fence_before();
        mbar_arrive(&B.o_free);
#pragma unroll
        for (int half = 0; half < D / 64; ++half) {
          uint4 ch8[8];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            ch8[ch] = make_uint4(packed[32 * half + 4 * ch], packed[32 * half + 4 * ch + 1],
                                 packed[32 * half + 4 * ch + 2], packed[32 * half + 4 * ch + 3]);
          stage_and_store(ch8, 64 * half);
        }
      }
      if (valid_row && prm.lse != nullptr)
        prm.lse[tok] = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      mbar_arrive(&B.meta_empty[c % R]);
    }
    if (lane == 0) bulk_wait_all();   // the epilogue's O copies have landed
    __syncwarp();
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

// 4-D map of 16-bit elements over a natural-order tensor viewed as [B*H*T, Hg, W, D]:
// box = 64 channels x 8 columns x 8 rows x 1 frame (one P x P patch = one block),
// 128-byte swizzle: the box lands as 64 rows of 128 bytes in the patch's row-major order,
// the order of the reordered layout.
bool make_map_nat(CUtensorMap* map, const void* base, long long frames, int Hg, int W, int D, bool fp16,
                  int box_h = 8);
bool make_map_nat(CUtensorMap* map, const void* base, long long frames, int Hg, int W, int D, bool fp16,
                  int box_h) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(W),
                        static_cast<cuuint64_t>(Hg), static_cast<cuuint64_t>(frames)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(W) * D * 2,
                           static_cast<cuuint64_t>(Hg) * W * D * 2};
  cuuint32_t box[4] = {64u, 8u, static_cast<cuuint32_t>(box_h), 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// K / V maps for one-copy block loads: the D columns split into 64-column panels as the
// outermost dimension (stride 128 bytes), box = 64 columns x one block x all panels.
// Natural order: [B*H*T, Hg, W, D] viewed as (64 ch, W, Hg, frames, D/64); reordered:
// [rows, D] viewed as (64 ch, rows, D/64).
bool make_map_kv(CUtensorMap* map, const void* base, long long rows, int D, bool fp16) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64u, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(D / 64)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, 128u};
  cuuint32_t box[3] = {64u, 64u, static_cast<cuuint32_t>(D / 64)};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_kv_nat(CUtensorMap* map, const void* base, long long frames, int Hg, int W, int D, bool fp16) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[5] = {64u, static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(Hg),
                        static_cast<cuuint64_t>(frames), static_cast<cuuint64_t>(D / 64)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(W) * D * 2,
                           static_cast<cuuint64_t>(Hg) * W * D * 2, 128u};
  cuuint32_t box[5] = {64u, 8u, 8u, 1u, static_cast<cuuint32_t>(D / 64)};
  cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  return enc(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// f32 O maps for the epilogue's stores: box = 32 floats (128 bytes) x 32 rows, or x 8
// columns x 4 rows x 1 frame of a natural-order tensor; 128-byte swizzle.
bool make_map_f32(CUtensorMap* map, const void* base, long long rows, int D) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 4};
  cuuint32_t box[2] = {32u, 32u};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_nat_f32(CUtensorMap* map, const void* base, long long frames, int Hg, int W, int D) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(W),
                        static_cast<cuuint64_t>(Hg), static_cast<cuuint64_t>(frames)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 4, static_cast<cuuint64_t>(W) * D * 4,
                           static_cast<cuuint64_t>(Hg) * W * D * 4};
  cuuint32_t box[4] = {32u, 8u, 4u, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
template <int D, bool VF16, bool NAT>
cudaError_t launch_fwd(const void* q, const void* k, const void* v, const Dims& d,
                       const FwdParams& prm, cudaStream_t st, bool* map_ok, bool* regs_ok) {
  CUtensorMap mq, mk, mv, mo;
  const long long rows = static_cast<long long>(d.BH) * d.S;
  const long long frames = static_cast<long long>(d.BH) * d.T;
  if constexpr (NAT) {
    *map_ok = make_map_nat(&mq, q, frames, d.Hg, d.W, D, false) &&
              make_map_kv_nat(&mk, k, frames, d.Hg, d.W, D, false) &&
              make_map_kv_nat(&mv, v, frames, d.Hg, d.W, D, VF16);
  } else {
    *map_ok = make_map_16(&mq, q, rows, D, 64, false) && make_map_kv(&mk, k, rows, D, false) &&
              make_map_kv(&mv, v, rows, D, VF16);
  }
  // O: tiled stores of 32-row parts, 128 bytes of each row per copy
  if (*map_ok)
    *map_ok = prm.o_f32 ? (NAT ? make_map_nat_f32(&mo, prm.o, frames, d.Hg, d.W, D)
                               : make_map_f32(&mo, prm.o, rows, D))
                        : (NAT ? make_map_nat(&mo, prm.o, frames, d.Hg, d.W, D, false, 4)
                               : make_map_16(&mo, prm.o, rows, D, 32, false));
  if (!*map_ok) return cudaErrorInvalidValue;
  using C = FwdCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, VF16, NAT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // The warpgroups' register split assumes the block launches with kLaunchRegs registers
  // per thread; with fewer, the increases could never be granted.  Refuse to launch.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_fwd_kernel<D, VF16, NAT>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) {
    *regs_ok = false;
    return cudaErrorInvalidConfiguration;
  }
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = prm.items < sms ? prm.items : sms;
  attn_fwd_kernel<D, VF16, NAT><<<grid, kThreads, C::kSmemBytes, st>>>(mq, mk, mv, mo, prm);
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
                                       float* lse, nabla_layout layout, void* workspace,
                                       size_t workspace_bytes, nabla_stream_t stream) {
  Dims d;
  nabla_status rc = check_shape(s, &d);
  if (rc != NABLA_OK) return rc;
  if (!q || !k || !v || !o || !mask_bits) return NABLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return NABLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(mask_bits) & 3) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
    return NABLA_ERR_INVALID_ARG;
  if (o_dtype != NABLA_BF16 && o_dtype != NABLA_F32) return NABLA_ERR_INVALID_ARG;
  if (v_dtype != NABLA_BF16 && v_dtype != NABLA_F16) return NABLA_ERR_INVALID_ARG;
  if (layout != NABLA_LAYOUT_REORDERED && layout != NABLA_LAYOUT_NATURAL) return NABLA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return NABLA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < nabla_fwd_workspace_bytes(s) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return NABLA_ERR_WORKSPACE;
  if (static_cast<long long>(d.BH) * d.S >= (1ll << 31)) return NABLA_ERR_UNSUPPORTED;
  FwdParams prm;
  prm.bits = mask_bits;
  prm.nw = d.nw;
  prm.q = q;
  prm.o = o;
  prm.lse = lse;
  prm.status = static_cast<uint32_t*>(workspace);
  prm.nb = d.nb;
  prm.S = d.S;
  prm.T = d.T;
  prm.HW = d.Hb * d.Wb;
  prm.Hb = d.Hb;
  prm.Wb = d.Wb;
  prm.Hg = d.Hg;
  prm.W = d.W;
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
  bool map_ok = true, regs_ok = true;
  const bool vf16 = v_dtype == NABLA_F16;
  const bool nat = layout == NABLA_LAYOUT_NATURAL;
  cudaError_t e;
  if (nat)
    e = d.D == 64 ? (vf16 ? launch_fwd<64, true, true>(q, k, v, d, prm, st, &map_ok, &regs_ok)
                          : launch_fwd<64, false, true>(q, k, v, d, prm, st, &map_ok, &regs_ok))
                  : (vf16 ? launch_fwd<128, true, true>(q, k, v, d, prm, st, &map_ok, &regs_ok)
                          : launch_fwd<128, false, true>(q, k, v, d, prm, st, &map_ok, &regs_ok));
  else
    e = d.D == 64 ? (vf16 ? launch_fwd<64, true, false>(q, k, v, d, prm, st, &map_ok, &regs_ok)
                          : launch_fwd<64, false, false>(q, k, v, d, prm, st, &map_ok, &regs_ok))
                  : (vf16 ? launch_fwd<128, true, false>(q, k, v, d, prm, st, &map_ok, &regs_ok)
                          : launch_fwd<128, false, false>(q, k, v, d, prm, st, &map_ok, &regs_ok));
  if (!regs_ok) return NABLA_ERR_UNSUPPORTED;
  return cuda_status(e);
}
