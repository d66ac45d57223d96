// Block-sparse flash-attention backward over the kept 64 x 64 tiles (sm_100a).
//
// The NABLA pages ("NABLA: Neighborhood Adaptive Block-Level Attention", gist.science,
// Chinese edition, technical summary, "Core contributions: two-stage acceleration";
// lsdiaocha.cn article, section 3, pre-training 10.9 s -> 7.5 s per iteration) credit the
// method with faster training as well as inference.  The binary mask has no gradient,
// so the backward pass is ordinary softmax-attention backward restricted to the kept
// tiles, with the mask held constant:
//   P = exp(scale Q K^T - LSE),  dP = dO V^T,  Dr = rowsum(dO * O),
//   dS = P * (dP - Dr),  dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K.
//
// Deterministic, no floating-point atomics, three launches:
//   1. preprocess: Dr = rowsum(dO * O), LSE in log2 units and fp16 copies of Q, K, V, dO
//      in the fractal block order, gathered from the natural token order when the
//      tensors come in it (HBM-bound);
//   2. dK/dV: one CTA per pair of key blocks (the same patch in frames 2u and 2u + 1, as
//      the forward pairs query blocks: their column lists overlap most; 128 key rows ->
//      M = 128 MMAs) walks the ascending union of the two blocks' query-block (column)
//      lists.  Per query block: S^T = K Q^T and dP^T = V dO^T into TMEM (double-buffered);
//      P^T and dS^T are formed in registers and written back over them as 16-bit
//      operands; dV += P^T dO and dK += dS^T Q read those from TMEM (A operand) and
//      accumulate in TMEM;
//   3. dQ: one CTA per pair of query blocks walks the union of the row lists:
//      S = Q K^T and dP = dO V^T into TMEM, dS written back over dP, dQ += dS K.
// Warp roles: warp 0 = TMA producer (four-stage ring; the whole warp walks the lists, 32
// entries per load), warp 1 = MMA issuer and TMEM owner, warps 4-11 = element-wise math
// (a key or query row per TMEM lane, each 64-wide tile split in two column halves between
// warps w and w + 4) and epilogue (fp32 gradients staged in the freed ring and stored
// with tiled TMA stores, at the natural token indices when the tensors came in that
// order).  Every wait is bounded.
#include <math.h>

#include <cudaTypedefs.h>

#include <cuda_fp16.h>

#include "common.cuh"

namespace nabla {

bool make_map_16(CUtensorMap* map, const void* base, long long rows, int D, int box_rows,
                 bool fp16);
bool make_map_kv(CUtensorMap* map, const void* base, long long rows, int D, bool fp16);
bool make_map_f32(CUtensorMap* map, const void* base, long long rows, int D);
bool make_map_nat_f32(CUtensorMap* map, const void* base, long long frames, int Hg, int W, int D);

namespace {

constexpr int kThreads = 384;             // warp 0 TMA, warp 1 MMA, warps 4-11 element-wise
constexpr int kMathWarp0 = 4;
constexpr int kMathThreads = 256;
constexpr uint32_t kEnd = 0xFFFFFFFFu;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Reordered row -> natural token of the same head (NABLA_LAYOUT_NATURAL): block r / 64
// is the 8 x 8 patch (frame, patch row, patch column) of the fractal order, token r % 64
// the row-major position inside it.
struct NatMap {
  int on;
  int HW, Wb, Hg, W;
  long long S;
  __device__ __forceinline__ long long token(long long bh, int blk, int r64) const {
    const int tf = blk / HW, rr = blk - tf * HW, hb = rr / Wb, wb = rr - hb * Wb;
    return bh * S + (static_cast<long long>(tf) * Hg + hb * 8 + (r64 >> 3)) * W + wb * 8 + (r64 & 7);
  }
  __device__ __forceinline__ long long token_of_row(long long row) const {
    const long long bh = row / S;
    const int r = static_cast<int>(row - bh * S);
    return token(bh, r >> 6, r & 63);
  }
};

// -------------------------------------------------------------------------------------
// 1. preprocess: delta = rowsum(dO * O), lse2 = LSE * log2(e)
// -------------------------------------------------------------------------------------
// Also writes fp16 copies of Q, K, V and dO for the MMAs of the backward pass: P and dS
// are then rounded to fp16 (11-bit significand) instead of bf16 (8-bit), which keeps the
// gradients within 2e-2 of fp64 where bf16 P / dS would not (|dS| reaches ~30).  bf16 ->
// fp16 is exact for 2^-14 <= |x| <= 65504; smaller magnitudes lose low bits (absolute error
// below 6e-8); larger ones cannot be represented and are reported as a device status.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(
    const void* __restrict__ o, int o_f32, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, const __nv_bfloat16* __restrict__ q,
    const __nv_bfloat16* __restrict__ k, const void* __restrict__ v, int v_f16,
    __half* __restrict__ q16, __half* __restrict__ k16, __half* __restrict__ v16,
    __half* __restrict__ do16, float* __restrict__ delta, float* __restrict__ lse2,
    long long rows, uint32_t* status, NatMap nat) {
  // D / 8 lanes per row, 8 contiguous elements (16 bytes of a 16-bit tensor) per lane.
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  const int lane = threadIdx.x & 31;
  const long long row = (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * kRowsPerWarp +
                        lane / kLanesPerRow;
  const bool active = row < rows;
  // the outputs are written at the reordered row; with natural-order inputs the row's
  // token is read from its natural index (the gather of the fractal flatten)
  const long long src_row = nat.on && active ? nat.token_of_row(row) : row;
  const long long base = (active ? row : 0) * D + (lane % kLanesPerRow) * 8;
  const long long sbase = (active ? src_row : 0) * D + (lane % kLanesPerRow) * 8;
  float acc = 0.f;
  bool range_ok = true;
  if (active) {
    auto widen = [](uint4 u, float* f) {
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    };
    auto to_f16 = [&](const float* f) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        range_ok = range_ok && fabsf(f[2 * i]) <= 65504.f && fabsf(f[2 * i + 1]) <= 65504.f;
        const __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
      return make_uint4(w[0], w[1], w[2], w[3]);
    };
    float g[8], of[8], t[8];
    widen(*reinterpret_cast<const uint4*>(dout + sbase), g);
    if (o_f32) {
      const float4 o0 = *reinterpret_cast<const float4*>(static_cast<const float*>(o) + sbase);
      const float4 o1 = *reinterpret_cast<const float4*>(static_cast<const float*>(o) + sbase + 4);
      of[0] = o0.x; of[1] = o0.y; of[2] = o0.z; of[3] = o0.w;
      of[4] = o1.x; of[5] = o1.y; of[6] = o1.z; of[7] = o1.w;
    } else {
      widen(*reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(o) + sbase), of);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc = fmaf(g[i], of[i], acc);
    *reinterpret_cast<uint4*>(do16 + base) = to_f16(g);
    widen(*reinterpret_cast<const uint4*>(q + sbase), t);
    *reinterpret_cast<uint4*>(q16 + base) = to_f16(t);
    widen(*reinterpret_cast<const uint4*>(k + sbase), t);
    *reinterpret_cast<uint4*>(k16 + base) = to_f16(t);
    if (!v_f16) {
      widen(*reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(v) + sbase), t);
      *reinterpret_cast<uint4*>(v16 + base) = to_f16(t);
    } else if (nat.on) {   // an fp16 V in the natural order is gathered as it is
      const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __half*>(v) + sbase);
      // an infinite or NaN half (exponent bits all set) is out of the range
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        range_ok = range_ok && (w[i] & 0x7C00u) != 0x7C00u && (w[i] & 0x7C000000u) != 0x7C000000u;
      *reinterpret_cast<uint4*>(v16 + base) = u;
    }
  }
#pragma unroll
  for (int off = kLanesPerRow / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (!__all_sync(0xffffffffu, range_ok) && lane == 0) record_status(status, kDevFp16Range);
  if (active && lane % kLanesPerRow == 0) {
    delta[row] = acc;
    lse2[row] = lse[src_row] * kLog2e;
  }
}

struct BwdParams {
  const int32_t* order;      // work items (head * npairs + pair), longest first
  int npairs;
  const int32_t* list_idx;   // column lists (dK/dV pass) or row lists (dQ pass)
  const int32_t* list_cnt;
  const float* delta;
  const float* lse2;
  float* out0;               // dV (dK/dV pass) or dQ (dQ pass)
  float* out1;               // dK (dK/dV pass)
  uint32_t* status;
  int nb;
  int T, HW;                 // frames, blocks per frame (pairing of blocks, tile_blocks())
  long long S;
  float scale_log2;
  float scale;
  NatMap nat;                // outputs at natural token indices when nat.on
};

// Walks the ascending union of two sorted lists with a whole warp; every lane gets the
// same result, -1 at the end.  f: bit0 = in the first list, bit1 = in the second.  The
// lists are read 32 entries at a time (one coalesced load per list), the next 32 already
// in flight, so a step costs a few shuffles instead of a dependent global load.
struct WarpUnion {
  const int32_t* l0;
  const int32_t* l1;
  int c0, c1, a, b, base0, base1;
  int v0, v1, n0, n1;        // this lane's entry of the current and of the next chunk
  __device__ static int load(const int32_t* l, int c, int pos) { return pos < c ? __ldg(l + pos) : 0x7FFFFFFF; }
  __device__ void init(const int32_t* list0, int cnt0, const int32_t* list1, int cnt1, int lane) {
    l0 = list0;
    l1 = list1;
    c0 = cnt0;
    c1 = cnt1;
    a = b = base0 = base1 = 0;
    v0 = load(l0, c0, lane);
    v1 = load(l1, c1, lane);
    n0 = load(l0, c0, 32 + lane);
    n1 = load(l1, c1, 32 + lane);
  }
  __device__ int next(uint32_t* f, int lane) {
    if (a - base0 == 32) {          // warp-uniform
      base0 += 32;
      v0 = n0;
      n0 = load(l0, c0, base0 + 32 + lane);
    }
    if (b - base1 == 32) {
      base1 += 32;
      v1 = n1;
      n1 = load(l1, c1, base1 + 32 + lane);
    }
    const int ja = __shfl_sync(0xffffffffu, v0, a - base0);
    const int jb = __shfl_sync(0xffffffffu, v1, b - base1);
    const int xa = a < c0 ? ja : 0x7FFFFFFF;
    const int xb = b < c1 ? jb : 0x7FFFFFFF;
    if (xa == 0x7FFFFFFF && xb == 0x7FFFFFFF) return -1;
    if (xa < xb) { *f = 1; ++a; return xa; }
    if (xb < xa) { *f = 2; ++b; return xb; }
    *f = 3; ++a; ++b; return xa;
  }
};

template <int D>
struct BwdCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kPairBytes = 128 * D * 2;       // one 128-row operand (resident)
  static constexpr int kTileBytes = 64 * D * 2;        // one 64-row operand (streamed)
  static constexpr uint32_t kTmemCols = 512;
  // TMEM: buffer b at columns [128b, 128b+64) = S (or S^T), [128b+64, 128b+128) = dP (or
  // dP^T); the element-wise pass overwrites them in place with the 16-bit P and dS
  // operands of the next MMAs.  Accumulators from column 256.
  static constexpr uint32_t kColAcc0 = 256, kColAcc1 = 384;
};

// Column of the packed 16-bit operand for K chunk kk (16 values, 8 columns) of a 64-wide
// tile written in place by two thread groups: group h packs its 32 values into the first
// 16 of the 32 columns it read, [32h, 32h+16).
__device__ __forceinline__ uint32_t packed_col(int kk) { return kk < 2 ? kk * 8 : 32 + (kk - 2) * 8; }

// Epilogue store of 32 f32 columns [x0, x0 + 32) of a warp's 32 rows (this lane's row:
// v[0..31], already scaled): the rows are staged in the 128-byte-swizzled layout of a
// tiled copy at `stage` (4 KB, used once), and one lane stores them with TMA -- rows
// 32 q32 .. 32 q32 + 31 of block `blk` of head bh: 32 reordered rows, or a 4 x 8 token
// part of the block's 8 x 8 patch.  The copy runs on after the CTA has moved on; the
// CTA waits only for it to have read the staging before it exits.
__device__ __forceinline__ void store_rows_f32(const CUtensorMap* map, unsigned char* stage, const uint32_t (&v)[32],
                                               int lane, int x0, long long bh, int blk, int q32,
                                               const NatMap& nat, int T) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch)
    *reinterpret_cast<uint4*>(stage + lane * 128 + ((ch ^ (lane & 7)) << 4)) =
        make_uint4(v[4 * ch], v[4 * ch + 1], v[4 * ch + 2], v[4 * ch + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    if (nat.on) {
      const int tf = blk / nat.HW, rr = blk - tf * nat.HW, hb = rr / nat.Wb, wb = rr - hb * nat.Wb;
      tma_store_4d(map, stage, x0, wb * 8, hb * 8 + 4 * q32, static_cast<int>(bh * T + tf));
    } else {
      tma_store_2d(map, stage, x0, static_cast<int>(bh * nat.S + static_cast<long long>(blk) * 64 + 32 * q32));
    }
    bulk_commit_group();
  }
}

// -------------------------------------------------------------------------------------
// 2. dK / dV over column lists
// -------------------------------------------------------------------------------------
template <int D>
struct DkdvLayout {
  using C = BwdCfg<D>;
  static constexpr int kStages = 4;
  static constexpr int kStageBytes = 2 * C::kTileBytes + 512;    // Q_i, dO_i, lse2_i, delta_i
  static constexpr int kStageStride = (kStageBytes + 1023) / 1024 * 1024;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + C::kPairBytes;
  static constexpr int kOffStage = kOffV + C::kPairBytes;
  static constexpr int kOffBar = kOffStage + kStages * kStageStride;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
};

// One CTA per pair of key blocks (ja, jb) = tile_blocks(pair): rows 0-63 of the resident
// K and V operands are block ja, rows 64-127 block jb.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap map_q64,
                         const __grid_constant__ CUtensorMap map_do64,
                         const __grid_constant__ CUtensorMap map_k64,
                         const __grid_constant__ CUtensorMap map_v64,
                         const __grid_constant__ CUtensorMap map_out0,
                         const __grid_constant__ CUtensorMap map_out1, const BwdParams prm) {
  using C = BwdCfg<D>;
  using L = DkdvLayout<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sK = smem + L::kOffK;
  unsigned char* sV = smem + L::kOffV;
  unsigned char* sStage = smem + L::kOffStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;                    // [kStages]
  uint64_t* empty = bars + L::kStages;      // [kStages]
  uint64_t* kv_full = bars + 2 * L::kStages;
  uint64_t* sd_full = kv_full + 1;          // [2]
  uint64_t* p_full = sd_full + 2;           // [2]
  uint64_t* acc_bar = p_full + 2;
  uint64_t* drain = acc_bar + 1;
  uint32_t* meta = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* tmem_slot = meta + L::kStages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int item = prm.order[blockIdx.x];
  const long long bh = item / prm.npairs;
  const int nb = prm.nb;
  const int2 jab = tile_blocks(item - static_cast<int>(bh) * prm.npairs, prm.T, prm.HW, nb);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(kv_full, 1);
    mbar_init(&sd_full[0], 1);
    mbar_init(&sd_full[1], 1);
    mbar_init(&p_full[0], kMathThreads);
    mbar_init(&p_full[1], kMathThreads);
    mbar_init(acc_bar, 1);
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

  if (warp == 0) {
    // the whole warp walks the lists; lane 0 waits on the ring and issues the copies
    if (lane == 0) {
      tma_prefetch_desc(&map_q64);
      tma_prefetch_desc(&map_do64);
      tma_prefetch_desc(&map_k64);
      tma_prefetch_desc(&map_v64);
      // a lone block (jab.y < 0) is loaded twice; its upper rows are never kept
      const int ka = static_cast<int>(bh * prm.S + static_cast<long long>(jab.x) * 64);
      const int kb = static_cast<int>(bh * prm.S + static_cast<long long>(jab.y >= 0 ? jab.y : jab.x) * 64);
      mbar_arrive_expect_tx(kv_full, 2 * C::kPairBytes);
#pragma unroll
      for (int pn = 0; pn < C::kPanels; ++pn) {
        tma_load_2d(sK + pn * 16384, &map_k64, kv_full, pn * 64, ka);
        tma_load_2d(sK + pn * 16384 + 8192, &map_k64, kv_full, pn * 64, kb);
        tma_load_2d(sV + pn * 16384, &map_v64, kv_full, pn * 64, ka);
        tma_load_2d(sV + pn * 16384 + 8192, &map_v64, kv_full, pn * 64, kb);
      }
    }
    WarpUnion wk;
    wk.init(prm.list_idx + (bh * nb + jab.x) * static_cast<long long>(nb),
            min(max(prm.list_cnt[bh * nb + jab.x], 0), nb),
            prm.list_idx + (bh * nb + (jab.y >= 0 ? jab.y : jab.x)) * static_cast<long long>(nb),
            jab.y >= 0 ? min(max(prm.list_cnt[bh * nb + jab.y], 0), nb) : 0, lane);
    int it = 0;
    bool ended = false;
    while (true) {
      uint32_t f = 0;
      const int i = wk.next(&f, lane);
      const int s = it % L::kStages;
      const int n = it / L::kStages;
      int ok = 1;
      if (lane == 0 && n > 0) ok = mbar_wait(&empty[s], (n - 1) & 1, prm.status, kDevTimeoutKvEmpty) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (i < 0 || i >= nb) {
        if (lane == 0) {
          meta[s] = kEnd;
          mbar_arrive(&full[s]);
        }
        ended = true;
        break;
      }
      if (lane == 0) {
        meta[s] = static_cast<uint32_t>(i) | (f << 28);
        unsigned char* st = sStage + s * L::kStageStride;
        mbar_arrive_expect_tx(&full[s], 2 * C::kTileBytes + 512);
        const long long qrow = bh * prm.S + static_cast<long long>(i) * 64;
        // one copy per operand: all D columns of the 64 rows (panels 8 KB apart)
        tma_load_3d(st, &map_q64, &full[s], 0, static_cast<int>(qrow), 0);
        tma_load_3d(st + C::kTileBytes, &map_do64, &full[s], 0, static_cast<int>(qrow), 0);
        bulk_load(st + 2 * C::kTileBytes, prm.lse2 + qrow, 256, &full[s]);
        bulk_load(st + 2 * C::kTileBytes + 256, prm.delta + qrow, 256, &full[s]);
      }
      ++it;
    }
    if (lane == 0) {
      // Copies still in flight: the last kStages iterations, except that placing the end
      // marker waited for the oldest of them to be consumed (its stage was reused), and a
      // parity wait on that stage would now look two phases back.
      const int keep = ended ? L::kStages - 1 : L::kStages;
      const int first = it > keep ? it - keep : 0;
      for (int x = first; x < it; ++x)
        mbar_wait(&full[x % L::kStages], (x / L::kStages) & 1, prm.status, kDevTimeoutDrain);
      mbar_wait(kv_full, 0, prm.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f16_f32(128, 64, false, false);
      constexpr uint32_t idesc_acc = idesc_f16_f32(128, D, false, true);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      const uint32_t st_addr = smem_u32(sStage);
      // S^T = K Q_i^T and dP^T = V dO_i^T into buffer x & 1
      auto issue_sd = [&](int x) {
        const int s = x % L::kStages;
        const uint32_t qa = st_addr + s * L::kStageStride;
        const uint32_t da = qa + C::kTileBytes;
        const uint32_t col = (x & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2, w = kk & 3;
          mma_bf16_ss(tmem + col, sdesc_sw128(k_addr + pn * 16384 + w * 32, 16, 1024),
                      sdesc_sw128(qa + pn * 8192 + w * 32, 16, 1024), idesc_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2, w = kk & 3;
          mma_bf16_ss(tmem + col + 64, sdesc_sw128(v_addr + pn * 16384 + w * 32, 16, 1024),
                      sdesc_sw128(da + pn * 8192 + w * 32, 16, 1024), idesc_s, kk > 0);
        }
        mma_commit(&sd_full[x & 1]);
      };
      // dV += P^T dO_i and dK += dS^T Q_i, with P^T and dS^T read from TMEM
      auto issue_acc = [&](int x) {
        const int s = x % L::kStages;
        const uint32_t qa = st_addr + s * L::kStageStride;
        const uint32_t da = qa + C::kTileBytes;
        const uint32_t col = (x & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_bf16_ts(tmem + C::kColAcc0, tmem + col + packed_col(kk), sdesc_sw128(da + kk * 2048, 8192, 1024),
                      idesc_acc, (x > 0 || kk > 0) ? 1u : 0u);
          mma_bf16_ts(tmem + C::kColAcc1, tmem + col + 64 + packed_col(kk),
                      sdesc_sw128(qa + kk * 2048, 8192, 1024), idesc_acc, (x > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(kv_full, 0, prm.status, kDevTimeoutQFull);
      if (ok) ok = mbar_wait(&full[0], 0, prm.status, kDevTimeoutTmaFull);
      if (ok && meta[0] != kEnd) {
        tc_fence_after();
        issue_sd(0);
        for (int it = 0;; ++it) {
          const int s1 = (it + 1) % L::kStages;
          if (!mbar_wait(&full[s1], ((it + 1) / L::kStages) & 1, prm.status, kDevTimeoutTmaFull)) break;
          const bool end1 = meta[s1] == kEnd;
          tc_fence_after();
          // buffer (it + 1) & 1 was last read by issue_acc(it - 1), issued before: MMAs of
          // one thread run in order
          if (!end1) issue_sd(it + 1);
          if (!mbar_wait(&p_full[it & 1], (it >> 1) & 1, prm.status, kDevTimeoutPFull)) break;
          tc_fence_after();
          issue_acc(it);
          mma_commit(&empty[it % L::kStages]);
          if (end1) break;
        }
      }
      mma_commit(acc_bar);
      mma_commit(drain);
      mbar_wait(drain, 0, prm.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp >= kMathWarp0) {
    // 8 warps: key row = TMEM lane ((warp & 3) * 32 + lane), column half h of each 64-wide
    // tile (warps 4-7: queries 0-31, warps 8-11: queries 32-63)
    const int mw = warp - kMathWarp0;
    const int h = mw >> 2;
    const int row = (mw & 3) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((mw & 3) * 32) << 16;
    const bool upper = row >= 64;
    const float sl2 = prm.scale_log2;
    int it = 0;
    bool ok = true;
    for (;; ++it) {
      const int s = it % L::kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (it / L::kStages) & 1, prm.status, kDevTimeoutTmaFull));
      if (!ok) break;
      const uint32_t mt = meta[s];
      if (mt == kEnd) break;
      const bool keep = upper ? ((mt >> 29) & 1u) : ((mt >> 28) & 1u);
      const float* s_lse = reinterpret_cast<const float*>(sStage + s * L::kStageStride + 2 * C::kTileBytes) + 32 * h;
      const float* s_del = s_lse + 64;
      ok = __all_sync(0xffffffffu, mbar_wait(&sd_full[it & 1], (it >> 1) & 1, prm.status, kDevTimeoutSFull));
      if (!ok) break;
      tc_fence_after();
      const uint32_t col = tmem + lane_base + (it & 1) * 128 + 32 * h;
      uint32_t pk[16], dk[16];
      if (keep) {
        uint32_t sv[32], dv[32];
        tmem_ld32(col, sv);
        tmem_ld32(col + 64, dv);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(sv[c]), sl2, -s_lse[c]));
          const float p1 = fast_exp2(fmaf(__uint_as_float(sv[c + 1]), sl2, -s_lse[c + 1]));
          pk[c >> 1] = pack_f16x2(p0, p1);
          dk[c >> 1] = pack_f16x2(p0 * (__uint_as_float(dv[c]) - s_del[c]),
                                  p1 * (__uint_as_float(dv[c + 1]) - s_del[c + 1]));
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) { pk[c] = 0u; dk[c] = 0u; }
      }
      tmem_st16(col, pk);
      tmem_st16(col + 64, dk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[it & 1]);
    }
    // ---- epilogue: dV and scale * dK (fp32), columns [64h, 64h + 64) of the row ----------
    const int blk = upper ? jab.y : jab.x;
    const bool valid = blk >= 0;
    const long long tok = prm.nat.on ? prm.nat.token(bh, valid ? blk : 0, row & 63)
                                     : bh * prm.S + static_cast<long long>(valid ? blk : 0) * 64 + (row & 63);
    bool have = ok && it > 0;
    if (have) {
      have = __all_sync(0xffffffffu, mbar_wait(acc_bar, 0, prm.status, kDevTimeoutOBar));
      tc_fence_after();
    }
    if (have) {
      // Every MMA has completed and every copy into the stage ring has landed and been
      // read (the last accumulation waited for all of them), so the ring is free: each
      // warp stages its 32 rows x 64 columns of dV and dK there (4 KB per 32 columns).
      unsigned char* stage = sStage + mw * (D / 2) * 4 * 32 * 2;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const float mul = which == 0 ? 1.f : prm.scale;
        const uint32_t colbase = (which == 0 ? C::kColAcc0 : C::kColAcc1) + (D / 2) * h;
#pragma unroll 1
        for (int c0 = 0; c0 < D / 2; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_base + colbase + c0, ov);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * mul);
          if (valid)   // warp-uniform: a warp's rows are one block
            store_rows_f32(which == 0 ? &map_out0 : &map_out1, stage, ov, lane, (D / 2) * h + c0, bh, blk,
                           (mw & 3) & 1, prm.nat, prm.T);
          stage += 4096;
        }
      }
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
    } else {
      // no step, or a wait gave up: zeros, stored directly (copies may still be landing
      // in the stage ring)
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        float* out = which == 0 ? prm.out0 : prm.out1;
#pragma unroll 1
        for (int c0 = 0; c0 < D / 2; c0 += 4)
          if (valid) *reinterpret_cast<float4*>(out + tok * D + (D / 2) * h + c0) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// -------------------------------------------------------------------------------------
// 3. dQ over row lists
// -------------------------------------------------------------------------------------
template <int D>
struct DqLayout {
  using C = BwdCfg<D>;
  static constexpr int kStages = 4;
  static constexpr int kStageBytes = 2 * C::kTileBytes;        // K_j, V_j
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kOffQ + C::kPairBytes;
  static constexpr int kOffStage = kOffDO + C::kPairBytes;
  static constexpr int kOffBar = kOffStage + kStages * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
};

// One CTA per pair of query blocks (ia, ib) = tile_blocks(pair).
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap map_q64,
                       const __grid_constant__ CUtensorMap map_do64,
                       const __grid_constant__ CUtensorMap map_k64,
                       const __grid_constant__ CUtensorMap map_v64,
                       const __grid_constant__ CUtensorMap map_out0, const BwdParams prm) {
  using C = BwdCfg<D>;
  using L = DqLayout<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = smem + L::kOffQ;
  unsigned char* sDO = smem + L::kOffDO;
  unsigned char* sStage = smem + L::kOffStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + L::kStages;
  uint64_t* q_full = bars + 2 * L::kStages;
  uint64_t* sd_full = q_full + 1;
  uint64_t* p_full = sd_full + 2;
  uint64_t* acc_bar = p_full + 2;
  uint64_t* drain = acc_bar + 1;
  uint32_t* meta = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* tmem_slot = meta + L::kStages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int item = prm.order[blockIdx.x];
  const long long bh = item / prm.npairs;
  const int nb = prm.nb;
  const int2 iab = tile_blocks(item - static_cast<int>(bh) * prm.npairs, prm.T, prm.HW, nb);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(&sd_full[0], 1);
    mbar_init(&sd_full[1], 1);
    mbar_init(&p_full[0], kMathThreads);
    mbar_init(&p_full[1], kMathThreads);
    mbar_init(acc_bar, 1);
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

  if (warp == 0) {
    // the whole warp walks the lists; lane 0 waits on the ring and issues the copies
    if (lane == 0) {
      tma_prefetch_desc(&map_q64);
      tma_prefetch_desc(&map_do64);
      tma_prefetch_desc(&map_k64);
      tma_prefetch_desc(&map_v64);
      const int qa = static_cast<int>(bh * prm.S + static_cast<long long>(iab.x) * 64);
      const int qb = static_cast<int>(bh * prm.S + static_cast<long long>(iab.y >= 0 ? iab.y : iab.x) * 64);
      mbar_arrive_expect_tx(q_full, 2 * C::kPairBytes);
#pragma unroll
      for (int pn = 0; pn < C::kPanels; ++pn) {
        tma_load_2d(sQ + pn * 16384, &map_q64, q_full, pn * 64, qa);
        tma_load_2d(sQ + pn * 16384 + 8192, &map_q64, q_full, pn * 64, qb);
        tma_load_2d(sDO + pn * 16384, &map_do64, q_full, pn * 64, qa);
        tma_load_2d(sDO + pn * 16384 + 8192, &map_do64, q_full, pn * 64, qb);
      }
    }
    WarpUnion wk;
    wk.init(prm.list_idx + (bh * nb + iab.x) * static_cast<long long>(nb),
            min(max(prm.list_cnt[bh * nb + iab.x], 0), nb),
            prm.list_idx + (bh * nb + (iab.y >= 0 ? iab.y : iab.x)) * static_cast<long long>(nb),
            iab.y >= 0 ? min(max(prm.list_cnt[bh * nb + iab.y], 0), nb) : 0, lane);
    int it = 0;
    bool ended = false;
    while (true) {
      uint32_t f = 0;
      const int j = wk.next(&f, lane);
      const int s = it % L::kStages;
      const int n = it / L::kStages;
      int ok = 1;
      if (lane == 0 && n > 0) ok = mbar_wait(&empty[s], (n - 1) & 1, prm.status, kDevTimeoutKvEmpty) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (j < 0 || j >= nb) {
        if (lane == 0) {
          meta[s] = kEnd;
          mbar_arrive(&full[s]);
        }
        ended = true;
        break;
      }
      if (lane == 0) {
        meta[s] = static_cast<uint32_t>(j) | (f << 28);
        unsigned char* st = sStage + s * L::kStageBytes;
        mbar_arrive_expect_tx(&full[s], 2 * C::kTileBytes);
        const int krow = static_cast<int>(bh * prm.S + static_cast<long long>(j) * 64);
        // one copy per operand: all D columns of the 64 rows (panels 8 KB apart)
        tma_load_3d(st, &map_k64, &full[s], 0, krow, 0);
        tma_load_3d(st + C::kTileBytes, &map_v64, &full[s], 0, krow, 0);
      }
      ++it;
    }
    if (lane == 0) {
      // Copies still in flight (as in the dK/dV pass).
      const int keep = ended ? L::kStages - 1 : L::kStages;
      const int first = it > keep ? it - keep : 0;
      for (int x = first; x < it; ++x)
        mbar_wait(&full[x % L::kStages], (x / L::kStages) & 1, prm.status, kDevTimeoutDrain);
      mbar_wait(q_full, 0, prm.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f16_f32(128, 64, false, false);
      constexpr uint32_t idesc_acc = idesc_f16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ), do_addr = smem_u32(sDO);
      const uint32_t st_addr = smem_u32(sStage);
      // S = Q K_j^T and dP = dO V_j^T into buffer x & 1
      auto issue_sd = [&](int x) {
        const int s = x % L::kStages;
        const uint32_t ka = st_addr + s * L::kStageBytes;
        const uint32_t va = ka + C::kTileBytes;
        const uint32_t col = (x & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2, w = kk & 3;
          mma_bf16_ss(tmem + col, sdesc_sw128(q_addr + pn * 16384 + w * 32, 16, 1024),
                      sdesc_sw128(ka + pn * 8192 + w * 32, 16, 1024), idesc_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2, w = kk & 3;
          mma_bf16_ss(tmem + col + 64, sdesc_sw128(do_addr + pn * 16384 + w * 32, 16, 1024),
                      sdesc_sw128(va + pn * 8192 + w * 32, 16, 1024), idesc_s, kk > 0);
        }
        mma_commit(&sd_full[x & 1]);
      };
      // dQ += dS K_j with dS read from TMEM (written over dP)
      auto issue_acc = [&](int x) {
        const int s = x % L::kStages;
        const uint32_t ka = st_addr + s * L::kStageBytes;
        const uint32_t col = (x & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ts(tmem + C::kColAcc0, tmem + col + 64 + packed_col(kk), sdesc_sw128(ka + kk * 2048, 8192, 1024),
                      idesc_acc, (x > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(q_full, 0, prm.status, kDevTimeoutQFull);
      if (ok) ok = mbar_wait(&full[0], 0, prm.status, kDevTimeoutTmaFull);
      if (ok && meta[0] != kEnd) {
        tc_fence_after();
        issue_sd(0);
        for (int it = 0;; ++it) {
          const int s1 = (it + 1) % L::kStages;
          if (!mbar_wait(&full[s1], ((it + 1) / L::kStages) & 1, prm.status, kDevTimeoutTmaFull)) break;
          const bool end1 = meta[s1] == kEnd;
          tc_fence_after();
          if (!end1) issue_sd(it + 1);
          if (!mbar_wait(&p_full[it & 1], (it >> 1) & 1, prm.status, kDevTimeoutPFull)) break;
          tc_fence_after();
          issue_acc(it);
          mma_commit(&empty[it % L::kStages]);
          if (end1) break;
        }
      }
      mma_commit(acc_bar);
      mma_commit(drain);
      mbar_wait(drain, 0, prm.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp >= kMathWarp0) {
    // 8 warps: query row = TMEM lane, column half h of each 64-key tile
    const int mw = warp - kMathWarp0;
    const int h = mw >> 2;
    const int row = (mw & 3) * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>((mw & 3) * 32) << 16;
    const bool upper = row >= 64;
    const int blk = upper ? iab.y : iab.x;
    const bool valid = blk >= 0;
    // tok: the row in the reordered order (lse2 and delta); otok: where dQ goes
    const long long tok = bh * prm.S + static_cast<long long>(valid ? blk : 0) * 64 + (row & 63);
    const long long otok = prm.nat.on ? prm.nat.token(bh, valid ? blk : 0, row & 63) : tok;
    const float my_lse2 = valid ? prm.lse2[tok] : 0.f;
    const float my_delta = valid ? prm.delta[tok] : 0.f;
    const float sl2 = prm.scale_log2;
    int it = 0;
    bool ok = true;
    for (;; ++it) {
      const int s = it % L::kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (it / L::kStages) & 1, prm.status, kDevTimeoutTmaFull));
      if (!ok) break;
      const uint32_t mt = meta[s];
      if (mt == kEnd) break;
      const bool keep = upper ? ((mt >> 29) & 1u) : ((mt >> 28) & 1u);
      ok = __all_sync(0xffffffffu, mbar_wait(&sd_full[it & 1], (it >> 1) & 1, prm.status, kDevTimeoutSFull));
      if (!ok) break;
      tc_fence_after();
      const uint32_t col = tmem + lane_base + (it & 1) * 128 + 32 * h;
      uint32_t dk[16];
      if (keep) {
        uint32_t sv[32], dv[32];
        tmem_ld32(col, sv);
        tmem_ld32(col + 64, dv);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(sv[c]), sl2, -my_lse2));
          const float p1 = fast_exp2(fmaf(__uint_as_float(sv[c + 1]), sl2, -my_lse2));
          dk[c >> 1] = pack_f16x2(p0 * (__uint_as_float(dv[c]) - my_delta),
                                  p1 * (__uint_as_float(dv[c + 1]) - my_delta));
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) dk[c] = 0u;
      }
      tmem_st16(col + 64, dk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[it & 1]);
    }
    bool have = ok && it > 0;
    if (have) {
      have = __all_sync(0xffffffffu, mbar_wait(acc_bar, 0, prm.status, kDevTimeoutOBar));
      tc_fence_after();
    }
    if (have) {
      // the stage ring is free (as in the dK/dV pass): 32 rows x 64 columns of dQ per warp
      unsigned char* stage = sStage + mw * (D / 2) * 4 * 32;
#pragma unroll 1
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        uint32_t ov[32];
        tmem_ld32(tmem + lane_base + C::kColAcc0 + (D / 2) * h + c0, ov);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * prm.scale);
        if (valid)
          store_rows_f32(&map_out0, stage, ov, lane, (D / 2) * h + c0, bh, blk, (mw & 3) & 1, prm.nat, prm.T);
        stage += 4096;
      }
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
    } else {
#pragma unroll 1
      for (int c0 = 0; c0 < D / 2; c0 += 4)
        if (valid) *reinterpret_cast<float4*>(prm.out0 + otok * D + (D / 2) * h + c0) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D>
cudaError_t launch_bwd(const void* q, const void* k, const void* v, int v_f16, const void* o, int o_f32,
                       const void* dout, const float* lse, const int32_t* ridx, const int32_t* rcnt,
                       const int32_t* cidx, const int32_t* ccnt, const Dims& d, float scale,
                       float* dq, float* dk, float* dv, void* ws, cudaStream_t st, bool* map_ok,
                       bool natural) {
  NatMap nat;
  nat.on = natural ? 1 : 0;
  nat.HW = d.Hb * d.Wb;
  nat.Wb = d.Wb;
  nat.Hg = d.Hg;
  nat.W = d.W;
  nat.S = d.S;
  const long long rows = static_cast<long long>(d.BH) * d.S;
  float* delta = reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes);
  float* lse2 = delta + align_up(static_cast<size_t>(rows), 64);
  char* sched = reinterpret_cast<char*>(lse2 + align_up(static_cast<size_t>(rows), 64));
  __half* h16 = reinterpret_cast<__half*>(sched + 2 * schedule_scratch_bytes(d));
  const size_t tensor_elems = static_cast<size_t>(rows) * D;
  __half *q16 = h16, *k16 = h16 + tensor_elems, *v16 = h16 + 2 * tensor_elems,
         *do16 = h16 + 3 * tensor_elems;
  uint32_t* status = static_cast<uint32_t*>(ws);
  int32_t* order_cols = nullptr;
  int32_t* order_rows = nullptr;
  // key-block pairs and query-block pairs both follow tile_blocks() (same patch, frames
  // 2u and 2u + 1), whose kept lists overlap most
  cudaError_t e = build_schedule(ccnt, nullptr, d, sched, &order_cols, st, /*frame_pairs=*/true);
  if (e == cudaSuccess)
    e = build_schedule(rcnt, nullptr, d, sched + schedule_scratch_bytes(d), &order_rows, st, /*frame_pairs=*/true);
  if (e != cudaSuccess) return e;
  constexpr int kRowsPerCta = 8 * (256 / D);
  if (v_f16 && !natural) v16 = static_cast<__half*>(const_cast<void*>(v));   // used as it is
  bwd_preprocess_kernel<D><<<static_cast<unsigned>((rows + kRowsPerCta - 1) / kRowsPerCta), 256, 0, st>>>(
      o, o_f32, static_cast<const __nv_bfloat16*>(dout), lse, static_cast<const __nv_bfloat16*>(q),
      static_cast<const __nv_bfloat16*>(k), v, v_f16, q16, k16, v16,
      do16, delta, lse2, rows, status, nat);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // per-panel maps for the resident 128-row operands (two 64-row blocks per panel), and
  // one-copy maps (panels as the outermost dimension) for the streamed 64-row stages
  CUtensorMap mq64, mdo64, mk64, mv64, mq3, mdo3, mk3, mv3;
  *map_ok = make_map_16(&mq64, q16, rows, D, 64, true) && make_map_16(&mdo64, do16, rows, D, 64, true) &&
            make_map_16(&mk64, k16, rows, D, 64, true) && make_map_16(&mv64, v16, rows, D, 64, true) &&
            make_map_kv(&mq3, q16, rows, D, true) && make_map_kv(&mdo3, do16, rows, D, true) &&
            make_map_kv(&mk3, k16, rows, D, true) && make_map_kv(&mv3, v16, rows, D, true);
  if (!*map_ok) return cudaErrorInvalidValue;
  // f32 gradient maps for the epilogues' tiled stores
  CUtensorMap mdq, mdk, mdv;
  const long long frames = static_cast<long long>(d.BH) * d.T;
  *map_ok = natural ? (make_map_nat_f32(&mdq, dq, frames, d.Hg, d.W, D) &&
                       make_map_nat_f32(&mdk, dk, frames, d.Hg, d.W, D) &&
                       make_map_nat_f32(&mdv, dv, frames, d.Hg, d.W, D))
                    : (make_map_f32(&mdq, dq, rows, D) && make_map_f32(&mdk, dk, rows, D) &&
                       make_map_f32(&mdv, dv, rows, D));
  if (!*map_ok) return cudaErrorInvalidValue;

  BwdParams p;
  p.delta = delta;
  p.lse2 = lse2;
  p.status = status;
  p.nb = d.nb;
  p.T = d.T;
  p.HW = d.Hb * d.Wb;
  p.S = d.S;
  p.scale_log2 = scale * kLog2e;
  p.scale = scale;
  p.nat = nat;
  const unsigned grid = static_cast<unsigned>(d.BH) * static_cast<unsigned>((d.nb + 1) / 2);
  p.npairs = (d.nb + 1) / 2;

  p.order = order_cols;
  p.list_idx = cidx;
  p.list_cnt = ccnt;
  p.out0 = dv;
  p.out1 = dk;
  e = cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           DkdvLayout<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_bwd_dkdv_kernel<D><<<grid, kThreads, DkdvLayout<D>::kSmemBytes, st>>>(mq3, mdo3, mk64, mv64, mdv, mdk, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  p.order = order_rows;
  p.list_idx = ridx;
  p.list_cnt = rcnt;
  p.out0 = dq;
  p.out1 = nullptr;
  e = cudaFuncSetAttribute(attn_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           DqLayout<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_bwd_dq_kernel<D><<<grid, kThreads, DqLayout<D>::kSmemBytes, st>>>(mq64, mdo64, mk3, mv3, mdq, p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace nabla

using namespace nabla;

extern "C" size_t nabla_bwd_workspace_bytes(nabla_shape s) {
  Dims d;
  if (check_shape(s, &d) != NABLA_OK) return 0;
  const size_t rows = align_up(static_cast<size_t>(d.BH) * d.S, 64);
  return kStatusBytes + 2 * rows * sizeof(float) + 2 * schedule_scratch_bytes(d) +
         4 * static_cast<size_t>(d.BH) * d.S * d.D * 2;
}

extern "C" nabla_status nabla_attn_bwd(const void* q, const void* k, const void* v,
                                       nabla_dtype v_dtype, const void* o,
                                       nabla_dtype o_dtype, const void* dout, const float* lse,
                                       const int32_t* row_idx, const int32_t* row_cnt,
                                       const int32_t* col_idx, const int32_t* col_cnt,
                                       nabla_shape s, float scale, float* dq, float* dk, float* dv,
                                       nabla_layout layout, void* workspace, size_t workspace_bytes,
                                       nabla_stream_t stream) {
  Dims d;
  nabla_status rc = check_shape(s, &d);
  if (rc != NABLA_OK) return rc;
  if (!q || !k || !v || !o || !dout || !lse || !row_idx || !row_cnt || !col_idx || !col_cnt ||
      !dq || !dk || !dv)
    return NABLA_ERR_INVALID_ARG;
  const void* al16[] = {q, k, v, o, dout, lse, dq, dk, dv};
  for (const void* p : al16)
    if (!aligned16(p)) return NABLA_ERR_INVALID_ARG;
  const void* al4[] = {row_idx, row_cnt, col_idx, col_cnt};
  for (const void* p : al4)
    if (reinterpret_cast<uintptr_t>(p) & 3) return NABLA_ERR_INVALID_ARG;
  if (o_dtype != NABLA_BF16 && o_dtype != NABLA_F32) return NABLA_ERR_INVALID_ARG;
  if (v_dtype != NABLA_BF16 && v_dtype != NABLA_F16) return NABLA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return NABLA_ERR_INVALID_ARG;
  if (layout != NABLA_LAYOUT_REORDERED && layout != NABLA_LAYOUT_NATURAL) return NABLA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < nabla_bwd_workspace_bytes(s) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return NABLA_ERR_WORKSPACE;
  if (static_cast<long long>(d.BH) * d.S >= (1ll << 31)) return NABLA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_status(e);
  bool map_ok = true;
  e = d.D == 64 ? launch_bwd<64>(q, k, v, v_dtype == NABLA_F16, o, o_dtype == NABLA_F32, dout, lse, row_idx, row_cnt, col_idx,
                                 col_cnt, d, scale, dq, dk, dv, workspace, st, &map_ok,
                                 layout == NABLA_LAYOUT_NATURAL)
                : launch_bwd<128>(q, k, v, v_dtype == NABLA_F16, o, o_dtype == NABLA_F32, dout, lse, row_idx, row_cnt, col_idx,
                                  col_cnt, d, scale, dq, dk, dv, workspace, st, &map_ok,
                                  layout == NABLA_LAYOUT_NATURAL);
  return cuda_status(e);
}
