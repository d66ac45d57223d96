// Block-sparse flash-attention forward over the kept 64 x 64 tiles (sm_100a).
//
// "NABLA: Neighborhood Adaptive Block-Level Attention" (gist.science, Chinese edition),
// technical summary, Methodology, "expansion": each kept entry (i, j) of the pooled
// block mask is one full N x N tile of the token attention matrix, computed exactly;
// the pages run this through FlexAttention.  Here it is a hand-written kernel:
//
//  * one CTA = one tile of 128 query rows = two consecutive query blocks (2p, 2p+1) of
//    one head, so the tensor core runs M = 128 MMAs; the CTA walks the ascending union
//    of the two blocks' kept-key lists and masks (-inf) the half of the rows whose block
//    does not keep the current key block;
//  * warp 0 (one lane) streams K and V tiles with TMA (128-byte swizzle) into a ring of
//    shared-memory stages; warp 1 (one lane) issues tcgen05.mma: S = Q K^T into one of two
//    TMEM score buffers, and O += P V into a TMEM accumulator; warps 4-7 run the online
//    softmax, one query row per thread (TMEM lane = row), write P (bf16) into shared
//    memory for the second MMA, and rescale O only when a row maximum grows by more
//    than 2^8 (conditional rescaling);
//  * the epilogue divides by the row sum and writes O (bf16 or f32) and the natural-log
//    LSE.  Every barrier wait is bounded; a timeout records a status code and the CTA
//    drains its own copies / MMAs and frees TMEM before returning.
#include <math.h>

#include <cudaTypedefs.h>

#include "common.cuh"

namespace nabla {
namespace {

constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;          // warps 4..7
constexpr uint32_t kEnd = 0xFFFFFFFFu;    // end-of-list marker in the stage metadata

template <int D>
struct FwdCfg {
  static constexpr int kPanels = D / 64;                  // 128-byte swizzle panels
  static constexpr int kStages = (D == 128) ? 2 : 4;   // two CTAs per SM
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVTileBytes = 64 * D * 2;         // one K or one V tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kKVTileBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 256;              // S0 | S1 | O
  static constexpr uint32_t kColS0 = 0, kColS1 = 64, kColO = 128;
};

struct FwdParams {
  const int32_t* order;      // work items (head * npairs + pair), longest first
  int npairs;
  const int32_t* row_idx;
  const int32_t* row_cnt;
  void* o;
  float* lse;
  uint32_t* status;
  int nb;
  long long S;
  float scale_log2;
  int o_f32;
};

template <int D, bool VF16>
__global__ void __launch_bounds__(kThreads, 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const FwdParams prm) {
  using C = FwdCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sK = smem + C::kOffK;
  unsigned char* sV = smem + C::kOffV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;                       // [kStages]
  uint64_t* empty = bars + C::kStages;         // [kStages]
  uint64_t* q_full = bars + 2 * C::kStages;
  uint64_t* s_full = q_full + 1;               // [2]
  uint64_t* p_full = s_full + 2;               // [2]
  uint64_t* o_bar = p_full + 2;                // one phase per PV (rescale waits)
  uint64_t* o_final = o_bar + 1;               // single phase: every PV has landed
  uint64_t* drain = o_final + 1;
  uint32_t* meta = reinterpret_cast<uint32_t*>(drain + 1);   // [kStages]
  uint32_t* tmem_slot = meta + C::kStages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int item = prm.order[blockIdx.x];
  const long long bh = item / prm.npairs;
  const int pair = item - static_cast<int>(bh) * prm.npairs;
  const int nb = prm.nb;
  const int i0 = 2 * pair;
  const bool has_i1 = (i0 + 1) < nb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_full[0], 128);
    mbar_init(&p_full[1], 128);
    mbar_init(o_bar, 1);
    mbar_init(o_final, 1);
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
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      const int qrow = static_cast<int>(bh * prm.S + static_cast<long long>(i0) * 64);
      mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
      for (int pn = 0; pn < C::kPanels; ++pn)
        tma_load_2d(sQ + pn * (128 * 128), &map_q, q_full, pn * 64, qrow);
      const int32_t* l0 = prm.row_idx + (bh * nb + i0) * static_cast<long long>(nb);
      const int32_t* l1 = l0 + nb;
      const int c0 = min(max(prm.row_cnt[bh * nb + i0], 0), nb);
      const int c1 = has_i1 ? min(max(prm.row_cnt[bh * nb + i0 + 1], 0), nb) : 0;
      int a = 0, b = 0, it = 0;
      bool ok = true, ended = false;
      while (true) {
        int j = -1;
        uint32_t f = 0;
        if (a < c0 && b < c1) {
          const int ja = l0[a], jb = l1[b];
          if (ja < jb) { j = ja; f = 1; ++a; }
          else if (jb < ja) { j = jb; f = 2; ++b; }
          else { j = ja; f = 3; ++a; ++b; }
        } else if (a < c0) { j = l0[a++]; f = 1; }
        else if (b < c1) { j = l1[b++]; f = 2; }
        const int s = it % C::kStages;
        const int n = it / C::kStages;
        if (n > 0 && !mbar_wait(&empty[s], (n - 1) & 1, prm.status, kDevTimeoutKvEmpty)) { ok = false; break; }
        if (j < 0) {
          meta[s] = kEnd;
          mbar_arrive(&full[s]);
          ended = true;
          break;
        }
        meta[s] = static_cast<uint32_t>(j) | (f << 28);
        mbar_arrive_expect_tx(&full[s], 2 * C::kKVTileBytes);
        const int krow = static_cast<int>(bh * prm.S + static_cast<long long>(j) * 64);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn) {
          tma_load_2d(sK + s * C::kKVTileBytes + pn * 8192, &map_k, &full[s], pn * 64, krow);
          tma_load_2d(sV + s * C::kKVTileBytes + pn * 8192, &map_v, &full[s], pn * 64, krow);
        }
        ++it;
      }
      // Drain: every issued copy must have landed before the CTA may exit.
      (void)ok;
      // Copies still in flight: the last kStages iterations, except that placing the end
      // marker waited for the oldest of them to be consumed (its stage was reused), and a
      // parity wait on that stage would now look two phases back.
      const int keep = ended ? C::kStages - 1 : C::kStages;
      const int first = it > keep ? it - keep : 0;
      for (int x = first; x < it; ++x)
        mbar_wait(&full[x % C::kStages], (x / C::kStages) & 1, prm.status, kDevTimeoutDrain);
      mbar_wait(q_full, 0, prm.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idesc_o = VF16 ? idesc_f16_f32(128, D, false, true)
                                        : idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const uint32_t v_addr = smem_u32(sV);
      auto issue_s = [&](int x) {
        const int st = x % C::kStages;
        const uint32_t d_tmem = tmem + ((x & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int pn = kk >> 2, w = kk & 3;
          const uint64_t ad = sdesc_sw128(q_addr + pn * (128 * 128) + w * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(k_addr + st * C::kKVTileBytes + pn * 8192 + w * 32, 16, 1024);
          mma_bf16_ss(d_tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[x & 1]);
      };
      // O += P V with P (bf16) read from TMEM where the softmax warps stored it, over the
      // first 32 columns of the score buffer it came from.
      auto issue_pv = [&](int x) {
        const int st = x % C::kStages;
        const uint32_t p_tmem = tmem + ((x & 1) ? C::kColS1 : C::kColS0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = sdesc_sw128(v_addr + st * C::kKVTileBytes + kk * 2048, 8192, 1024);
          mma_bf16_ts(tmem + C::kColO, p_tmem + kk * 8, bd, idesc_o, (x > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, prm.status, kDevTimeoutQFull);
      if (ok) ok = mbar_wait(&full[0], 0, prm.status, kDevTimeoutTmaFull);
      if (ok && meta[0] != kEnd) {
        tc_fence_after();
        issue_s(0);
        for (int it = 0;; ++it) {
          const int s1 = (it + 1) % C::kStages;
          const int n1 = (it + 1) / C::kStages;
          if (!mbar_wait(&full[s1], n1 & 1, prm.status, kDevTimeoutTmaFull)) break;
          const bool end1 = meta[s1] == kEnd;
          tc_fence_after();
          if (!end1) issue_s(it + 1);
          if (!mbar_wait(&p_full[it & 1], (it >> 1) & 1, prm.status, kDevTimeoutPFull)) break;
          tc_fence_after();
          issue_pv(it);
          mma_commit(&empty[it % C::kStages]);
          mma_commit(o_bar);
          if (end1) break;
        }
      }
      // o_final completes once when every MMA issued above has finished; the epilogue
      // waits on it (a per-PV parity wait could be satisfied two phases early).
      mma_commit(o_final);
      // Drain: all MMAs of this CTA complete before TMEM is released.
      mma_commit(drain);
      mbar_wait(drain, 0, prm.status, kDevTimeoutDrain);
    }
    __syncwarp();
  } else if (warp >= kSoftmaxWarp0) {
    // ------------------------------------------------------------------ softmax + epilogue
    const int row = threadIdx.x - kSoftmaxWarp0 * 32;            // 0..127 = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp - kSoftmaxWarp0) * 32) << 16;
    const bool upper = row >= 64;
    const float sl2 = prm.scale_log2;
    float m_ref = -INFINITY;
    float l = 0.f;
    int it = 0;
    bool ok = true;
    for (;; ++it) {
      const int s = it % C::kStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (it / C::kStages) & 1, prm.status, kDevTimeoutTmaFull));
      if (!ok) break;
      const uint32_t mt = meta[s];
      if (mt == kEnd) break;
      const bool keep = upper ? ((mt >> 29) & 1u) : ((mt >> 28) & 1u);
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[it & 1], (it >> 1) & 1, prm.status, kDevTimeoutSFull));
      if (!ok) break;
      tc_fence_after();
      uint32_t sa[32], sb[32];
      {
        const uint32_t col = (it & 1) ? C::kColS1 : C::kColS0;
        tmem_ld32(tmem + lane_base + col, sa);
        tmem_ld32(tmem + lane_base + col + 32, sb);
        tmem_wait_ld();
      }
      float factor = 1.f;
      bool rescale = false;
      if (keep) {
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) mx = fmaxf(mx, fmaxf(__uint_as_float(sa[c]), __uint_as_float(sb[c])));
        const float rm = mx * sl2;
        if (rm > m_ref + 8.0f) {
          if (m_ref != -INFINITY) {
            factor = fast_exp2(m_ref - rm);
            rescale = true;
          }
          m_ref = rm;
        }
      }
      // Warp-uniform O correction (tcgen05.ld/st are warp-collective); lanes that do not
      // rescale multiply by 1.
      if (__any_sync(0xffffffffu, rescale)) {
        l *= factor;
        // O holds the sum of the previous iterations; wait for the last PV to land.
        ok = __all_sync(0xffffffffu, mbar_wait(o_bar, (it - 1) & 1, prm.status, kDevTimeoutOBar));
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_base + C::kColO + c0, ov);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * factor);
          tmem_st32(tmem + lane_base + C::kColO + c0, ov);
        }
        tmem_wait_st();
      }
      // P = 2^(s*scale*log2e - m) as bf16 pairs, written over the score buffer in TMEM.
      // Every fourth element uses the FMA-pipe exponential to offload the MUFU unit.
      const uint32_t pcol = tmem + lane_base + ((it & 1) ? C::kColS1 : C::kColS0);
      float sum = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t (&sv)[32] = half ? sb : sa;
        uint32_t packed[16];
        if (keep) {
#pragma unroll
          for (int c = 0; c < 16; c += 2) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * c]), sl2, -m_ref));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * c + 1]), sl2, -m_ref));
            const float p2 = fast_exp2(fmaf(__uint_as_float(sv[2 * c + 2]), sl2, -m_ref));
            const float p3 = poly_exp2(fmaf(__uint_as_float(sv[2 * c + 3]), sl2, -m_ref));
            // The row sum takes the rounded weights that enter the PV product, so the
            // output is an exact convex combination of those weights.
            if constexpr (VF16) {
              packed[c] = pack_f16x2(p0, p1);
              packed[c + 1] = pack_f16x2(p2, p3);
              sum += (f16lo(packed[c]) + f16hi(packed[c])) + (f16lo(packed[c + 1]) + f16hi(packed[c + 1]));
            } else {
              packed[c] = pack_bf16x2(p0, p1);
              packed[c + 1] = pack_bf16x2(p2, p3);
              sum += (bf16lo(packed[c]) + bf16hi(packed[c])) + (bf16lo(packed[c + 1]) + bf16hi(packed[c + 1]));
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) packed[c] = 0u;
        }
        tmem_st16(pcol + half * 16, packed);
      }
      l += sum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[it & 1]);
    }
    // ---- epilogue -----------------------------------------------------------------------
    const int nit = it;
    const bool valid_row = upper ? has_i1 : true;
    const long long tok = bh * prm.S + static_cast<long long>(i0) * 64 + row;
    bool have_o = ok && nit > 0;
    if (have_o) {
      have_o = __all_sync(0xffffffffu, mbar_wait(o_final, 0, prm.status, kDevTimeoutOBar));
      tc_fence_after();
    }
    const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t ov[32];
      if (have_o) {
        tmem_ld32(tmem + lane_base + C::kColO + c0, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) ov[c] = 0u;
      }
      if (valid_row) {
        if (prm.o_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(prm.o) + tok * D + c0);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_float4(__uint_as_float(ov[4 * c]) * inv_l, __uint_as_float(ov[4 * c + 1]) * inv_l,
                                 __uint_as_float(ov[4 * c + 2]) * inv_l, __uint_as_float(ov[4 * c + 3]) * inv_l);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.o) + tok * D + c0);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            dst[c] = make_uint4(pack_bf16x2(__uint_as_float(ov[8 * c]) * inv_l, __uint_as_float(ov[8 * c + 1]) * inv_l),
                                pack_bf16x2(__uint_as_float(ov[8 * c + 2]) * inv_l, __uint_as_float(ov[8 * c + 3]) * inv_l),
                                pack_bf16x2(__uint_as_float(ov[8 * c + 4]) * inv_l, __uint_as_float(ov[8 * c + 5]) * inv_l),
                                pack_bf16x2(__uint_as_float(ov[8 * c + 6]) * inv_l, __uint_as_float(ov[8 * c + 7]) * inv_l));
        }
      }
    }
    if (valid_row && prm.lse != nullptr)
      prm.lse[tok] = (l > 0.f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
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
            make_map_16(&mv, v, rows, D, 64, VF16);
  if (!*map_ok) return cudaErrorInvalidValue;
  using C = FwdCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, VF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const unsigned items = static_cast<unsigned>(d.BH) * static_cast<unsigned>((d.nb + 1) / 2);
  attn_fwd_kernel<D, VF16><<<items, kThreads, C::kSmemBytes, st>>>(mq, mk, mv, prm);
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
                                       nabla_dtype v_dtype, const int32_t* row_idx, const int32_t* row_cnt,
                                       nabla_shape s, float scale, void* o, nabla_dtype o_dtype,
                                       float* lse, void* workspace, size_t workspace_bytes,
                                       nabla_stream_t stream) {
  Dims d;
  nabla_status rc = check_shape(s, &d);
  if (rc != NABLA_OK) return rc;
  if (!q || !k || !v || !o || !row_idx || !row_cnt) return NABLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return NABLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(row_idx) & 3) || (reinterpret_cast<uintptr_t>(row_cnt) & 3) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
    return NABLA_ERR_INVALID_ARG;
  if (o_dtype != NABLA_BF16 && o_dtype != NABLA_F32) return NABLA_ERR_INVALID_ARG;
  if (v_dtype != NABLA_BF16 && v_dtype != NABLA_F16) return NABLA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return NABLA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < nabla_fwd_workspace_bytes(s) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return NABLA_ERR_WORKSPACE;
  if (static_cast<long long>(d.BH) * d.S >= (1ll << 31)) return NABLA_ERR_UNSUPPORTED;
  FwdParams prm;
  prm.row_idx = row_idx;
  prm.row_cnt = row_cnt;
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
  ce = build_schedule(row_cnt, d, static_cast<char*>(workspace) + kStatusBytes, &order, st);
  if (ce != cudaSuccess) return cuda_status(ce);
  prm.order = order;
  prm.npairs = (d.nb + 1) / 2;
  bool map_ok = true;
  const bool vf16 = v_dtype == NABLA_F16;
  cudaError_t e = d.D == 64 ? (vf16 ? launch_fwd<64, true>(q, k, v, d, prm, st, &map_ok)
                                    : launch_fwd<64, false>(q, k, v, d, prm, st, &map_ok))
                            : (vf16 ? launch_fwd<128, true>(q, k, v, d, prm, st, &map_ok)
                                    : launch_fwd<128, false>(q, k, v, d, prm, st, &map_ok));
  return cuda_status(e);
}
