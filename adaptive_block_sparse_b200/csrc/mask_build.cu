// Adaptive block mask: pooled scores, row softmax, CDF threshold, STA union, bitmask and
// row / column lists.
//
// "NABLA: Neighborhood Adaptive Block-Level Attention" (gist.science, Chinese edition),
// technical summary, Methodology, "adaptive mask construction": Q and K are pooled per
// block, full attention is computed on the pooled map, and per row the blocks whose
// cumulative probability exceeds 1 - thr are kept; "hybrid integration with STA": the
// final mask is the union with a static window mask.  lsdiaocha.cn article, section 4:
// sort each row and accumulate the probability.
//
// Decision precision: this kernel takes the whole decision in fp64 (pooled means,
// logits, softmax, ranked mass), so it agrees with an fp64 statement of the method
// except for blocks whose ranked mass lies within rounding (~1e-15) of thr.  It serves
// as the exact tier: for every row when the fast tier does not apply, and for the rows
// the fast tier could not certify.
//
// Selection without a sort: block j is kept iff E_j < thr, where E_j is the mass ranked
// strictly before j (probability descending, ties by lower index).  The kept set is a
// prefix of that ranking, so it is found by narrowing an interval of fp64 bit patterns
// of the probabilities (non-negative doubles order like their bit patterns) where the
// "mass at or above" crosses thr until it holds at most a few blocks; those are ranked
// (probability descending, index ascending) and walked in order.  The logits are
// computed with fp64 tensor-core MMA (m8n8k4), two key tiles per warp at a time, the
// dims permuted so that each key's mean is read in whole 128-byte lines.
#include <math.h>

#include "common.cuh"

namespace nabla {

cudaError_t pool_blocks_device(const void* x, double* pool, const Dims& d, cudaStream_t st, bool natural);
cudaError_t mask_fast_prepare_tokens(const void* q, const void* k, bool natural, double* qp_out,
                                     double* kp_out, const Dims& d, double scale, void* scratch,
                                     uint32_t* status, cudaStream_t st);
size_t mask_fast_scratch_bytes(const Dims& d);
bool mask_fast_supported(const Dims& d);
cudaError_t mask_fast_prepare(const double* qp, const double* kp, const Dims& d, double scale,
                              void* scratch, uint32_t* status, cudaStream_t st);
cudaError_t mask_fast_select(const Dims& d, double scale, double thr, const nabla_window& w,
                             uint32_t* bits, int32_t* ridx, int32_t* rcnt, void* scratch,
                             int32_t** rescue_list, int32_t** rescue_cnt, cudaStream_t st);

namespace {

constexpr int kThreads = 256;   // 8 warps; one pooled row per warp during selection
                                // (two CTAs per SM where shared memory allows)
constexpr int kWarps = kThreads / 32;
constexpr int kRowBudget = 163840;  // bytes of shared memory for the fp64 score rows
constexpr int kCand = 16;       // the cut's search stops at this many candidates

template <int D>
__global__ void __launch_bounds__(kThreads, 2) mask_rows_kernel(
    const double* __restrict__ qpool, const double* __restrict__ kpool, int nb, int nw, int R,
    double scale, double thr, int sta_on, int wt2, int wh2, int ww2, int Hb, int Wb,
    uint32_t* __restrict__ bits, int32_t* __restrict__ row_idx, int32_t* __restrict__ row_cnt,
    const int32_t* __restrict__ rlist, const int32_t* __restrict__ rlist_cnt, int BH) {
  // Rows: R consecutive rows from blockIdx.x * R of head blockIdx.y, or (rlist != nullptr)
  // the listed rows: group g of head h = rows rlist[h*nb + gR ...], R at a time; the
  // groups of all heads are numbered head after head and CTA c takes every gridDim.x-th
  // one from c, so a few heads with many listed rows spread over every SM.
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int rows_s[8];
  __shared__ unsigned long long cand_key[kWarps * kCand];   // per warp: cut candidates
  __shared__ int cand_idx[kWarps * kCand];
  __shared__ int cand_keep[kWarps * kCand];
  double* qs = reinterpret_cast<double*>(smem_raw);                             // 8 x D
  double* prow = qs + 8 * D;                                                    // R x nb

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  long long bh = blockIdx.y;
  int listed = 0;
  int hh = -1;                    // rescue mode: head of the current group,
  long long hbase = 0, hnext = 0; // whose groups are [hbase, hnext) in the global numbering
  for (long long u = rlist != nullptr ? blockIdx.x : 0;; u += gridDim.x) {
  int nrows, g;
  if (rlist != nullptr) {
    while (u >= hnext && hh < BH) {
      ++hh;
      if (hh >= BH) break;
      listed = min(max(rlist_cnt[hh], 0), nb);
      hbase = hnext;
      hnext += (listed + R - 1) / R;
    }
    if (hh >= BH) break;
    bh = hh;
    g = static_cast<int>(u - hbase);
    nrows = min(R, listed - g * R);
  } else {
    if (u > 0) break;
    g = 0;
    nrows = min(R, nb - static_cast<int>(blockIdx.x) * R);
  }
  __syncthreads();
  if (tid < R)
    rows_s[tid] = tid < nrows ? (rlist != nullptr ? rlist[bh * nb + g * R + tid]
                                                  : static_cast<int>(blockIdx.x) * R + tid)
                              : 0;
  __syncthreads();

  for (int e = tid; e < 8 * D; e += kThreads) {
    const int r = e / D;
    qs[e] = (r < nrows) ? qpool[(bh * nb + rows_s[r]) * D + (e - r * D)] : 0.0;
  }
  // ---- pooled logits A = Qp Kp^T * scale (fp64 tensor-core MMA, m8n8k4) ---------------
  // The (up to 8) rows of the group are the M = 8 side; each warp takes 8 key blocks at a
  // time (N = 8) and walks D in steps of 4.  Fragments: A[row = lane/4][k = lane%4],
  // B[k = lane%4][key = lane/4], C[row = lane/4][key = 2*(lane%4) + {0,1}].  The dot
  // product runs over the D dims in a permuted order: step kk, lane k takes dim
  // 16 (kk / 4) + 4 k + kk % 4, so that over four steps the four lanes of a key read one
  // 128-byte line of the key's mean, each lane 32 contiguous bytes (two 16-byte loads when
  // the means are 16-byte aligned), instead of 32 bytes of the line per step.
  __syncthreads();
  {
    const int gid = lane >> 2, tig = lane & 3;
    double afrag[D / 4];
#pragma unroll
    for (int kk = 0; kk < D / 4; ++kk) afrag[kk] = qs[gid * D + 16 * (kk >> 2) + 4 * tig + (kk & 3)];
    const bool vec = (reinterpret_cast<uintptr_t>(kpool) & 15) == 0;   // uniform
    // Two 8-key tiles per iteration: two independent accumulation chains, their key
    // loads in flight together.
    for (int jt = warp; jt * 8 < nb; jt += 2 * kWarps) {
      const int jt2 = jt + kWarps;
      const bool two = jt2 * 8 < nb;               // warp-uniform
      const int key = jt * 8 + gid, key2 = jt2 * 8 + gid;
      const bool v1 = key < nb, v2 = two && key2 < nb;
      const double* kr = kpool + (bh * nb + (v1 ? key : 0)) * D + 4 * tig;
      const double* kr2 = kpool + (bh * nb + (v2 ? key2 : 0)) * D + 4 * tig;
      double c0 = 0.0, c1 = 0.0, c2 = 0.0, c3 = 0.0;
#pragma unroll
      for (int g4 = 0; g4 < D / 16; ++g4) {
        double b[4], b2[4];
        if (vec) {
          const double2 z = make_double2(0.0, 0.0);
          const double2 x0 = v1 ? __ldg(reinterpret_cast<const double2*>(kr + 16 * g4)) : z;
          const double2 x1 = v1 ? __ldg(reinterpret_cast<const double2*>(kr + 16 * g4 + 2)) : z;
          const double2 y0 = v2 ? __ldg(reinterpret_cast<const double2*>(kr2 + 16 * g4)) : z;
          const double2 y1 = v2 ? __ldg(reinterpret_cast<const double2*>(kr2 + 16 * g4 + 2)) : z;
          b[0] = x0.x; b[1] = x0.y; b[2] = x1.x; b[3] = x1.y;
          b2[0] = y0.x; b2[1] = y0.y; b2[2] = y1.x; b2[3] = y1.y;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            b[e] = v1 ? __ldg(kr + 16 * g4 + e) : 0.0;
            b2[e] = v2 ? __ldg(kr2 + 16 * g4 + e) : 0.0;
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                       : "+d"(c0), "+d"(c1)
                       : "d"(afrag[4 * g4 + e]), "d"(b[e]));
          if (two)
            asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                         : "+d"(c2), "+d"(c3)
                         : "d"(afrag[4 * g4 + e]), "d"(b2[e]));
        }
      }
      if (gid < nrows) {
        const int key0 = jt * 8 + 2 * tig;
        if (key0 < nb) prow[gid * nb + key0] = c0 * scale;
        if (key0 + 1 < nb) prow[gid * nb + key0 + 1] = c1 * scale;
        const int key1 = jt2 * 8 + 2 * tig;
        if (two && key1 < nb) prow[gid * nb + key1] = c2 * scale;
        if (two && key1 + 1 < nb) prow[gid * nb + key1 + 1] = c3 * scale;
      }
    }
  }
  __syncthreads();

  const bool keep_all = thr >= 1.0;
  const bool keep_none = thr <= 0.0;
  const uint32_t lt_mask = (1u << lane) - 1u;

  for (int r = warp; r < nrows; r += kWarps) {
    double* row = prow + r * nb;
    const int i = rows_s[r];
    // ---- row softmax (fp64) -------------------------------------------------------------
    double m = -INFINITY;
    for (int j = lane; j < nb; j += 32) m = fmax(m, row[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    double ssum = 0.0;
    for (int j = lane; j < nb; j += 32) {
      const double e = exp(row[j] - m);
      row[j] = e;
      ssum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
    for (int j = lane; j < nb; j += 32) row[j] = row[j] / ssum;
    __syncwarp();

    // ---- the cut: a bracket of fp64 bit patterns, then the last few candidates ----------
    // Non-negative doubles order like their bit patterns.  The keep rule (keep j iff the
    // mass ranked strictly above it is < thr; rank by P descending, index ascending) keeps
    // every block with key >= hi and drops every block with key < lo, for any lo < hi with
    // mass(P >= lo) >= thr > mass(P >= hi).  The search narrows [lo, hi) until it holds
    // at most kCand blocks (or a single key, all ties); those candidates are ranked and
    // walked in order from mass(P >= hi).  Masses are summed per lane in index order, then
    // by a fixed butterfly: deterministic, fp64-accurate.
    // mode 0: keep all.  mode 1: candidates in [lo, hi) decided by cand_keep.  mode 2:
    // [lo, hi) is the single key lo, the first `tie_keep` of its blocks (by index) kept.
    unsigned long long klo = 0, khi = 0;
    int mode = 0;
    int tie_keep = 0;
    int ncand = 0;
    if (!keep_all && !keep_none) {
      auto mass_cnt_ge = [&](unsigned long long kk, int* cnt) {
        double acc = 0.0;
        int c = 0;
        for (int j = lane; j < nb; j += 32) {
          const double pj = row[j];
          if (static_cast<unsigned long long>(__double_as_longlong(pj)) >= kk) {
            acc += pj;
            ++c;
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        *cnt = __reduce_add_sync(0xffffffffu, c);
        return acc;
      };
      // Bracket: first guess one sixteenth of the row maximum; below it, the lower end
      // from mass(P >= x) >= 1 - nb x; then probes interpolated linearly in the key, each
      // kept within the middle half of the bracket.  The computed mass is monotone in
      // the key, so every bracket that satisfies the invariant leads to the same walk.
      double pm = 0.0;
      for (int j = lane; j < nb; j += 32) pm = fmax(pm, row[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) pm = fmax(pm, __shfl_xor_sync(0xffffffffu, pm, o));
      constexpr unsigned long long kSixteenth = 4ull << 52;   // 2^-4 in the exponent field
      const unsigned long long kpm = static_cast<unsigned long long>(__double_as_longlong(pm));
      const unsigned long long guess = kpm > kSixteenth ? kpm - kSixteenth : 0ull;
      int clo = 0, chi = 0;
      unsigned long long lo, hi;
      double mlo, mhi;
      bool bracket = true;
      const double mg = mass_cnt_ge(guess, &clo);
      if (mg >= thr) {
        lo = guess;
        mlo = mg;
        hi = 0x3FF0000000000001ull;                 // just above 1.0
        mhi = 0.0;
        chi = 0;
      } else {
        hi = guess;
        mhi = mg;
        chi = clo;
        lo = static_cast<unsigned long long>(__double_as_longlong(0.5 * (1.0 - thr) / nb));
        mlo = mass_cnt_ge(lo, &clo);
        if (!(mlo >= thr)) {
          lo = 0ull;
          mlo = mass_cnt_ge(0ull, &clo);
          bracket = mlo >= thr;
        }
      }
      if (bracket) {
        while (clo - chi > kCand && hi - lo > 1ull) {
          const unsigned long long w = hi - lo;
          const double f = fmin(fmax((mlo - thr) / (mlo - mhi), 0.25), 0.75);
          unsigned long long step = static_cast<unsigned long long>(static_cast<double>(w) * f);
          step = step < 1ull ? 1ull : (step > w - 1ull ? w - 1ull : step);
          const unsigned long long mid = lo + step;
          int cm = 0;
          const double mm = mass_cnt_ge(mid, &cm);
          if (mm >= thr) {
            lo = mid;
            clo = cm;
            mlo = mm;
          } else {
            hi = mid;
            chi = cm;
            mhi = mm;
          }
        }
        const double mass_hi = mhi;
        klo = lo;
        khi = hi;
        if (clo - chi <= kCand) {
          // gather the candidates (index order), rank them, walk them
          mode = 1;
          unsigned long long* ck = cand_key + warp * kCand;
          int* ci = cand_idx + warp * kCand;
          for (int j0 = 0; j0 < nb; j0 += 32) {
            const int j = j0 + lane;
            unsigned long long key = 0;
            bool in = false;
            if (j < nb) {
              key = static_cast<unsigned long long>(__double_as_longlong(row[j]));
              in = key >= lo && key < hi;
            }
            const uint32_t bal = __ballot_sync(0xffffffffu, in);
            if (in) {
              const int pos = ncand + __popc(bal & lt_mask);
              ck[pos] = key;
              ci[pos] = j;
            }
            ncand += __popc(bal);
          }
          __syncwarp();
          // rank by (key descending, index ascending); E of a candidate = mass above hi +
          // the candidates ranked before it
          int* cr = cand_keep + warp * kCand;      // ranks first, then the decisions
          int rank = 0;
          if (lane < ncand) {
            const unsigned long long kc = ck[lane];
            const int ic = ci[lane];
            for (int d = 0; d < ncand; ++d) rank += (ck[d] > kc || (ck[d] == kc && ci[d] < ic)) ? 1 : 0;
            cr[lane] = rank;
          }
          __syncwarp();
          double e = mass_hi;
          if (lane < ncand)
            for (int d = 0; d < ncand; ++d)
              if (cr[d] < rank) e += __longlong_as_double(static_cast<long long>(ck[d]));
          __syncwarp();
          if (lane < ncand) cr[lane] = e < thr ? 1 : 0;
          __syncwarp();
        } else {
          // a single key holding more than kCand blocks: ties, ranked by index; the r-th
          // has ranked mass mass_hi + r * p
          mode = 2;
          const double pt = __longlong_as_double(static_cast<long long>(lo));
          const int n_at = clo - chi;
          int r = 0;
          while (r < n_at && mass_hi + r * pt < thr) ++r;
          tie_keep = r;
        }
      }
    }

    // ---- emit bitmask words and the ascending row list ---------------------------------
    const int ti = i / (Hb * Wb);
    const int hi = (i / Wb) % Hb;
    const int wi = i % Wb;
    int run = 0;
    int tie_seen = 0;
    for (int w = 0; w < nw; ++w) {
      const int j = w * 32 + lane;
      bool k = false;
      bool is_tie = false;
      if (j < nb) {
        const unsigned long long key = static_cast<unsigned long long>(__double_as_longlong(row[j]));
        if (keep_all) k = true;
        else if (keep_none) k = false;
        else if (mode == 0) k = true;
        else if (key >= khi) k = true;
        else if (key < klo) k = false;
        else if (mode == 2) is_tie = true;
        else {
          for (int d = 0; d < ncand; ++d)
            if (cand_idx[warp * kCand + d] == j) k = cand_keep[warp * kCand + d] != 0;
        }
      }
      const uint32_t tb = __ballot_sync(0xffffffffu, is_tie);
      if (is_tie) k = (tie_seen + __popc(tb & lt_mask)) < tie_keep;
      tie_seen += __popc(tb);
      if (sta_on && j < nb) {
        const int tj = j / (Hb * Wb);
        const int hj = (j / Wb) % Hb;
        const int wj = j % Wb;
        k = k || (abs(ti - tj) <= wt2 && abs(hi - hj) <= wh2 && abs(wi - wj) <= ww2);
      }
      const uint32_t kb = __ballot_sync(0xffffffffu, k);
      if (lane == 0) bits[(bh * nb + i) * nw + w] = kb;
      if (row_idx != nullptr && k) row_idx[(bh * nb + i) * nb + run + __popc(kb & lt_mask)] = j;
      run += __popc(kb);
    }
    if (row_cnt != nullptr && lane == 0) row_cnt[bh * nb + i] = run;
    __syncwarp();
  }
  }  // row groups
}

// Column lists (transpose of the bitmask): one warp per 32-column word of one head.
__global__ void __launch_bounds__(32) col_lists_kernel(const uint32_t* __restrict__ bits, int nb,
                                                       int nw, int32_t* __restrict__ col_idx,
                                                       int32_t* __restrict__ col_cnt) {
  const int w = blockIdx.x;
  const long long bh = blockIdx.y;
  const int lane = threadIdx.x;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int mycnt = 0;
  for (int i0 = 0; i0 < nb; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t word = (i < nb) ? bits[(bh * nb + i) * nw + w] : 0u;
#pragma unroll 4
    for (int c = 0; c < 32; ++c) {
      const bool set = (word >> c) & 1u;
      const uint32_t b = __ballot_sync(0xffffffffu, set);
      const int base = __shfl_sync(0xffffffffu, mycnt, c);
      const int col = 32 * w + c;
      if (set && col < nb && col_idx != nullptr) col_idx[(bh * nb + col) * nb + base + __popc(b & lt_mask)] = i;
      if (lane == c) mycnt += __popc(b);
    }
  }
  if (32 * w + lane < nb) col_cnt[bh * nb + 32 * w + lane] = mycnt;
}

// Masks that do not depend on the data: thr >= 1 keeps every block; thr <= 0 keeps none,
// which leaves the static window alone ([ZH-TS] "hybrid integration with STA": the union
// with an empty NABLA mask is the STA mask).  One warp per row, one ballot per word.
__global__ void __launch_bounds__(256) static_mask_kernel(int nb, int nw, long long rows, int keep_all,
                                                          int sta_on, int wt2, int wh2, int ww2,
                                                          int Hb, int Wb, uint32_t* __restrict__ bits) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int i = static_cast<int>(row % nb);
  const int ti = i / (Hb * Wb), hi = (i / Wb) % Hb, wi = i % Wb;
  for (int w = 0; w < nw; ++w) {
    const int j = 32 * w + lane;
    bool k = false;
    if (j < nb) {
      if (keep_all) {
        k = true;
      } else if (sta_on) {
        const int tj = j / (Hb * Wb), hj = (j / Wb) % Hb, wj = j % Wb;
        k = abs(ti - tj) <= wt2 && abs(hi - hj) <= wh2 && abs(wi - wj) <= ww2;
      }
    }
    const uint32_t kb = __ballot_sync(0xffffffffu, k);
    if (lane == 0) bits[row * nw + w] = kb;
  }
}

// Row lists from a bitmask: one warp per row.
__global__ void __launch_bounds__(256) row_lists_kernel(const uint32_t* __restrict__ bits, int nb,
                                                        int nw, long long rows,
                                                        int32_t* __restrict__ row_idx,
                                                        int32_t* __restrict__ row_cnt) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  int run = 0;
  for (int w0 = 0; w0 < nw; w0 += 32) {
    const int w = w0 + lane;
    uint32_t word = (w < nw) ? bits[row * nw + w] : 0u;
    if (w == nw - 1 && (nb & 31)) word &= (1u << (nb & 31)) - 1u;
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int pos = run + incl - c;
    while (word) {
      const int b = __ffs(word) - 1;
      if (row_idx != nullptr) row_idx[row * nb + pos] = 32 * w + b;
      ++pos;
      word &= word - 1u;
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) row_cnt[row] = run;
}

int rows_per_cta(int nb) {
  int r = kRowBudget / (nb * 8);
  return r < 1 ? 1 : (r > 8 ? 8 : r);
}

size_t mask_rows_smem(int nb, int D, int R) {
  return static_cast<size_t>(8) * D * 8 + static_cast<size_t>(R) * nb * 8;
}

template <int D>
cudaError_t launch_mask_rows(const double* qp, const double* kp, const Dims& d, double scale,
                             double thr, const nabla_window& w, uint32_t* bits, int32_t* ridx,
                             int32_t* rcnt, const int32_t* rlist, const int32_t* rlist_cnt,
                             cudaStream_t st) {
  const int R = rows_per_cta(d.nb);
  const size_t smem = mask_rows_smem(d.nb, D, R);
  cudaError_t e = cudaFuncSetAttribute(mask_rows_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int sta_on = (w.t | w.h | w.w) != 0;
  // Listed rows: as many CTAs as fit on the GPU at once walk the groups of every head
  // (the counts are on the device); all rows: one CTA per group of R rows of each head.
  int dev = 0, sms = 148, per_sm = 1;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (rlist != nullptr &&
      (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mask_rows_kernel<D>, kThreads, smem) != cudaSuccess ||
       per_sm < 1))
    per_sm = 1;
  dim3 grid(rlist != nullptr ? sms * per_sm : (d.nb + R - 1) / R, rlist != nullptr ? 1 : d.BH);
  mask_rows_kernel<D><<<grid, kThreads, smem, st>>>(qp, kp, d.nb, d.nw, R, scale, thr, sta_on,
                                                   w.t / 2, w.h / 2, w.w / 2, d.Hb, d.Wb, bits,
                                                   ridx, rcnt, rlist, rlist_cnt, d.BH);
  return cudaGetLastError();
}

// A list needs its counts; counts may come without the list.
nabla_status check_lists(const int32_t* idx, const int32_t* cnt) {
  if (idx != nullptr && cnt == nullptr) return NABLA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(idx) & 3) || (reinterpret_cast<uintptr_t>(cnt) & 3))
    return NABLA_ERR_INVALID_ARG;
  return NABLA_OK;
}

cudaError_t launch_col_lists(const uint32_t* bits, const Dims& d, int32_t* cidx, int32_t* ccnt,
                             cudaStream_t st) {
  dim3 grid(d.nw, d.BH);
  col_lists_kernel<<<grid, 32, 0, st>>>(bits, d.nb, d.nw, cidx, ccnt);
  return cudaGetLastError();
}

}  // namespace
}  // namespace nabla

using namespace nabla;

constexpr int kMaxSweep = 64;   // thresholds per nabla_build_mask_sweep call

extern "C" size_t nabla_mask_workspace_bytes(nabla_shape s) {
  Dims d;
  if (check_shape(s, &d) != NABLA_OK) return 0;
  const size_t pool = align_up(static_cast<size_t>(d.BH) * d.nb * d.D * sizeof(double), 256);
  return kStatusBytes + 2 * pool + (mask_fast_supported(d) ? mask_fast_scratch_bytes(d) : 0);
}

extern "C" nabla_status nabla_build_mask(const void* q, const void* k, const double* q_pool,
                                         const double* k_pool, nabla_shape s, double thr,
                                         nabla_window sta, double scale, uint32_t* mask_bits,
                                         int32_t* row_idx, int32_t* row_cnt, int32_t* col_idx,
                                         int32_t* col_cnt, nabla_layout layout, void* workspace,
                                         size_t workspace_bytes, nabla_stream_t stream) {
  Dims d;
  nabla_status rc = check_shape(s, &d);
  if (rc != NABLA_OK) return rc;
  if (layout != NABLA_LAYOUT_REORDERED && layout != NABLA_LAYOUT_NATURAL) return NABLA_ERR_INVALID_ARG;
  const bool natural = layout == NABLA_LAYOUT_NATURAL;
  if (!(thr >= 0.0 && thr <= 1.0)) return NABLA_ERR_INVALID_ARG;   // also rejects NaN
  if (!(scale > 0.0) || !isfinite(scale)) return NABLA_ERR_INVALID_ARG;
  const int sizes[3] = {sta.t, sta.h, sta.w};
  const bool sta_off = sta.t == 0 && sta.h == 0 && sta.w == 0;
  if (!sta_off)
    for (int a = 0; a < 3; ++a)
      if (sizes[a] < 1 || (sizes[a] % 2) == 0) return NABLA_ERR_INVALID_ARG;
  if (!mask_bits || (reinterpret_cast<uintptr_t>(mask_bits) & 3)) return NABLA_ERR_INVALID_ARG;
  if ((rc = check_lists(row_idx, row_cnt)) != NABLA_OK) return rc;
  if ((rc = check_lists(col_idx, col_cnt)) != NABLA_OK) return rc;
  const bool data_free = thr <= 0.0 || thr >= 1.0;   // the mask ignores Q and K
  if (data_free) {
    const size_t need0 = nabla_mask_workspace_bytes(s);
    if (!workspace || workspace_bytes < need0 || (reinterpret_cast<uintptr_t>(workspace) & 255))
      return NABLA_ERR_WORKSPACE;
    cudaStream_t st0 = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, kStatusBytes, st0) != cudaSuccess) return NABLA_ERR_CUDA;
    const long long rows = static_cast<long long>(d.BH) * d.nb;
    static_mask_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st0>>>(
        d.nb, d.nw, rows, thr >= 1.0 ? 1 : 0, sta_off ? 0 : 1, sta.t / 2, sta.h / 2, sta.w / 2,
        d.Hb, d.Wb, mask_bits);
    cudaError_t e0 = cudaGetLastError();
    if (e0 == cudaSuccess && row_cnt)
      row_lists_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st0>>>(mask_bits, d.nb, d.nw,
                                                                              rows, row_idx, row_cnt);
    if (e0 == cudaSuccess) e0 = cudaGetLastError();
    if (e0 == cudaSuccess && col_cnt) e0 = launch_col_lists(mask_bits, d, col_idx, col_cnt, st0);
    return cuda_status(e0);
  }
  if (!q_pool && (!q || !aligned16(q))) return NABLA_ERR_INVALID_ARG;
  if (!k_pool && (!k || !aligned16(k))) return NABLA_ERR_INVALID_ARG;
  if ((q_pool && (reinterpret_cast<uintptr_t>(q_pool) & 7)) ||
      (k_pool && (reinterpret_cast<uintptr_t>(k_pool) & 7)))
    return NABLA_ERR_INVALID_ARG;
  const size_t need = nabla_mask_workspace_bytes(s);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return NABLA_ERR_WORKSPACE;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t pool_bytes = align_up(static_cast<size_t>(d.BH) * d.nb * d.D * sizeof(double), 256);
  if (cudaMemsetAsync(workspace, 0, kStatusBytes, st) != cudaSuccess) return NABLA_ERR_CUDA;
  double* qp_ws = reinterpret_cast<double*>(static_cast<char*>(workspace) + kStatusBytes);
  double* kp_ws = reinterpret_cast<double*>(static_cast<char*>(workspace) + kStatusBytes + pool_bytes);
  cudaError_t e = cudaSuccess;
  const double* qp = q_pool;
  const double* kp = k_pool;
  void* fast_scratch = static_cast<char*>(workspace) + kStatusBytes + 2 * pool_bytes;
  // Fast tier (tensor-core logits, certified fp32 cut) for every row, then the fp64
  // kernel for the rows it could not certify.  Without the fast tier: fp64 for all rows.
  // Given Q and K but no pools, the fast tier pools them itself together with the fp16
  // split of the means (one pass over each tensor).
  const int32_t* rlist = nullptr;
  const int32_t* rlist_cnt = nullptr;
  if (mask_fast_supported(d)) {
    if (!qp && !kp) {
      e = mask_fast_prepare_tokens(q, k, natural, qp_ws, kp_ws, d, scale, fast_scratch,
                                   static_cast<uint32_t*>(workspace), st);
      qp = qp_ws;
      kp = kp_ws;
    } else {
      if (!qp && (e = pool_blocks_device(q, qp_ws, d, st, natural)) == cudaSuccess) qp = qp_ws;
      if (e == cudaSuccess && !kp && (e = pool_blocks_device(k, kp_ws, d, st, natural)) == cudaSuccess) kp = kp_ws;
      if (e == cudaSuccess)
        e = mask_fast_prepare(qp, kp, d, scale, fast_scratch, static_cast<uint32_t*>(workspace), st);
    }
    if (e != cudaSuccess) return cuda_status(e);
    int32_t* rl = nullptr;
    int32_t* rc = nullptr;
    e = mask_fast_select(d, scale, thr, sta, mask_bits, row_idx, row_cnt, fast_scratch, &rl, &rc, st);
    if (e != cudaSuccess) return cuda_status(e);
    rlist = rl;
    rlist_cnt = rc;
  } else {
    if (!qp && (e = pool_blocks_device(q, qp_ws, d, st, natural)) == cudaSuccess) qp = qp_ws;
    if (e == cudaSuccess && !kp && (e = pool_blocks_device(k, kp_ws, d, st, natural)) == cudaSuccess) kp = kp_ws;
    if (e != cudaSuccess) return cuda_status(e);
  }
  e = d.D == 64 ? launch_mask_rows<64>(qp, kp, d, scale, thr, sta, mask_bits, row_idx, row_cnt,
                                       rlist, rlist_cnt, st)
                : launch_mask_rows<128>(qp, kp, d, scale, thr, sta, mask_bits, row_idx, row_cnt,
                                        rlist, rlist_cnt, st);
  if (e != cudaSuccess) return cuda_status(e);
  if (col_cnt) {
    if ((e = launch_col_lists(mask_bits, d, col_idx, col_cnt, st)) != cudaSuccess) return cuda_status(e);
  }
  return NABLA_OK;
}

extern "C" nabla_status nabla_mask_lists(const uint32_t* mask_bits, nabla_shape s, int32_t* row_idx,
                                         int32_t* row_cnt, int32_t* col_idx, int32_t* col_cnt,
                                         nabla_stream_t stream) {
  Dims d;
  nabla_status rc = check_shape(s, &d);
  if (rc != NABLA_OK) return rc;
  if (!mask_bits || (reinterpret_cast<uintptr_t>(mask_bits) & 3)) return NABLA_ERR_INVALID_ARG;
  if ((rc = check_lists(row_idx, row_cnt)) != NABLA_OK) return rc;
  if ((rc = check_lists(col_idx, col_cnt)) != NABLA_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (row_cnt) {
    const long long rows = static_cast<long long>(d.BH) * d.nb;
    row_lists_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(mask_bits, d.nb, d.nw,
                                                                          rows, row_idx, row_cnt);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
  }
  if (col_cnt) {
    if ((e = launch_col_lists(mask_bits, d, col_idx, col_cnt, st)) != cudaSuccess) return cuda_status(e);
  }
  return NABLA_OK;
}

// Several thresholds on one pooled map: the pooled means and the pooled logits are
// formed once, then the cut (and the fp64 rescue of the rows it cannot certify) runs per
// threshold.  Mask t goes to mask_bits + t * (B*H*nb*nw), its per-row counts (optional)
// to row_cnt + t * (B*H*nb).
extern "C" nabla_status nabla_build_mask_sweep(const void* q, const void* k, const double* q_pool,
                                               const double* k_pool, nabla_shape s,
                                               const double* thrs, int n_thr, nabla_window sta,
                                               double scale, uint32_t* mask_bits, int32_t* row_cnt,
                                               void* workspace, size_t workspace_bytes,
                                               nabla_stream_t stream) {
  Dims d;
  nabla_status rc = check_shape(s, &d);
  if (rc != NABLA_OK) return rc;
  if (!thrs || n_thr < 1 || n_thr > kMaxSweep) return NABLA_ERR_INVALID_ARG;
  bool any_data = false;
  for (int t = 0; t < n_thr; ++t) {
    if (!(thrs[t] >= 0.0 && thrs[t] <= 1.0)) return NABLA_ERR_INVALID_ARG;   // also NaN
    any_data = any_data || (thrs[t] > 0.0 && thrs[t] < 1.0);
  }
  if (!(scale > 0.0) || !isfinite(scale)) return NABLA_ERR_INVALID_ARG;
  const int sizes[3] = {sta.t, sta.h, sta.w};
  const bool sta_off = sta.t == 0 && sta.h == 0 && sta.w == 0;
  if (!sta_off)
    for (int a = 0; a < 3; ++a)
      if (sizes[a] < 1 || (sizes[a] % 2) == 0) return NABLA_ERR_INVALID_ARG;
  if (!mask_bits || (reinterpret_cast<uintptr_t>(mask_bits) & 3)) return NABLA_ERR_INVALID_ARG;
  if (row_cnt && (reinterpret_cast<uintptr_t>(row_cnt) & 3)) return NABLA_ERR_INVALID_ARG;
  if (any_data) {
    if (!q_pool && (!q || !aligned16(q))) return NABLA_ERR_INVALID_ARG;
    if (!k_pool && (!k || !aligned16(k))) return NABLA_ERR_INVALID_ARG;
    if ((q_pool && (reinterpret_cast<uintptr_t>(q_pool) & 7)) ||
        (k_pool && (reinterpret_cast<uintptr_t>(k_pool) & 7)))
      return NABLA_ERR_INVALID_ARG;
  }
  const size_t need = nabla_mask_workspace_bytes(s);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return NABLA_ERR_WORKSPACE;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long rows = static_cast<long long>(d.BH) * d.nb;
  const size_t mask_words = static_cast<size_t>(rows) * d.nw;
  const size_t pool_bytes = align_up(static_cast<size_t>(d.BH) * d.nb * d.D * sizeof(double), 256);
  if (cudaMemsetAsync(workspace, 0, kStatusBytes, st) != cudaSuccess) return NABLA_ERR_CUDA;
  cudaError_t e = cudaSuccess;
  const double* qp = q_pool;
  const double* kp = k_pool;
  void* fast_scratch = static_cast<char*>(workspace) + kStatusBytes + 2 * pool_bytes;
  const bool fast = mask_fast_supported(d);
  if (any_data) {
    double* qp_ws = reinterpret_cast<double*>(static_cast<char*>(workspace) + kStatusBytes);
    double* kp_ws = reinterpret_cast<double*>(static_cast<char*>(workspace) + kStatusBytes + pool_bytes);
    if (!qp) {
      if ((e = pool_blocks_device(q, qp_ws, d, st, false)) != cudaSuccess) return cuda_status(e);
      qp = qp_ws;
    }
    if (!kp) {
      if ((e = pool_blocks_device(k, kp_ws, d, st, false)) != cudaSuccess) return cuda_status(e);
      kp = kp_ws;
    }
    if (fast && (e = mask_fast_prepare(qp, kp, d, scale, fast_scratch, static_cast<uint32_t*>(workspace), st)) !=
                    cudaSuccess)
      return cuda_status(e);
  }
  for (int t = 0; t < n_thr; ++t) {
    const double thr = thrs[t];
    uint32_t* bits = mask_bits + t * mask_words;
    int32_t* cnt = row_cnt ? row_cnt + t * static_cast<size_t>(rows) : nullptr;
    if (thr <= 0.0 || thr >= 1.0) {
      static_mask_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(
          d.nb, d.nw, rows, thr >= 1.0 ? 1 : 0, sta_off ? 0 : 1, sta.t / 2, sta.h / 2, sta.w / 2,
          d.Hb, d.Wb, bits);
      if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
      if (cnt) {
        row_lists_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(bits, d.nb, d.nw, rows,
                                                                              nullptr, cnt);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e);
      }
      continue;
    }
    const int32_t* rlist = nullptr;
    const int32_t* rlist_cnt = nullptr;
    if (fast) {
      int32_t* rl = nullptr;
      int32_t* rcn = nullptr;
      if ((e = mask_fast_select(d, scale, thr, sta, bits, nullptr, cnt, fast_scratch, &rl, &rcn, st)) !=
          cudaSuccess)
        return cuda_status(e);
      rlist = rl;
      rlist_cnt = rcn;
    }
    e = d.D == 64 ? launch_mask_rows<64>(qp, kp, d, scale, thr, sta, bits, nullptr, cnt, rlist, rlist_cnt, st)
                  : launch_mask_rows<128>(qp, kp, d, scale, thr, sta, bits, nullptr, cnt, rlist, rlist_cnt, st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  return NABLA_OK;
}
